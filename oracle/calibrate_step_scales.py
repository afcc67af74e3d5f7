"""Step scales of the synthetic codecs, set on the oracle's own payload (test infrastructure).

The synthetic codec's quantiser steps are Delta_c = k * 0.02 * sigma_c^0.5 (dckv_synth).  The
configurations are stated as rates -- about 220 bytes per coded row (about 55x below bf16's
12,288) and about 110 (about 100x) -- which follow the DCKV summary's claims ("What it claims":
more than 55x and more than 100x fewer bytes).  This script finds k for each rate by bisection on
the payload the oracle actually writes: it draws a calibration sample with dckv_synth (two
4,096-token prompts, seeds 5000 and 5001, which no test or benchmark uses), runs the oracle's
encoder (transform, quantiser, mean models, centres, rANS, container) at a trial k, and measures
the blob's bytes outside the kept bf16 rows per coded row.  The payload falls as k grows, so
bisection on log k converges.  Each entry is keyed by what changes the payload: the target, the
rows per rANS chunk (a chunk's fixed 136 bytes), the share of Student-t rows (their escapes) and
whether the codec is the linear one.

The result is written to dckv_synth/step_scales.json, from which dckv_synth.calibrated_codec reads
k.  Run from the repository root:  python -m oracle.calibrate_step_scales
"""
from __future__ import annotations

import json
import math
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import dckv_synth as S  # noqa: E402
from oracle import codec as O  # noqa: E402

OUT = os.path.join(ROOT, "dckv_synth", "step_scales.json")
SAMPLE_SEEDS = (5000, 5001)
SAMPLE_LEN = 4096

# (target bytes per coded row, rows per chunk, Student-t fraction, linear codec)
ENTRIES = [
    (220.0, 16, 0.0, False),
    (110.0, 32, 0.0, False),
    (220.0, 16, 0.01, False),
    (220.0, 16, 0.0, True),
]


def payload_per_row(src, xb, tok, offs, k, chunk_rows, linear):
    """Oracle payload (blob bytes outside the kept rows) per coded row at step scale k."""
    cod = S.codec(src, step_scale=k, linear=linear)
    blob = O.encode(xb, tok, offs, cod, chunk_rows=chunk_rows)
    lay = O.prompt_layout(np.diff(offs))
    n = sum(L["n"] for L in lay)
    kept = sum(L["N"] - L["n"] for L in lay)
    return (len(blob) - kept * O.ROW_DIM * 2) / n


def calibrate(src, target, chunk_rows, st_frac, linear, iters=11):
    import torch

    x, tok, offs = S.batch(src, [SAMPLE_LEN] * len(SAMPLE_SEEDS), list(SAMPLE_SEEDS), student_t_frac=st_frac)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    tk = tok.numpy()
    k0 = S.codec(src, step_scale=None, target_bytes=target, linear=linear).step_scale
    lo, hi = math.log(k0 / 2.0), math.log(k0 * 2.0)
    f_lo = payload_per_row(src, xb, tk, offs, math.exp(lo), chunk_rows, linear)
    f_hi = payload_per_row(src, xb, tk, offs, math.exp(hi), chunk_rows, linear)
    if not (f_lo > target > f_hi):
        raise RuntimeError(f"target {target} not bracketed: {f_lo:.1f} .. {f_hi:.1f}")
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        f = payload_per_row(src, xb, tk, offs, math.exp(mid), chunk_rows, linear)
        if f > target:
            lo = mid
        else:
            hi = mid
    k = float(np.float32(math.exp(0.5 * (lo + hi))))
    return k, payload_per_row(src, xb, tk, offs, k, chunk_rows, linear), k0


def main():
    src = S.source(0)
    out = {"sample": f"{len(SAMPLE_SEEDS)} prompts of {SAMPLE_LEN} tokens, seeds {list(SAMPLE_SEEDS)}, source seed 0",
           "quantity": "oracle blob bytes outside the kept rows, per coded row",
           "entries": []}
    for target, g, st, lin in ENTRIES:
        t0 = time.time()
        k, got, k0 = calibrate(src, target, g, st, lin)
        out["entries"].append(dict(target_bytes=target, chunk_rows=g, student_t_frac=st, linear=lin,
                                   step_scale=k, payload_per_row=round(got, 3), gaussian_estimate_k=k0))
        print(f"target {target} G {g} t {st} linear {lin}: k = {k:.6f} (Gaussian estimate {k0:.4f}), "
              f"payload {got:.2f} B/row, {time.time() - t0:.0f} s", flush=True)
    with open(OUT, "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()

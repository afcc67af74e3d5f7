"""Step-by-step fp64 definition of the DCKV codec (oracle; test infrastructure only).

Pages cited (all from "DCKV: Learned Transform Coding of the Prompt KV Cache in Hybrid
Language Models", trove.briskstack.com summary, section "How it works"):
  [rows]   first paragraph: 6 full-attention layers, 12,288 B/token bf16, first 4 and
           last 128 positions kept bf16, pre-RoPE keys and values of all six layers
           stacked into one 6,144-dim row, RoPE reapplied after decoding;
  [xform]  bullet "Transform": one shared basis, 6,144 -> 2,048 coefficients, PCA start
           plus one hidden layer of 256 GELU units; components whose scale is below
           0.05 quantisation steps are dropped;
  [code]   bullet "Coding": rANS under Laplace distributions; codes beyond +-127 are
           escaped at 64 bits each;
  [cond]   bullet "Conditional entropy models": even positions predict code means from
           the prompt token's input embedding, odd positions also from the decoded
           coefficients of both neighbours (1-D checkerboard, two parallel passes);
  [steps]  section "What it claims": per-component quantisation steps.
The coder constants (32 interleaved 32-bit states, 16-bit renormalisation, 16-bit
frequency precision, scale index clamp(round(8 log2(b/b0)), 0, 63), residual
q - round(mu), RoPE base 1e7 over all 256 dims) are part of the codec specification.
"""
from __future__ import annotations

import ctypes
import math
import os
import struct
import subprocess

import numpy as np
from scipy.special import erf

__all__ = [
    "ROW_DIM", "N_COEF", "N_HIDDEN", "HEAD_KEPT", "TAIL_KEPT", "ESC_LIMIT", "ESC_SYMBOL",
    "N_SYMBOLS", "PREC_TOTAL", "LANES", "B0_STEPS", "N_SCALES", "ROPE_BASE", "MAGIC",
    "VERSION", "HEADER_BYTES", "DEFAULT_CHUNK_ROWS",
    "bf16_to_f64", "f64_to_bf16", "gelu", "transform", "scale_index", "quantise",
    "laplace_tables", "prompt_layout", "chunk_list", "mean_even", "mean_odd", "codec_means_even",
    "codec_means_odd", "centres",
    "symbols", "rans_encode", "rans_decode", "encode", "decode", "parse_blob", "analyse",
    "assemble_blob",
    "byte_report", "model_code_length_bits", "rope", "reconstruct", "kept_positions",
    "output_rows",
]

ROW_DIM = 6144
N_COEF = 2048
N_HIDDEN = 256
N_LAYERS = 6
N_KV_HEADS = 2
HEAD_DIM = 256
HEAD_KEPT = 4
TAIL_KEPT = 128
ESC_LIMIT = 127
R_MAX = 2 * ESC_LIMIT  # residual q - centre in [-254, 254]
N_SYMBOLS = 2 * R_MAX + 2  # 509 residuals + ESC
ESC_SYMBOL = N_SYMBOLS - 1
PREC_BITS = 16
PREC_TOTAL = 1 << PREC_BITS
LANES = 32
RANS_L = 1 << 16
B0_STEPS = 0.05
N_SCALES = 64
ROPE_BASE = 1.0e7
MAGIC = 0x564B4344  # "DCKV"
VERSION = 1
HEADER_BYTES = 64
DEFAULT_CHUNK_ROWS = 32
INT32_MIN, INT32_MAX = -(2 ** 31), 2 ** 31 - 1


# ----------------------------------------------------------------------------------------
# number formats
# ----------------------------------------------------------------------------------------
def bf16_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> fp64 values (exact)."""
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16))
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16(v) -> np.ndarray:
    """fp64 -> bf16 bits, one round-to-nearest-even step straight from fp64.

    The 52-bit fp64 fraction is cut to bf16's 7 bits; values must be finite and inside
    the normal bf16 range (true for every row this codec produces)."""
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float64))
    u = v.view(np.uint64)
    keep = u >> np.uint64(45)
    rem = u & np.uint64((1 << 45) - 1)
    half = np.uint64(1 << 44)
    up = (rem > half) | ((rem == half) & ((keep & np.uint64(1)) == np.uint64(1)))
    keep = keep + up.astype(np.uint64)
    r = (keep << np.uint64(45)).view(np.float64)
    r32 = r.astype(np.float32)  # exact: r has at most 8 significant bits
    out = (r32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    zero = v == 0.0
    out[zero] = np.where(np.signbit(v[zero]), 0x8000, 0).astype(np.uint16)
    return out


def _as_f64_rows(x) -> np.ndarray:
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return bf16_to_f64(x)
    return x.astype(np.float64)


# ----------------------------------------------------------------------------------------
# transform and quantiser  [xform], [steps]
# ----------------------------------------------------------------------------------------
def gelu(h):
    """GELU, exact erf form (the pages name GELU without a variant; reading: erf form)."""
    h = np.asarray(h, dtype=np.float64)
    return 0.5 * h * (1.0 + erf(h / math.sqrt(2.0)))


def transform(x, codec) -> np.ndarray:
    """y = (x - mu) B + GELU((x - mu) W1) W2  [xform].

    B is the shared 6,144 x 2,048 basis, W1 (6,144 x 256) and W2 (256 x 2,048) the
    one-hidden-layer correction; no biases (reading).  fp64 throughout.  A codec without
    W1 / W2 is the linear codec the pages compare DCKV with ("Evidence": payload 5% above
    its models' code length, 96 MiB of weights): y = (x - mu) B."""
    xc = _as_f64_rows(x) - np.asarray(codec.mu, np.float64)[None, :]
    lin = xc @ np.asarray(codec.basis, np.float64)
    if codec.w1 is None or codec.w2 is None:
        return lin
    hid = gelu(xc @ np.asarray(codec.w1, np.float64))
    return lin + hid @ np.asarray(codec.w2, np.float64)


def scale_index(laplace_b, delta):
    """Per-component table index and drop mask  [xform], [code].

    beta_c = b_c / Delta_c is the Laplace scale in quantisation steps; components with
    beta_c < 0.05 steps are dropped; s_c = clamp(round(8 log2(beta_c / b0)), 0, 63) with
    b0 = 0.05 steps (reading: b0 is the drop threshold, so s = 0 is the smallest coded
    scale).  Returns (s int64 [2048], keep bool [2048]); s is 0 for dropped components."""
    beta = np.asarray(laplace_b, np.float64) / np.asarray(delta, np.float64)
    keep = beta >= B0_STEPS
    s = np.zeros(beta.shape, np.int64)
    s[keep] = np.clip(np.rint(8.0 * np.log2(beta[keep] / B0_STEPS)), 0, N_SCALES - 1).astype(np.int64)
    return s, keep


def quantise(y, delta, keep):
    """q_c = round(y_c / Delta_c), ties to even; dropped components are 0  [steps].

    Returns (q int64, ratio fp64 = y / Delta) -- the ratio is what the parity rule's
    half-step test looks at.  Codes saturate to the int32 range."""
    ratio = np.asarray(y, np.float64) / np.asarray(delta, np.float64)[None, :]
    q = np.clip(np.rint(ratio), INT32_MIN, INT32_MAX).astype(np.int64)
    q[:, ~np.asarray(keep, bool)] = 0
    return q, ratio


# ----------------------------------------------------------------------------------------
# entropy model  [code], [cond]
# ----------------------------------------------------------------------------------------
def laplace_tables():
    """Integer frequency tables, one row per scale index s  [code].

    beta_s = 0.05 * 2^(s/8) steps.  For residual r in [-254, 254] (symbol r + 254):
    p(r) = mass of Laplace(0, beta_s) on [r - 1/2, r + 1/2]; ESC (symbol 509) gets the
    mass beyond +-254.5.  freq = 1 + floor(p * (2^16 - 510)); what is left of 2^16 goes
    to r = 0.  cdf runs in symbol order (cdf[0] = 0, cdf[510] = 2^16).
    Returns freq uint32 [64, 510], cdf uint32 [64, 511]."""
    freq = np.zeros((N_SCALES, N_SYMBOLS), np.int64)
    r = np.arange(-R_MAX, R_MAX + 1, dtype=np.float64)
    ar = np.abs(r)
    for s in range(N_SCALES):
        beta = B0_STEPS * 2.0 ** (s / 8.0)
        p = np.where(ar == 0, -np.expm1(-0.5 / beta),
                     0.5 * np.exp(-(ar - 0.5) / beta) * -np.expm1(-1.0 / beta))
        p_esc = np.exp(-(R_MAX + 0.5) / beta)
        f = 1 + np.floor(np.append(p, p_esc) * (PREC_TOTAL - N_SYMBOLS)).astype(np.int64)
        f[R_MAX] += PREC_TOTAL - f.sum()
        freq[s] = f
    cdf = np.zeros((N_SCALES, N_SYMBOLS + 1), np.int64)
    cdf[:, 1:] = np.cumsum(freq, axis=1)
    return freq.astype(np.uint32), cdf.astype(np.uint32)


def mean_even(embed_rows_bits, w_even_bits) -> np.ndarray:
    """Even-position code means: mu = e(token) W_e, in code units  [cond]."""
    return bf16_to_f64(embed_rows_bits) @ bf16_to_f64(w_even_bits)


def codec_means_even(codec, toks) -> np.ndarray:
    """Even-position means of a codec; a codec without mean models (the linear codec's
    unconditional zero-mean tables, "Evidence") gives zeros."""
    if codec.embed is None:
        return np.zeros((len(toks), N_COEF))
    return mean_even(codec.embed[toks], codec.w_even)


def codec_means_odd(codec, toks, q_left, q_right) -> np.ndarray:
    """Odd-position means of a codec (zeros without mean models, as above)."""
    if codec.embed is None:
        return np.zeros((len(toks), N_COEF))
    return mean_odd(codec.embed[toks], q_left, q_right, codec.w_odd)


def mean_odd(embed_rows_bits, q_left, q_right, w_odd_bits) -> np.ndarray:
    """Odd-position code means: mu = [e(token), bf16(q_left), bf16(q_right)] W_o  [cond].

    The neighbours' decoded coefficients enter as bf16(q) against weights that carry the
    step Delta_c (reading: a reparametrisation of 'linear on the decoded coefficients
    q * Delta'); a missing right neighbour is a zero vector (reading)."""
    def q_bf16(q):
        return bf16_to_f64(f64_to_bf16(np.asarray(q, np.float32).astype(np.float64)))

    inp = np.concatenate([bf16_to_f64(embed_rows_bits), q_bf16(q_left), q_bf16(q_right)], axis=1)
    return inp @ bf16_to_f64(w_odd_bits)


def centres(mu) -> np.ndarray:
    """centre = clamp(round(mu), -127, 127) (ties to even)  [code], [cond]."""
    return np.clip(np.rint(np.asarray(mu, np.float64)), -ESC_LIMIT, ESC_LIMIT).astype(np.int64)


def symbols(q, centre, keep):
    """Symbols of the kept components, row-major: ESC if |q| > 127 else q - centre + 254.

    Returns (sym int64 [rows, K_eff], esc_mask bool [rows, K_eff])  [code]."""
    qk = np.asarray(q)[:, keep]
    ck = np.asarray(centre)[:, keep]
    esc = np.abs(qk) > ESC_LIMIT
    sym = np.where(esc, ESC_SYMBOL, qk - ck + R_MAX)
    return sym.astype(np.int64), esc


# ----------------------------------------------------------------------------------------
# rows and chunks  [rows], [cond]
# ----------------------------------------------------------------------------------------
def kept_positions(n_tokens: int):
    """Positions stored verbatim: the first 4 and the last 128 (all of them if N <= 132)."""
    if n_tokens <= HEAD_KEPT + TAIL_KEPT:
        return list(range(n_tokens))
    return list(range(HEAD_KEPT)) + list(range(n_tokens - TAIL_KEPT, n_tokens))


def prompt_layout(seq_lens):
    """Per prompt: N, coded rows n = N - 132 (>= 0), n_e = ceil(n/2), n_o = floor(n/2),
    token base and coded-row base.  Coded row i sits at position 4 + i; its parity is i's."""
    out = []
    tbase = 0
    rbase = 0
    for N in seq_lens:
        N = int(N)
        n = max(0, N - HEAD_KEPT - TAIL_KEPT)
        out.append(dict(N=N, n=n, n_e=(n + 1) // 2, n_o=n // 2, tok_base=tbase, row_base=rbase))
        tbase += N
        rbase += n
    return out


def chunk_list(layout, chunk_rows: int):
    """Chunks of `chunk_rows` consecutive same-parity rows: every even chunk (prompt order)
    first, then every odd chunk.  Entries are (prompt, parity, first j, rows), where row
    j of parity p is coded row i = 2 j + p of its prompt."""
    ev, od = [], []
    for b, L in enumerate(layout):
        for j0 in range(0, L["n_e"], chunk_rows):
            ev.append((b, 0, j0, min(chunk_rows, L["n_e"] - j0)))
        for j0 in range(0, L["n_o"], chunk_rows):
            od.append((b, 1, j0, min(chunk_rows, L["n_o"] - j0)))
    return ev + od, len(ev), len(od)


# ----------------------------------------------------------------------------------------
# rANS (C helper)
# ----------------------------------------------------------------------------------------
_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "_build", "librans_oracle.so")
_lib = None


def build_lib(force: bool = False) -> str:
    """Compile rans_oracle.c with gcc (plain -O2)."""
    src = os.path.join(_HERE, "rans_oracle.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-shared", "-fPIC", "-o", tmp, src])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build_lib())
        P = ctypes.c_void_p
        lib.oracle_rans_encode.restype = ctypes.c_long
        lib.oracle_rans_encode.argtypes = [P, P, ctypes.c_long, P, P, P, P, ctypes.c_long]
        lib.oracle_rans_decode.restype = ctypes.c_long
        lib.oracle_rans_decode.argtypes = [P, P, ctypes.c_long, P, ctypes.c_long, P, P, P]
        lib.oracle_rans_states_after.restype = ctypes.c_int
        lib.oracle_rans_states_after.argtypes = [P, P, ctypes.c_long, P, ctypes.c_long, P, P, P]
        _lib = lib
    return _lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def rans_encode(sym, scl, freq, cdf):
    """One chunk: returns (states uint32 [32], words uint16 [n]) in decoder order."""
    lib = _load()
    sym = np.ascontiguousarray(sym, np.uint16)
    scl = np.ascontiguousarray(scl, np.uint8)
    freq = np.ascontiguousarray(freq, np.uint32)
    cdf = np.ascontiguousarray(cdf, np.uint32)
    cap = max(1, sym.size)
    words = np.zeros(cap, np.uint16)
    states = np.zeros(LANES, np.uint32)
    n = lib.oracle_rans_encode(_ptr(sym), _ptr(scl), sym.size, _ptr(freq), _ptr(cdf),
                               _ptr(states), _ptr(words), cap)
    if n < 0:
        raise ValueError("rans_encode failed")
    return states, words[:n].copy()


def rans_decode(states, words, scl, freq, cdf, n_symbols=None):
    """One chunk: returns (symbols uint16 [S], words consumed); raises on a stream
    overrun or if a state does not end at L (the encoder's start value)."""
    lib = _load()
    scl = np.ascontiguousarray(scl, np.uint8)
    S = scl.size if n_symbols is None else int(n_symbols)
    states = np.ascontiguousarray(states, np.uint32)
    words = np.ascontiguousarray(words, np.uint16)
    freq = np.ascontiguousarray(freq, np.uint32)
    cdf = np.ascontiguousarray(cdf, np.uint32)
    out = np.zeros(max(1, S), np.uint16)
    wp = _ptr(words) if words.size else None
    w = lib.oracle_rans_decode(_ptr(states), wp, words.size, _ptr(scl), S, _ptr(freq), _ptr(cdf),
                               _ptr(out))
    if w < 0:
        raise ValueError(f"rans_decode failed ({w})")
    fin = np.zeros(LANES, np.uint32)
    lib.oracle_rans_states_after(_ptr(states), wp, words.size, _ptr(scl), S, _ptr(freq), _ptr(cdf),
                                 _ptr(fin))
    if np.any(fin != RANS_L):
        raise ValueError("rans_decode: final states differ from L")
    return out[:S], int(w)


def model_code_length_bits(sym, scl, freq, n_esc: int) -> float:
    """Sum of -log2(freq/2^16) over coded symbols plus 64 bits per escape."""
    f = np.asarray(freq, np.float64)[np.asarray(scl, np.int64), np.asarray(sym, np.int64)]
    return float(-np.log2(f / PREC_TOTAL).sum() + 64.0 * n_esc)


# ----------------------------------------------------------------------------------------
# RoPE and reconstruction  [rows]
# ----------------------------------------------------------------------------------------
def rope(head_vecs, positions):
    """Rotate-half RoPE over all 256 dims, base 1e7: pairs (d, d + 128) at
    theta_d = 1e7^(-2d/256), rotated by position * theta_d (reading: the Qwen / HF
    convention).  head_vecs [..., rows, 256] fp64, positions [rows]."""
    v = np.asarray(head_vecs, np.float64)
    half = HEAD_DIM // 2
    d = np.arange(half, dtype=np.float64)
    theta = ROPE_BASE ** (-2.0 * d / HEAD_DIM)
    ang = np.asarray(positions, np.float64)[:, None] * theta[None, :]
    c, s = np.cos(ang), np.sin(ang)
    a, b = v[..., :half], v[..., half:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def reconstruct(q, codec) -> np.ndarray:
    """x_hat = mu + sum_c q_c Delta_c B[:, c] (linear synthesis; the decoder has no x to
    evaluate the encoder's correction on)  [rows], [xform].

    With synthesis weights V1 [2048, 256] and V2 [256, 6144] (the decoder-side learned
    synthesis the weight count on the pages leaves room for, "How to use it": 176 MiB
    against 96 MiB for the linear codec) the same kind of one-hidden-layer GELU correction
    is added on the decoded coefficients: + GELU((q Delta) V1) V2, no biases."""
    qd = np.asarray(q, np.float64) * np.asarray(codec.delta, np.float64)[None, :]
    x = np.asarray(codec.mu, np.float64)[None, :] + qd @ np.asarray(codec.basis, np.float64).T
    v1 = getattr(codec, "v1", None)
    v2 = getattr(codec, "v2", None)
    if v1 is not None and v2 is not None:
        x = x + gelu(qd @ np.asarray(v1, np.float64)) @ np.asarray(v2, np.float64)
    return x


def output_rows(rows_f64, positions):
    """Apply RoPE to the key parts of full 6,144-dim rows; returns fp64 rows."""
    r = np.asarray(rows_f64, np.float64).reshape(-1, N_LAYERS, 2, N_KV_HEADS, HEAD_DIM).copy()
    for l in range(N_LAYERS):
        for h in range(N_KV_HEADS):
            r[:, l, 0, h, :] = rope(r[:, l, 0, h, :], positions)
    return r.reshape(-1, ROW_DIM)


def _scatter_out(rows_bits, k_out, v_out, tok_idx):
    r = rows_bits.reshape(-1, N_LAYERS, 2, N_KV_HEADS, HEAD_DIM)
    k_out[:, tok_idx] = np.transpose(r[:, :, 0], (1, 0, 2, 3))
    v_out[:, tok_idx] = np.transpose(r[:, :, 1], (1, 0, 2, 3))


# ----------------------------------------------------------------------------------------
# encode / decode
# ----------------------------------------------------------------------------------------
def _pad(buf: bytearray, align: int):
    while len(buf) % align:
        buf.append(0)


def analyse(x, tok, seq_offsets, codec):
    """Codes and centres of every prompt (the arithmetic of encoding, before the coder).

    Per prompt: transform -> quantise -> drop; even means from the token embedding; odd
    means from the embedding and both even neighbours; centres.  Returns a list of dicts
    with q, ratio (y / Delta), qe, qo, mu_e, mu_o, ce, co."""
    x = np.asarray(x)
    tok = np.asarray(tok, np.int64)
    offs = np.asarray(seq_offsets, np.int64)
    layout = prompt_layout(np.diff(offs))
    s_idx, keep = scale_index(codec.laplace_b, codec.delta)
    out = []
    for L in layout:
        t0 = L["tok_base"]
        n = L["n"]
        rows = x[t0 + HEAD_KEPT: t0 + HEAD_KEPT + n]
        if n > 0:
            y = transform(rows, codec)
            q, ratio = quantise(y, codec.delta, keep)
        else:
            q = np.zeros((0, N_COEF), np.int64)
            ratio = np.zeros((0, N_COEF))
        qe, qo = q[0::2], q[1::2]
        te = tok[t0 + HEAD_KEPT: t0 + HEAD_KEPT + n: 2]
        to = tok[t0 + HEAD_KEPT + 1: t0 + HEAD_KEPT + n: 2]
        mu_e = codec_means_even(codec, te) if qe.shape[0] else np.zeros((0, N_COEF))
        q_right = np.concatenate([qe[1:], np.zeros((1, N_COEF), np.int64)], 0)[: qo.shape[0]]
        mu_o = (codec_means_odd(codec, to, qe[: qo.shape[0]], q_right)
                if qo.shape[0] else np.zeros((0, N_COEF)))
        out.append(dict(q=q, ratio=ratio, qe=qe, qo=qo, mu_e=mu_e, mu_o=mu_o, ce=centres(mu_e), co=centres(mu_o)))
    return out


def assemble_blob(x, seq_offsets, codes, laplace_b, delta, chunk_rows: int = DEFAULT_CHUNK_ROWS,
                  aux: dict | None = None):
    """The coder and the container: symbols from (q, centre), rANS per chunk, escapes,
    kept rows, header and tables.  `codes` is a list (per prompt) of dicts with qe, qo,
    ce, co (codes and centres of even / odd rows)."""
    x = np.asarray(x)
    offs = np.asarray(seq_offsets, np.int64)
    lens = np.diff(offs)
    layout = prompt_layout(lens)
    s_idx, keep = scale_index(laplace_b, delta)
    kept_c = np.nonzero(keep)[0]
    k_eff = kept_c.size
    freq, cdf = laplace_tables()
    chunks, n_ev, n_od = chunk_list(layout, chunk_rows)
    syms = []
    for P in codes:
        se, esc_e = symbols(P["qe"], P["ce"], keep)
        so, esc_o = symbols(P["qo"], P["co"], keep)
        syms.append((se, so))

    streams = bytearray()
    offsets = []
    n_esc_total = 0
    code_bits = 0.0
    sections = []
    for (b, par, j0, nr) in chunks:
        P = codes[b]
        sym = syms[b][par][j0:j0 + nr].reshape(-1)
        qk = ((P["qe"] if par == 0 else P["qo"])[j0:j0 + nr])[:, kept_c].reshape(-1)
        scl = np.tile(s_idx[kept_c], nr).astype(np.uint8)
        states, words = rans_encode(sym, scl, freq, cdf)
        escv = qk[sym == ESC_SYMBOL]
        offsets.append(len(streams))
        sec = bytearray()
        sec += states.astype("<u4").tobytes()
        sec += struct.pack("<I", escv.size)
        sec += escv.astype("<i8").tobytes()
        sec += words.astype("<u2").tobytes()
        _pad(sec, 4)
        streams += sec
        sections.append(bytes(sec))
        n_esc_total += escv.size
        code_bits += model_code_length_bits(sym, scl, freq, escv.size)
    offsets.append(len(streams))
    if len(streams) >= 2 ** 32:
        raise ValueError("stream section exceeds 4 GiB")

    kept_rows = []
    for L in layout:
        for p in kept_positions(L["N"]):
            kept_rows.append(L["tok_base"] + p)
    n_kept = len(kept_rows)

    # layout: header | prompt lengths | chunk offsets | pad16 | kept rows | chunk sections
    blob = bytearray(HEADER_BYTES)
    blob += np.asarray(lens, "<u4").tobytes()
    blob += np.asarray(offsets, "<u4").tobytes()
    _pad(blob, 16)
    off_kept = len(blob)
    if n_kept:
        kr = x[np.asarray(kept_rows)]
        kr_bits = kr if kr.dtype == np.uint16 else f64_to_bf16(kr)
        blob += np.ascontiguousarray(kr_bits, "<u2").tobytes()
    off_streams = len(blob)
    blob += streams
    total = len(blob)
    struct.pack_into("<IHHIIIIII", blob, 0, MAGIC, VERSION, chunk_rows, len(lens), N_COEF,
                     k_eff, n_ev, n_od, n_kept)
    struct.pack_into("<QQQQ", blob, 32, total, off_streams, off_kept, 0)
    if aux is not None:
        aux.update(layout=layout, chunks=chunks, keep=keep, s_idx=s_idx, n_esc=n_esc_total,
                   code_bits=code_bits, freq=freq, cdf=cdf, sections=sections)
    return bytes(blob)


def encode(x, tok, seq_offsets, codec, chunk_rows: int = DEFAULT_CHUNK_ROWS, aux: dict | None = None):
    """Encode a batch of prompts into one blob (bytes).

    x: [sum N, 6144] rows (bf16 bits as uint16, or floats); tok: [sum N] token ids;
    seq_offsets: [B+1].  Steps: transform -> quantise -> drop -> even means from the
    token embedding -> odd means from embedding + both even neighbours -> centres ->
    symbols -> rANS per chunk -> blob.  If `aux` is a dict it receives the intermediates
    (per_prompt: q, ratio, centres, means per prompt and parity)."""
    per_prompt = analyse(x, tok, seq_offsets, codec)
    blob = assemble_blob(x, seq_offsets, per_prompt, codec.laplace_b, codec.delta, chunk_rows, aux)
    if aux is not None:
        aux["per_prompt"] = per_prompt
    return blob


def parse_blob(blob):
    """Header fields, prompt lengths and chunk offsets; raises ValueError if malformed."""
    blob = bytes(blob)
    if len(blob) < HEADER_BYTES:
        raise ValueError("blob shorter than its header")
    magic, ver, G, nb, ncoef, k_eff, n_ev, n_od, n_kept = struct.unpack_from("<IHHIIIIII", blob, 0)
    total, off_s, off_k, _ = struct.unpack_from("<QQQQ", blob, 32)
    if magic != MAGIC or ver != VERSION or ncoef != N_COEF or G == 0:
        raise ValueError("bad header")
    if total > len(blob):
        raise ValueError("blob truncated")
    p = HEADER_BYTES
    if p + 4 * (nb + n_ev + n_od + 1) > total:
        raise ValueError("tables overrun the blob")
    lens = np.frombuffer(blob, "<u4", nb, p).astype(np.int64)
    p += 4 * nb
    offs = np.frombuffer(blob, "<u4", n_ev + n_od + 1, p).astype(np.int64)
    p += 4 * (n_ev + n_od + 1)
    p = (p + 15) // 16 * 16
    if (off_k != p or off_s != off_k + n_kept * ROW_DIM * 2 or offs[0] != 0
            or np.any(np.diff(offs) < 4 * LANES + 4) or off_s + offs[-1] != total):
        raise ValueError("bad chunk table")
    return dict(chunk_rows=G, n_prompts=nb, k_eff=k_eff, n_chunks_even=n_ev, n_chunks_odd=n_od,
                n_kept=n_kept, total=total, off_streams=off_s, off_kept=off_k, lens=lens,
                chunk_offsets=offs)


def _chunk_payload(blob, hdr, c):
    base = hdr["off_streams"] + hdr["chunk_offsets"][c]
    end = hdr["off_streams"] + hdr["chunk_offsets"][c + 1]
    states = np.frombuffer(blob, "<u4", LANES, base).astype(np.uint32)
    n_esc = struct.unpack_from("<I", blob, base + 4 * LANES)[0]
    p = base + 4 * LANES + 4
    if p + 8 * n_esc > end:
        raise ValueError("escape section overruns its chunk")
    escv = np.frombuffer(blob, "<i8", n_esc, p).astype(np.int64)
    p += 8 * n_esc
    words = np.frombuffer(blob, "<u2", (end - p) // 2, p).astype(np.uint16)
    return states, escv, words


def decode(blob, tok, seq_offsets, codec, aux: dict | None = None):
    """Decode a blob: even pass (means from the embedding), then odd pass (means from the
    embedding and the decoded even neighbours), then x_hat = mu + (q * Delta) B^T, RoPE on
    the keys, bf16.  Returns k_out, v_out as bf16 bits [6, sum N, 2, 256]  [rows], [cond]."""
    blob = bytes(blob)
    hdr = parse_blob(blob)
    tok = np.asarray(tok, np.int64)
    offs = np.asarray(seq_offsets, np.int64)
    lens = np.diff(offs)
    if hdr["n_prompts"] != lens.size or np.any(hdr["lens"] != lens):
        raise ValueError("prompt lengths do not match the blob")
    layout = prompt_layout(lens)
    s_idx, keep = scale_index(codec.laplace_b, codec.delta)
    kept_c = np.nonzero(keep)[0]
    if hdr["k_eff"] != kept_c.size:
        raise ValueError("codec does not match the blob")
    freq, cdf = laplace_tables()
    chunks, n_ev, n_od = chunk_list(layout, hdr["chunk_rows"])
    if (n_ev, n_od) != (hdr["n_chunks_even"], hdr["n_chunks_odd"]):
        raise ValueError("chunk counts do not match")

    qe_all = [np.zeros((L["n_e"], N_COEF), np.int64) for L in layout]
    qo_all = [np.zeros((L["n_o"], N_COEF), np.int64) for L in layout]

    def run_pass(par):
        for c, (b, pp, j0, nr) in enumerate(chunks):
            if pp != par:
                continue
            L = layout[b]
            t0 = L["tok_base"] + HEAD_KEPT
            js = np.arange(j0, j0 + nr)
            toks = tok[t0 + 2 * js + par]
            if par == 0:
                mu = codec_means_even(codec, toks)
            else:
                qe = qe_all[b]
                right = np.concatenate([qe[1:], np.zeros((1, N_COEF), np.int64)], 0)
                mu = codec_means_odd(codec, toks, qe[js], right[js])
            cen = centres(mu)[:, kept_c].reshape(-1)
            states, escv, words = _chunk_payload(blob, hdr, c)
            scl = np.tile(s_idx[kept_c], nr).astype(np.uint8)
            sym, used = rans_decode(states, words, scl, freq, cdf)
            sym = sym.astype(np.int64)
            # the section ends on a 4-byte boundary: at most one zero pad word is left over
            if not (used == words.size or (used == words.size - 1 and words[-1] == 0)):
                raise ValueError("chunk stream length does not match its symbols")
            is_esc = sym == ESC_SYMBOL
            if is_esc.sum() != escv.size:
                raise ValueError("escape count mismatch")
            qk = sym - R_MAX + cen
            qk[is_esc] = escv
            dst = qe_all[b] if par == 0 else qo_all[b]
            dst[j0:j0 + nr][:, kept_c] = qk.reshape(nr, kept_c.size)

    run_pass(0)
    run_pass(1)

    n_tot = int(offs[-1])
    k_out = np.zeros((N_LAYERS, n_tot, N_KV_HEADS, HEAD_DIM), np.uint16)
    v_out = np.zeros_like(k_out)
    kept_ptr = hdr["off_kept"]
    pre_rope = []
    for b, L in enumerate(layout):
        t0 = L["tok_base"]
        kp = kept_positions(L["N"])
        if kp:
            kr = np.frombuffer(blob, "<u2", len(kp) * ROW_DIM, kept_ptr).reshape(len(kp), ROW_DIM)
            kept_ptr += len(kp) * ROW_DIM * 2
            rows = output_rows(bf16_to_f64(kr), np.asarray(kp))
            _scatter_out(f64_to_bf16(rows), k_out, v_out, t0 + np.asarray(kp))
        if L["n"]:
            q = np.zeros((L["n"], N_COEF), np.int64)
            q[0::2] = qe_all[b]
            q[1::2] = qo_all[b]
            xh = reconstruct(q, codec)
            pos = np.arange(HEAD_KEPT, HEAD_KEPT + L["n"])
            rows = output_rows(xh, pos)
            _scatter_out(f64_to_bf16(rows), k_out, v_out, t0 + pos)
            pre_rope.append(xh)
    if aux is not None:
        aux.update(qe=qe_all, qo=qo_all, xhat=pre_rope, header=hdr)
    return k_out, v_out


def byte_report(blob, aux: dict | None = None):
    """Byte breakdown: header+tables, states, escape counts, escape values, words,
    padding, kept rows; payload = everything except the kept rows.

    Blob layout (little endian): 64-byte header {u32 magic 'DCKV', u16 version, u16 chunk
    rows, u32 prompts, u32 coefficients, u32 kept components, u32 even chunks, u32 odd
    chunks, u32 kept rows, u64 total bytes, u64 stream offset, u64 kept-row offset, u64 0};
    u32 prompt lengths; u32 chunk-section offsets (relative to the stream offset, one more
    than the chunks); zero pad to 16; kept rows (bf16, prompt-major, ascending position);
    chunk sections, each {u32 states[32], u32 escape count, i64 escape codes, u16 words in
    decoder order, zero pad to 4}."""
    blob = bytes(blob)
    hdr = parse_blob(blob)
    n_ch = hdr["n_chunks_even"] + hdr["n_chunks_odd"]
    states = esc_cnt = esc_val = words = 0
    for c in range(n_ch):
        st, ev, w = _chunk_payload(blob, hdr, c)
        states += 4 * LANES
        esc_cnt += 4
        esc_val += 8 * ev.size
        words += 2 * w.size
    kept = hdr["off_streams"] - hdr["off_kept"]
    return dict(total=hdr["total"], header_tables=hdr["off_kept"], states=states,
                esc_counts=esc_cnt, esc_values=esc_val, words=words, kept_rows=kept,
                payload=hdr["total"] - kept,
                padding=hdr["total"] - kept - hdr["off_kept"] - states - esc_cnt - esc_val - words)

"""The synthetic inputs have the structure their recipe states (CPU)."""
import numpy as np
import torch

import dckv_synth as S


def test_structured_prompt_neighbour_and_token_structure():
    src = S.source(0)
    cod = S.codec(src, step_scale=1.0, literal_b=True)
    g, a = 0.6, 0.8
    x, tok = S.structured_prompt(src, cod.embed, 800, 5, token_gain=g, ar=a)
    assert x.dtype == torch.bfloat16 and x.shape == (800, S.ROW_DIM) and tok.shape == (800,)
    # undo the fixed linear map: z = ((x - mu) / s) Q diag(1/sigma) (Q orthonormal)
    xs = (x.double() - torch.from_numpy(src.mu).double()) / torch.from_numpy(src.chan_scale).double()
    z = (xs @ torch.from_numpy(src.q).double()) / torch.from_numpy(src.sigma)
    zt = z[:, :64]  # the leading directions, where bf16 rounding is negligible against sigma
    lag1 = float((zt[1:] * zt[:-1]).sum() / (zt * zt).sum())
    assert abs(lag1 - (1 - g * g) * a) < 0.05, lag1
    assert abs(float(zt.var()) - 1.0) < 0.1
    x2, _ = S.structured_prompt(src, cod.embed, 800, 5, token_gain=g, ar=a)
    assert torch.equal(x2, x)  # seeded
    # with g = 1 a row is a function of its token alone: equal tokens, equal rows
    xa, ta = S.structured_prompt(src, cod.embed, 800, 11, token_gain=1.0, ar=0.0)
    xb, tb = S.structured_prompt(src, cod.embed, 800, 12, token_gain=1.0, ar=0.0)
    pairs = [(i, j) for i in range(800) for j in np.nonzero(tb.numpy() == int(ta[i]))[0]]
    assert len(pairs) >= 5
    for i, j in pairs:
        assert torch.equal(xa[i], xb[j])
    assert not torch.equal(xa[0], xa[1]) or int(ta[0]) == int(ta[1])


def test_plain_prompt_rows_are_independent():
    src = S.source(0)
    x, tok = S.prompt(src, 800, 6)
    xs = (x.double() - torch.from_numpy(src.mu).double()) / torch.from_numpy(src.chan_scale).double()
    z = (xs @ torch.from_numpy(src.q).double()) / torch.from_numpy(src.sigma)
    zt = z[:, :64]
    lag1 = float((zt[1:] * zt[:-1]).sum() / (zt * zt).sum())
    assert abs(lag1) < 0.05, lag1


def test_calibrated_step_scales_reproduce_their_payload():
    """The stored step scales are what the calibration script's bisection found: every entry
    met its target within 1%, and re-running the oracle's encoder at the stored step scale on
    the calibration sample gives the recorded payload again (checked for the ~220 B/row,
    16-rows-per-chunk entry of the plain codec)."""
    import json
    import os

    from oracle import calibrate_step_scales as C

    with open(os.path.join(os.path.dirname(S.__file__), "step_scales.json")) as f:
        table = json.load(f)
    keys = {(e["target_bytes"], e["chunk_rows"], e["student_t_frac"], e["linear"]) for e in table["entries"]}
    assert keys == set(C.ENTRIES)
    for e in table["entries"]:
        assert abs(e["payload_per_row"] / e["target_bytes"] - 1.0) < 0.01, e
        assert S.calibrated_step_scale(e["target_bytes"], e["chunk_rows"], e["student_t_frac"],
                                       e["linear"]) == e["step_scale"]
    src = S.source(0)
    e = next(e for e in table["entries"] if e["target_bytes"] == 220.0 and e["student_t_frac"] == 0.0
             and not e["linear"])
    x, tok, offs = S.batch(src, [C.SAMPLE_LEN] * len(C.SAMPLE_SEEDS), list(C.SAMPLE_SEEDS))
    xb = x.view(torch.int16).numpy().view(np.uint16)
    got = C.payload_per_row(src, xb, tok.numpy(), offs, e["step_scale"], e["chunk_rows"], False)
    assert abs(got - e["payload_per_row"]) < 0.01, (got, e["payload_per_row"])
    cod = S.calibrated_codec(src, 220.0, 16)
    assert cod.step_scale == e["step_scale"]

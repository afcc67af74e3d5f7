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

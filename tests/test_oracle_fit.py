"""Pins of the oracle's closed-form fit of the conditional models (CPU).

Each test ties the fit to something other than its own formulas: a scalar worked by
hand, exact recovery of a known linear map, the ridge objective's minimum, the
checkerboard neighbour order spelled out row by row, the Laplace likelihood's maximum
found by search, and the end-to-end effect on the model code length.
"""
import numpy as np
import pytest

import dckv_synth as S
import oracle as O

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def test_fit_solve_scalar_worked_by_hand():
    # x = (1, 2, 3), y = (2, 4, 7), ridge 0.5:  sum xy = 31, sum x^2 = 14,
    # w = 31 / (14 + 0.5 * (14 + 1)) = 31 / 21.5
    x = np.array([[1.0], [2.0], [3.0]])
    y = np.array([[2.0], [4.0], [7.0]])
    w = O.fit_solve(x.T @ x, x.T @ y, 0.5)
    assert w.shape == (1, 1)
    assert abs(w[0, 0] - 31.0 / 21.5) < 1e-15


def test_fit_solve_recovers_a_known_linear_map_and_zeroes_dead_regressors():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((300, 10))
    x[:, 3] = 0.0  # a regressor that is always 0 (the code of a dropped component)
    w_true = rng.standard_normal((10, 4))
    w_true[3] = 0.0
    y = x @ w_true
    w = O.fit_solve(x.T @ x, x.T @ y, 1e-13)
    assert np.all(np.isfinite(w))
    assert np.max(np.abs(w - w_true)) < 1e-9
    assert np.all(w[3] == 0.0)


def test_fit_solve_minimises_the_ridge_objective():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((80, 7)) * np.array([1e-2, 1, 1, 30, 1, 5, 0.1])
    y = rng.standard_normal((80, 3))
    lam = 0.05
    w = O.fit_solve(x.T @ x, x.T @ y, lam)
    pen = lam * ((x * x).sum(0) + 1.0)

    def objective(v):
        r = y - x @ v
        return float((r * r).sum() + (pen[:, None] * v * v).sum())

    f0 = objective(w)
    for _ in range(20):
        d = rng.standard_normal(w.shape) * 1e-3
        assert objective(w + d) > f0 and objective(w - d) > f0


def _embed(vocab=8):
    rng = np.random.default_rng(7)
    return S.f32_to_bf16_bits(rng.standard_normal((vocab, O.N_COEF)).astype(np.float32))


@pytest.mark.parametrize("n", [6, 5])
def test_fit_regressors_follow_the_checkerboard(n):
    # coded rows i = 0..n-1; even rows 0, 2, 4; odd row 2j + 1 sits between 2j and 2j + 2
    rng = np.random.default_rng(n)
    q = rng.integers(-400, 400, size=(n, O.N_COEF))
    q[0, 0], q[1, 1] = 301, 40000  # 301 is not a bf16 value (rounds to 300); 40000 > clip
    toks = rng.integers(0, 8, size=n)
    emb = _embed()
    xe, ye, xo, yo = O.fit_regressors(q[0::2], q[1::2], toks[0::2], toks[1::2], emb)
    assert xe.shape == ((n + 1) // 2, O.N_COEF) and xo.shape == (n // 2, 3 * O.N_COEF)
    for j in range(n // 2):
        i = 2 * j + 1
        assert np.array_equal(xo[j, :O.N_COEF], O.bf16_to_f64(emb[toks[i]]))
        left = q[i - 1].astype(np.float64)
        right = q[i + 1].astype(np.float64) if i + 1 < n else np.zeros(O.N_COEF)
        assert np.array_equal(xo[j, O.N_COEF:2 * O.N_COEF], O.bf16_to_f64(O.f64_to_bf16(left)))
        assert np.array_equal(xo[j, 2 * O.N_COEF:], O.bf16_to_f64(O.f64_to_bf16(right)))
        assert np.array_equal(yo[j], np.clip(q[i], -32767, 32767))
    for j in range((n + 1) // 2):
        assert np.array_equal(xe[j], O.bf16_to_f64(emb[toks[2 * j]]))
        assert np.array_equal(ye[j], np.clip(q[2 * j], -32767, 32767))
    assert xe[0, 0] == O.bf16_to_f64(emb[toks[0]])[0] and ye[0, 0] == 301.0
    if n // 2 >= 1:
        assert xo[0, O.N_COEF] == 300.0  # bf16(301) as the left neighbour of row 1
        assert yo[0, 1] == 32767.0


def test_fit_statistics_sum_row_by_row_over_prompts():
    # two prompts (3 and 2 coded rows after the 132 kept positions, plus a short prompt)
    lens = [132 + 3, 50, 132 + 2]
    offs = np.concatenate([[0], np.cumsum(lens)])
    rng = np.random.default_rng(9)
    tok = rng.integers(0, 8, size=offs[-1])
    emb = _embed()
    codes = []
    for n in (3, 0, 2):
        q = rng.integers(-300, 300, size=(n, O.N_COEF))
        codes.append(dict(qe=q[0::2], qo=q[1::2]))
    st = O.fit_statistics_from_codes(codes, tok, offs, emb)
    assert st["n_e"] == 2 + 1 and st["n_o"] == 1 + 1
    # row by row: odd rows' regressors [e, bf16(left), bf16(right)]
    g = np.zeros((3 * O.N_COEF, 3 * O.N_COEF))
    c = np.zeros((3 * O.N_COEF, O.N_COEF))
    ge = np.zeros((O.N_COEF, O.N_COEF))
    for p, (t0, P) in enumerate(zip(offs[:-1], codes)):
        n = P["qe"].shape[0] + P["qo"].shape[0]
        for i in range(n):
            q = (P["qe"] if i % 2 == 0 else P["qo"])[i // 2]
            e = O.bf16_to_f64(emb[tok[t0 + 4 + i]])
            if i % 2 == 0:
                ge += np.outer(e, e)
                continue
            left = P["qe"][(i - 1) // 2]
            right = P["qe"][(i + 1) // 2] if i + 1 < n else np.zeros(O.N_COEF, np.int64)
            xr = np.concatenate([e, O.bf16_to_f64(O.f64_to_bf16(left.astype(np.float64))),
                                 O.bf16_to_f64(O.f64_to_bf16(right.astype(np.float64)))])
            g += np.outer(xr, xr)
            c += np.outer(xr, q.astype(np.float64))
    assert np.allclose(st["g_o"], g, rtol=1e-13, atol=1e-9)
    assert np.allclose(st["c_o"], c, rtol=1e-13, atol=1e-9)
    assert np.allclose(st["g_e"], ge, rtol=1e-13, atol=1e-12)


def test_fit_scales_are_the_laplace_likelihood_maximum():
    rng = np.random.default_rng(11)
    delta = np.full(O.N_COEF, 0.5, np.float32)
    b_old = np.full(O.N_COEF, 2.0, np.float32)
    b_old[7] = 0.01  # dropped (0.02 steps)
    q = rng.laplace(0.0, 3.0, size=(41, O.N_COEF)).round().astype(np.int64)
    c = rng.integers(-5, 6, size=(41, O.N_COEF))
    codes = [dict(qe=q[:21], ce=c[:21], qo=q[21:], co=c[21:])]
    total, rows = O.fit_scales_from_codes(codes, b_old, delta)
    assert rows == 41 and total[7] == 0
    r = (q - c)[:, 0].astype(np.float64)
    beta = total[0] / rows
    grid = np.linspace(0.2 * beta, 5 * beta, 4001)
    loglik = [-(np.log(2 * g) * r.size + np.abs(r).sum() / g) for g in grid]
    assert abs(grid[int(np.argmax(loglik))] - beta) <= (grid[1] - grid[0])
    b = O.scales_from_sums(total, rows, b_old, delta)
    assert b[7] == b_old[7]
    assert b[0] == np.float32(0.5 * (total[0] / 41.0))
    # a component predicted exactly keeps its place at the narrowest table (0.05 steps)
    codes[0]["ce"] = codes[0]["qe"].clip(-127, 127)
    codes[0]["co"] = codes[0]["qo"].clip(-127, 127)
    codes[0]["qe"][:, 1] = codes[0]["ce"][:, 1]
    codes[0]["qo"][:, 1] = codes[0]["co"][:, 1]
    total, rows = O.fit_scales_from_codes(codes, b_old, delta)
    b = O.scales_from_sums(total, rows, b_old, delta)
    assert total[1] == 0 and abs(float(b[1]) / 0.5 - 0.05) < 1e-8
    s, keep = O.scale_index(b, delta)
    assert keep[1] and s[1] == 0


def test_refit_on_structured_rows_lowers_the_code_length():
    # rows that depend on their token and their neighbours: fitting the mean models and
    # scales on them must lower the model code length of the same rows ("Evidence")
    src = S.source(0)
    cod = S.codec(src, step_scale=None, target_bytes=220.0)
    x, tok, offs = S.structured_batch(src, cod.embed, [132 + 400, 132 + 300], [3, 4], token_gain=0.6, ar=0.8)
    xb = x.view(__import__("torch").int16).numpy().view(np.uint16)
    tok = tok.numpy()
    aux0 = {}
    O.encode(xb, tok, offs, cod, aux=aux0)
    st = O.fit_statistics_from_codes(aux0["per_prompt"], tok, offs, cod.embed)
    w_e, w_o = O.fit_mean_models(st, 1e-3)
    means_only = O.refit_codec(cod, w_e, w_o)
    total, rows = O.fit_scales(xb, tok, offs, means_only)
    refit = O.refit_codec(cod, w_e, w_o, O.scales_from_sums(total, rows, cod.laplace_b, cod.delta))
    assert np.array_equal(O.scale_index(refit.laplace_b, refit.delta)[1], O.scale_index(cod.laplace_b, cod.delta)[1])
    aux1 = {}
    O.encode(xb, tok, offs, refit, aux=aux1)
    assert aux1["code_bits"] < 0.85 * aux0["code_bits"], (aux0["code_bits"], aux1["code_bits"])

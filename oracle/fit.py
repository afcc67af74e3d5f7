"""Closed-form fit of the conditional entropy models to a trained codec (oracle; test
infrastructure only).

Passage: "DCKV: Learned Transform Coding of the Prompt KV Cache in Hybrid Language
Models" (trove.briskstack.com summary), section "Evidence": fitting the conditional
models in closed form to an already-trained codec gives a saving similar to that of
the trained models, without retraining.  The models themselves are those of "How it
works", bullet "Conditional entropy models": even positions predict code means from
the token's input embedding, odd positions from the embedding and both decoded
neighbours.

The pages name the fit but not its formulas.  Readings (the plainest that the rest of
the pages supports):
  * "the conditional models" are the two mean models (W_e, W_o) and the per-component
    Laplace scales b_c; the transform (basis, correction, steps) stays as trained.
  * Mean models: ordinary least squares of the codes on the models' own inputs --
    even rows: e(tok) (bf16 embedding row); odd rows: [e(tok), bf16(q_left),
    bf16(q_right)] with the right neighbour 0 where the prompt has none -- solved from
    the normal equations with a ridge term on the diagonal:
        (G + lambda * (diag(G) + 1)) W = C,   G = X^T X,  C = X^T Y.
    The term is proportional to each regressor's own energy (so the embedding block and
    the code blocks, whose scales differ by orders of magnitude, are damped alike), plus
    lambda on every diagonal entry so that regressors that are always 0 (the codes of
    dropped components) get weight 0 instead of making the system singular.
  * Targets Y are the codes clipped to +-32767 (a bf16 hi/lo pair holds such integers
    exactly); codes of dropped components are 0 and are fitted like the others.
  * Scales: Laplace maximum likelihood with the location fixed at the table centre
    clamp(round(mu), -127, 127):  beta_c = sum |q - centre| / rows over the coded rows
    of both parities, b_c = Delta_c * max(beta_c, 0.05) for kept components; dropped
    components keep b_c.  The floor keeps the component set as trained: dropping is the
    transform's decision ("How it works", bullet "Transform"), and a dropped component
    decodes to 0, not to its predicted mean, so a well-predicted component must stay
    coded (its table is then the narrowest one, s = 0).
  * Fitted weights are stored as the codec stores them, bf16 (one round-to-nearest-even
    step from fp64).
Every step is fp64 numpy; numpy's matmul and solve are the only library primitives.
"""
from __future__ import annotations

import copy

import numpy as np

from .codec import (B0_STEPS, ESC_LIMIT, HEAD_KEPT, N_COEF, analyse, bf16_to_f64, f64_to_bf16, prompt_layout,
                    scale_index)

__all__ = ["FIT_CODE_CLIP", "fit_regressors", "fit_statistics_from_codes", "fit_statistics", "fit_solve",
           "fit_mean_models", "fit_scales_from_codes", "fit_scales", "scales_from_sums", "refit_codec"]

FIT_CODE_CLIP = 32767


def fit_regressors(qe, qo, tok_even, tok_odd, embed_bits):
    """One prompt's regressors and targets  ["Conditional entropy models"].

    qe / qo: codes of the even / odd coded rows (int, [n_e, 2048] / [n_o, 2048]);
    tok_even / tok_odd: their token ids.  Odd row j sits between even rows j (left) and
    j + 1 (right; a zero vector when the prompt ends first).
    Returns Xe [n_e, 2048], Ye [n_e, 2048], Xo [n_o, 6144], Yo [n_o, 2048] (fp64)."""
    qe = np.asarray(qe, np.int64)
    qo = np.asarray(qo, np.int64)
    emb_e = bf16_to_f64(np.asarray(embed_bits)[np.asarray(tok_even, np.int64)])
    emb_o = bf16_to_f64(np.asarray(embed_bits)[np.asarray(tok_odd, np.int64)])
    n_o = qo.shape[0]
    left = qe[:n_o]
    right = np.concatenate([qe[1:], np.zeros((1, N_COEF), np.int64)], 0)[:n_o]
    nb = lambda q: bf16_to_f64(f64_to_bf16(q.astype(np.float64)))  # bf16(q), as the model reads it
    xo = np.concatenate([emb_o, nb(left), nb(right)], axis=1)
    clip = lambda q: np.clip(q, -FIT_CODE_CLIP, FIT_CODE_CLIP).astype(np.float64)
    return emb_e, clip(qe), xo, clip(qo)


def fit_statistics_from_codes(codes, tok, seq_offsets, embed_bits):
    """Normal-equation statistics summed over prompts: G_e = Xe^T Xe [2048, 2048],
    C_e = Xe^T Ye [2048, 2048], G_o = Xo^T Xo [6144, 6144], C_o = Xo^T Yo [6144, 2048],
    and the row counts.  `codes` holds one dict per prompt with qe and qo."""
    tok = np.asarray(tok, np.int64)
    layout = prompt_layout(np.diff(np.asarray(seq_offsets, np.int64)))
    st = dict(g_e=np.zeros((N_COEF, N_COEF)), c_e=np.zeros((N_COEF, N_COEF)),
              g_o=np.zeros((3 * N_COEF, 3 * N_COEF)), c_o=np.zeros((3 * N_COEF, N_COEF)), n_e=0, n_o=0)
    for L, P in zip(layout, codes):
        n = L["n"]
        if n == 0:
            continue
        t0 = L["tok_base"] + HEAD_KEPT
        xe, ye, xo, yo = fit_regressors(P["qe"], P["qo"], tok[t0: t0 + n: 2], tok[t0 + 1: t0 + n: 2], embed_bits)
        st["g_e"] += xe.T @ xe
        st["c_e"] += xe.T @ ye
        st["g_o"] += xo.T @ xo
        st["c_o"] += xo.T @ yo
        st["n_e"] += xe.shape[0]
        st["n_o"] += xo.shape[0]
    return st


def fit_statistics(x, tok, seq_offsets, codec):
    """Statistics of a calibration batch under a trained codec's transform and quantiser."""
    return fit_statistics_from_codes(analyse(x, tok, seq_offsets, codec), tok, seq_offsets, codec.embed)


def fit_solve(g, c, ridge: float):
    """W = (G + ridge * (diag(G) + 1))^-1 C  (normal equations with the ridge term above)."""
    a = np.array(g, dtype=np.float64, copy=True)
    i = np.arange(a.shape[0])
    a[i, i] += ridge * (a[i, i] + 1.0)
    return np.linalg.solve(a, np.asarray(c, np.float64))


def fit_mean_models(stats, ridge: float):
    """Fitted mean-model weights (fp64): W_e [2048, 2048], W_o [6144, 2048]."""
    return fit_solve(stats["g_e"], stats["c_e"], ridge), fit_solve(stats["g_o"], stats["c_o"], ridge)


def fit_scales_from_codes(codes, laplace_b, delta):
    """Sum over coded rows of |q - centre| per component (kept components; int64, exact)
    and the number of coded rows.  `codes` holds one dict per prompt with qe, qo, ce, co
    (codes and table centres)."""
    _, keep = scale_index(laplace_b, delta)
    total = np.zeros(N_COEF, np.int64)
    rows = 0
    for P in codes:
        for q, c in ((P["qe"], P["ce"]), (P["qo"], P["co"])):
            q = np.asarray(q, np.int64)
            c = np.asarray(c, np.int64)
            assert np.all(np.abs(c) <= ESC_LIMIT)
            total += np.abs(q - c).sum(axis=0)
            rows += q.shape[0]
    total[~keep] = 0
    return total, rows


def fit_scales(x, tok, seq_offsets, codec):
    """Residual sums of a calibration batch under a codec (its mean models give the centres)."""
    return fit_scales_from_codes(analyse(x, tok, seq_offsets, codec), codec.laplace_b, codec.delta)


def scales_from_sums(abs_sum, rows, laplace_b, delta):
    """b_c = Delta_c * max(sum_c / rows, 0.05) for kept components (fp64, then fp32,
    raised by one fp32 ulp where rounding put b_c / Delta_c below 0.05); dropped
    components keep b_c."""
    _, keep = scale_index(laplace_b, delta)
    b = np.asarray(laplace_b, np.float32).copy()
    if rows > 0:
        d = np.asarray(delta, np.float32).astype(np.float64)
        fit = (d * np.maximum(np.asarray(abs_sum, np.float64) / float(rows), B0_STEPS)).astype(np.float32)
        # the fp32 value of Delta * 0.05 can fall just below the threshold: step up one ulp
        low = fit.astype(np.float64) / d < B0_STEPS
        fit[low] = np.nextafter(fit[low], np.float32(np.inf))
        b[keep] = fit[keep]
    return b


def refit_codec(codec, w_even, w_odd, laplace_b=None):
    """A copy of `codec` with fitted mean models (fp64 weights, stored bf16) and, if given,
    fitted Laplace scales."""
    out = copy.copy(codec)
    out.w_even = f64_to_bf16(np.asarray(w_even, np.float64))
    out.w_odd = f64_to_bf16(np.asarray(w_odd, np.float64))
    if laplace_b is not None:
        out.laplace_b = np.asarray(laplace_b, np.float32)
    out.note = getattr(codec, "note", "") + ", refit conditional models"
    return out

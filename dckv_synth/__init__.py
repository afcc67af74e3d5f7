"""Seeded synthetic inputs for the DCKV codec: KV rows, token ids and codec parameters.

This module only *draws* inputs.  It holds none of the codec's own arithmetic
(transform, quantiser, entropy model, rANS, inverse, RoPE); the CPU oracle and the
CUDA library each implement those independently and both consume what is drawn here.

Source of the shapes: "DCKV: Learned Transform Coding of the Prompt KV Cache in
Hybrid Language Models" (trove.briskstack.com summary), section "How it works":
Qwen3.5-2B keeps a KV cache in 6 full-attention layers, 12,288 bytes per token in
bf16; the first 4 and last 128 positions stay bf16; the other rows stack pre-RoPE
keys and values of all six layers (2 KV heads x 256 dims) into one 6,144-dim row,
projected to 2,048 coefficients with a 256-unit GELU correction.

Synthetic recipe (the pages publish no weights and no data):
  rows      x = bf16(mu + (Z diag(sigma) Q^T) * s), Z ~ N(0,1), sigma_i = i^-0.8
            (i = 1..6144), Q a seeded orthonormal matrix (Householder QR of a Gaussian
            matrix, sign-fixed), s = 4 on a seeded 1% of the key channels, else 1,
            mu ~ N(0, 0.1^2) per channel.  Optional Student-t (nu = 2) rows.
  codec     basis = Q[:, :2048]; W1 [6144,256], W2 [256,2048] ~ N(0, 0.01^2);
            Delta_c = k * 0.02 * sigma_c^0.5; Laplace scale b_c either 0.6 Delta_c
            (literal small config) or a closed-form fit (below); embedding table
            32,768 x 2,048 bf16; even mean model W_e [2048,2048] and odd mean model
            W_o [6144,2048] ~ N(0, 0.02^2), stored bf16.  The neighbour blocks of W_o
            act on decoded coefficients q_c * Delta_c; they are stored pre-multiplied
            by Delta_c so that both implementations feed bf16(q) into them.
  fitted b  b_c = Delta_c * E|rint(y_c / Delta_c)| with y_c ~ N(0, v_c), v_c the exact
            variance of the linear coefficient under the source model (outlier channel
            mixing included, correction MLP and Student-t rows ignored): the Laplace
            maximum-likelihood scale of the quantised coefficient, evaluated on the
            source distribution instead of a calibration sample.
  rate k    for the benchmark's configurations, read from step_scales.json (written by
            oracle/calibrate_step_scales.py: bisection on the payload the CPU oracle
            writes for a seeded calibration sample, per target rate, rows per rANS chunk,
            Student-t share and codec kind; calibrated_codec); otherwise chosen by
            bisection on a Gaussian-source estimate of the payload (codec(target_bytes=)).
"""
from __future__ import annotations

import json
import math
import os
from dataclasses import dataclass, field

import numpy as np

N_LAYERS = 6
N_KV_HEADS = 2
HEAD_DIM = 256
ROW_DIM = N_LAYERS * 2 * N_KV_HEADS * HEAD_DIM  # 6144
N_COEF = 2048
N_HIDDEN = 256
VOCAB = 32768
EMBED_DIM = 2048
HEAD_KEPT = 4
TAIL_KEPT = 128

_CACHE_DIR = os.environ.get(
    "DCKV_SYNTH_CACHE",
    os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "_build", "cache"),
)


def f32_to_bf16_bits(a) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16, returned as raw uint16 bits."""
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = a.view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    b = np.ascontiguousarray(np.asarray(b, dtype=np.uint16))
    return (b.astype(np.uint32) << 16).view(np.float32)


@dataclass
class Source:
    """The synthetic KV-row distribution (one seed)."""

    seed: int
    q: np.ndarray  # fp32 [6144, 6144], orthonormal columns
    sigma: np.ndarray  # fp64 [6144]
    chan_scale: np.ndarray  # fp32 [6144]
    mu: np.ndarray  # fp32 [6144]
    outlier_channels: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int64))


def _orthonormal(seed: int) -> np.ndarray:
    path = os.path.join(_CACHE_DIR, f"q_{ROW_DIM}_{seed}.npy")
    if os.path.exists(path):
        try:
            q = np.load(path)
            if q.shape == (ROW_DIM, ROW_DIM) and q.dtype == np.float32:
                return q
        except Exception:
            pass
    rng = np.random.default_rng([seed, 0x51])
    g = rng.standard_normal((ROW_DIM, ROW_DIM))
    q, r = np.linalg.qr(g)
    q *= np.sign(np.diag(r))[None, :]
    q = q.astype(np.float32)
    try:
        os.makedirs(_CACHE_DIR, exist_ok=True)
        tmp = path + f".{os.getpid()}.tmp.npy"
        np.save(tmp, q)
        os.replace(tmp, path)
    except OSError:
        pass
    return q


def source(seed: int = 0) -> Source:
    q = _orthonormal(seed)
    sigma = np.arange(1, ROW_DIM + 1, dtype=np.float64) ** -0.8
    rng = np.random.default_rng([seed, 0x52])
    # key channels: row index ((l*2 + kv)*2 + h)*256 + d with kv == 0
    idx = np.arange(ROW_DIM)
    key_chan = idx[((idx // (N_KV_HEADS * HEAD_DIM)) % 2) == 0]
    n_out = int(round(0.01 * key_chan.size))  # 31 of 3,072
    outl = np.sort(rng.choice(key_chan, size=n_out, replace=False))
    s = np.ones(ROW_DIM, np.float32)
    s[outl] = 4.0
    mu = (0.1 * rng.standard_normal(ROW_DIM)).astype(np.float32)
    return Source(seed=seed, q=q, sigma=sigma, chan_scale=s, mu=mu, outlier_channels=outl)


# ----------------------------------------------------------------------------------------
# codec parameters
# ----------------------------------------------------------------------------------------
@dataclass
class Codec:
    """Synthetic codec weights (what training would produce), as stored parameters."""

    mu: np.ndarray  # fp32 [6144]        codec mean
    basis: np.ndarray  # fp32 [6144, 2048]  shared linear basis (columns)
    w1: np.ndarray | None  # fp32 [6144, 256]   correction, first layer (None: linear codec)
    w2: np.ndarray | None  # fp32 [256, 2048]   correction, second layer
    delta: np.ndarray  # fp32 [2048]        quantiser steps (data units)
    laplace_b: np.ndarray  # fp32 [2048]    Laplace scales (data units)
    embed: np.ndarray | None  # u16 bf16 bits [32768, 2048] (None: unconditional tables)
    w_even: np.ndarray | None  # u16 bf16 bits [2048, 2048]   mu_even = e @ w_even
    w_odd: np.ndarray | None  # u16 bf16 bits [6144, 2048]    mu_odd = [e, bf16(qL), bf16(qR)] @ w_odd
    step_scale: float
    note: str = ""
    v1: np.ndarray | None = None  # fp32 [2048, 256]  decoder-side synthesis, first layer
    v2: np.ndarray | None = None  # fp32 [256, 6144]  decoder-side synthesis, second layer


def coefficient_variance(src: Source) -> np.ndarray:
    """Exact variance of (x - mu) @ basis under the source model (fp64, [2048])."""
    q = src.q.astype(np.float64)
    outl = src.outlier_channels
    extra = (src.chan_scale[outl].astype(np.float64) - 1.0)
    qo = q[outl, :]  # [31, 6144]
    m = (qo * extra[:, None]).T @ qo[:, :N_COEF]  # [6144, 2048]
    m[np.arange(N_COEF), np.arange(N_COEF)] += 1.0
    return (src.sigma ** 2) @ (m ** 2)


def _erfc(x):
    from scipy.special import erfc

    return erfc(x)


def _mean_abs_code(std_steps: np.ndarray) -> np.ndarray:
    """E|rint(u)| for u ~ N(0, std^2): sum_{m>=1} P(|u| >= m - 1/2)."""
    std_steps = np.maximum(std_steps, 1e-300)
    mmax = int(min(4000, np.ceil(np.max(std_steps) * 12 + 4)))
    m = np.arange(1, mmax + 1, dtype=np.float64) - 0.5
    t = _erfc(m[None, :] / (std_steps[:, None] * math.sqrt(2.0)))
    return t.sum(axis=1)


def _rate_estimate(std_steps: np.ndarray, beta: np.ndarray) -> float:
    """Gaussian-source estimate of the payload (bits per coded row) under Laplace(beta)."""
    from scipy.special import ndtr

    keep = beta >= 0.05
    sd = std_steps[keep]
    b = beta[keep]
    if sd.size == 0:
        return 0.0
    qmax = int(min(300, np.ceil(np.max(sd) * 8 + 3)))
    qs = np.arange(-qmax, qmax + 1, dtype=np.float64)
    lo = (qs[None, :] - 0.5) / sd[:, None]
    hi = (qs[None, :] + 0.5) / sd[:, None]
    p = np.clip(ndtr(hi) - ndtr(lo), 0.0, 1.0)
    # Laplace(0, b) mass of the unit cell around q
    def lap_cdf(x):
        return np.where(x < 0, 0.5 * np.exp(np.minimum(x, 0) / b[:, None]),
                        1.0 - 0.5 * np.exp(-np.maximum(x, 0) / b[:, None]))

    pl = lap_cdf(qs[None, :] + 0.5) - lap_cdf(qs[None, :] - 0.5)
    pl = np.maximum(pl, 2.0 ** -16)
    return float(np.sum(p * -np.log2(pl)))


def codec(
    src: Source,
    step_scale: float | None = 1.0,
    target_bytes: float | None = None,
    literal_b: bool = False,
    embed_std: float = 0.02,
    mean_gain: float = 1.0,
    neigh_gain: float = 1.0,
    zero_mlp: bool = False,
    seed: int | None = None,
    linear: bool = False,
    synthesis: bool = False,
    synthesis_gain: float = 1.0,
) -> Codec:
    """Draw a synthetic codec.

    step_scale / target_bytes: Delta_c = k * 0.02 * sigma_c^0.5, with k given or found by
    bisection so that the estimated payload is target_bytes per coded row.
    literal_b: b_c = 0.6 * Delta_c (the small configuration as written) instead of the fit.
    mean_gain / neigh_gain scale the mean-model weights (test variants with non-zero
    centres); zero_mlp sets the correction to zero (its initial state on the pages).
    linear: the linear codec the pages compare against -- no correction (w1 = w2 = None)
    and unconditional zero-mean tables (embed = w_even = w_odd = None).
    synthesis: add decoder-side synthesis weights V1 [2048, 256], V2 [256, 6144], both
    std 0.01 * synthesis_gain (0.01 like the encoder's correction).
    """
    seed = src.seed if seed is None else seed
    rng = np.random.default_rng([seed, 0x53])
    basis = np.ascontiguousarray(src.q[:, :N_COEF])
    w1 = (0.01 * rng.standard_normal((ROW_DIM, N_HIDDEN))).astype(np.float32)
    w2 = (0.01 * rng.standard_normal((N_HIDDEN, N_COEF))).astype(np.float32)
    if zero_mlp:
        w1[:] = 0
        w2[:] = 0
    sig_c = src.sigma[:N_COEF]
    std_y = np.sqrt(coefficient_variance(src))

    def params_for(k):
        delta = (k * 0.02 * np.sqrt(sig_c)).astype(np.float32)
        if literal_b:
            b = (0.6 * delta.astype(np.float64)).astype(np.float32)
        else:
            b = (delta.astype(np.float64) * _mean_abs_code(std_y / delta.astype(np.float64))).astype(np.float32)
        return delta, b

    if target_bytes is not None:
        lo, hi = math.log(0.05), math.log(2000.0)
        for _ in range(60):
            mid = 0.5 * (lo + hi)
            d, b = params_for(math.exp(mid))
            bits = _rate_estimate(std_y / d.astype(np.float64), b.astype(np.float64) / d.astype(np.float64))
            if bits / 8.0 > target_bytes:
                lo = mid
            else:
                hi = mid
        step_scale = float(math.exp(0.5 * (lo + hi)))
        step_scale = float(np.float32(step_scale))
    delta, b = params_for(step_scale)

    embed = f32_to_bf16_bits(embed_std * rng.standard_normal((VOCAB, EMBED_DIM), dtype=np.float32))
    w_even = f32_to_bf16_bits(0.02 * mean_gain * rng.standard_normal((EMBED_DIM, N_COEF)))
    w_odd_e = 0.02 * mean_gain * rng.standard_normal((EMBED_DIM, N_COEF))
    w_odd_n = 0.02 * neigh_gain * rng.standard_normal((2 * N_COEF, N_COEF))
    w_odd_n *= np.concatenate([delta, delta]).astype(np.float64)[:, None]
    w_odd = f32_to_bf16_bits(np.concatenate([w_odd_e, w_odd_n], axis=0))
    v1 = v2 = None
    if synthesis:
        srng = np.random.default_rng([seed, 0x5E])
        v1 = (0.01 * synthesis_gain * srng.standard_normal((N_COEF, N_HIDDEN))).astype(np.float32)
        v2 = (0.01 * synthesis_gain * srng.standard_normal((N_HIDDEN, ROW_DIM))).astype(np.float32)
    if linear:
        w1 = w2 = embed = w_even = w_odd = None
    return Codec(
        mu=src.mu.copy(), basis=basis, w1=w1, w2=w2, delta=delta, laplace_b=b,
        embed=embed, w_even=w_even, w_odd=w_odd, step_scale=float(step_scale),
        note=("literal b=0.6*Delta" if literal_b else "fitted b") + (", zero MLP" if zero_mlp else "")
        + (", linear codec" if linear else "") + (", synthesis MLP" if synthesis else ""),
        v1=v1, v2=v2,
    )


# ----------------------------------------------------------------------------------------
# prompts
# ----------------------------------------------------------------------------------------
def prompt(src: Source, n_tokens: int, seed: int, student_t_frac: float = 0.0, device="cpu"):
    """One prompt: x bf16 [N, 6144] (torch), token ids int32 [N] (torch), on `device`.

    Random streams come from torch generators on `device`, so the same seed gives
    different rows on CPU and GPU; every comparison draws once and feeds both sides.
    """
    import torch

    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(int(seed) * 7919 + 17)
    qt = torch.from_numpy(src.q).to(dev).t().contiguous()  # [6144(j), 6144(i)] = Q^T
    sig = torch.from_numpy(src.sigma.astype(np.float32)).to(dev)
    s = torch.from_numpy(src.chan_scale).to(dev)
    mu = torch.from_numpy(src.mu).to(dev)
    x = torch.empty((n_tokens, ROW_DIM), dtype=torch.bfloat16, device=dev)
    n_t = int(round(student_t_frac * n_tokens))
    t_rows = torch.zeros(n_tokens, dtype=torch.bool, device=dev)
    if n_t > 0:
        perm = torch.randperm(n_tokens, generator=g, device=dev)[:n_t]
        t_rows[perm] = True
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        step = 4096
        for r0 in range(0, n_tokens, step):
            r1 = min(n_tokens, r0 + step)
            z = torch.randn((r1 - r0, ROW_DIM), generator=g, device=dev, dtype=torch.float32)
            if n_t > 0:
                # Student-t, nu = 2, drawn per element: N / sqrt(chi2_2 / 2), chi2_2 = -2 ln U
                u = torch.rand((r1 - r0, ROW_DIM), generator=g, device=dev, dtype=torch.float32)
                u = u.clamp_min(1e-30)
                den = torch.sqrt(-torch.log(u))
                tz = z / den
                z = torch.where(t_rows[r0:r1, None], tz, z)
            w = (z * sig[None, :]) @ qt
            x[r0:r1] = (mu[None, :] + w * s[None, :]).to(torch.bfloat16)
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev
    tok = torch.randint(0, VOCAB, (n_tokens,), generator=g, device=dev, dtype=torch.int64).to(torch.int32)
    return x, tok


def batch(src: Source, lengths, seeds, student_t_frac: float = 0.0, device="cpu"):
    """Concatenated prompts: x [sum N, 6144], tok [sum N], seq_offsets int64 [B+1] (numpy)."""
    import torch

    xs, ts = [], []
    for n, sd in zip(lengths, seeds):
        x, t = prompt(src, int(n), int(sd), student_t_frac=student_t_frac, device=device)
        xs.append(x)
        ts.append(t)
    offs = np.zeros(len(lengths) + 1, np.int64)
    offs[1:] = np.cumsum(np.asarray(lengths, np.int64))
    return torch.cat(xs, 0), torch.cat(ts, 0), offs


def structured_prompt(src: Source, embed_bits, n_tokens: int, seed: int, token_gain: float = 0.5,
                      ar: float = 0.7, device="cpu"):
    """A prompt whose rows depend on their own token and on their neighbours: the input
    on which fitting the conditional models has something to find ("Evidence": the mean
    models predict codes from the token embedding and from both decoded neighbours).

    Latent z_t = sqrt(1 - g^2) u_t + g v(tok_t): u is an AR(1) process along the prompt's
    positions (u_t = a u_{t-1} + sqrt(1 - a^2) eps_t, unit variance), v(tok) = e(tok) P
    normalised to unit variance, e the embedding table the codec uses (bf16 bits) and P
    a seeded Gaussian [2048, 6144] matrix of the source.  Rows are then drawn as for plain
    prompts: x_t = bf16(mu + (z_t diag(sigma) Q^T) * s).  Returns x bf16 [N, 6144] and
    token ids int32 [N] (torch, on `device`).
    """
    import torch

    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(int(seed) * 7919 + 23)
    gp = torch.Generator(device=dev)
    gp.manual_seed(int(src.seed) * 31 + 5)
    tok = torch.randint(0, VOCAB, (n_tokens,), generator=g, device=dev, dtype=torch.int64)
    emb = torch.from_numpy(np.ascontiguousarray(embed_bits, np.uint16).view(np.int16)).to(dev)
    emb = emb.view(torch.bfloat16)
    rms = float(emb.float().pow(2).mean().sqrt())
    P = torch.randn((EMBED_DIM, ROW_DIM), generator=gp, device=dev, dtype=torch.float32)
    qt = torch.from_numpy(src.q).to(dev).t().contiguous()
    sig = torch.from_numpy(src.sigma.astype(np.float32)).to(dev)
    s = torch.from_numpy(src.chan_scale).to(dev)
    mu = torch.from_numpy(src.mu).to(dev)
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        eps = torch.randn((n_tokens, ROW_DIM), generator=g, device=dev, dtype=torch.float32)
        c = math.sqrt(1.0 - ar * ar)
        for t in range(1, n_tokens):
            eps[t] = ar * eps[t - 1] + c * eps[t]
        v = (emb[tok].float() @ P) / (rms * math.sqrt(EMBED_DIM))
        z = math.sqrt(1.0 - token_gain * token_gain) * eps + token_gain * v
        x = (mu[None, :] + ((z * sig[None, :]) @ qt) * s[None, :]).to(torch.bfloat16)
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev
    return x, tok.to(torch.int32)


def structured_batch(src: Source, embed_bits, lengths, seeds, token_gain: float = 0.5, ar: float = 0.7,
                     device="cpu"):
    """Concatenated structured prompts: x [sum N, 6144], tok [sum N], seq_offsets (numpy)."""
    import torch

    xs, ts = [], []
    for n, sd in zip(lengths, seeds):
        x, t = structured_prompt(src, embed_bits, int(n), int(sd), token_gain, ar, device)
        xs.append(x)
        ts.append(t)
    offs = np.zeros(len(lengths) + 1, np.int64)
    offs[1:] = np.cumsum(np.asarray(lengths, np.int64))
    return torch.cat(xs, 0), torch.cat(ts, 0), offs


_STEP_SCALES = os.path.join(os.path.dirname(os.path.abspath(__file__)), "step_scales.json")


def calibrated_step_scale(target_bytes: float, chunk_rows: int, student_t_frac: float = 0.0,
                          linear: bool = False) -> float:
    """Step scale k of a configuration from step_scales.json (source seed 0): the value at
    which the payload the CPU oracle writes for a seeded calibration sample is target_bytes
    per coded row, at the given rows per rANS chunk, Student-t share and codec kind."""
    with open(_STEP_SCALES) as f:
        table = json.load(f)
    for e in table["entries"]:
        if (e["target_bytes"] == float(target_bytes) and e["chunk_rows"] == int(chunk_rows)
                and abs(e["student_t_frac"] - float(student_t_frac)) < 1e-12 and e["linear"] == bool(linear)):
            return float(e["step_scale"])
    raise KeyError(f"no calibrated step scale for {target_bytes} B/row, {chunk_rows} rows per chunk, "
                   f"Student-t {student_t_frac}, linear {linear}")


def calibrated_codec(src: Source, target_bytes: float, chunk_rows: int = 16, student_t_frac: float = 0.0,
                     linear: bool = False, synthesis: bool = False) -> Codec:
    """The codec of a benchmark configuration: fitted Laplace scales at the calibrated step
    scale (decoder-side synthesis weights do not change the payload)."""
    if src.seed != 0:
        raise ValueError("step scales are calibrated for source seed 0")
    k = calibrated_step_scale(target_bytes, chunk_rows, student_t_frac, linear)
    c = codec(src, step_scale=k, linear=linear, synthesis=synthesis)
    c.note += f", step scale calibrated for {target_bytes:g} B/row"
    return c

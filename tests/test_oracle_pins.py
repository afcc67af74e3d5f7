"""Pins for the CPU oracle: each test ties it to something other than itself -- values the
pages print, hand-worked values, closed forms, library routines, invariants and exact
special cases -- so that a dropped term, a wrong sign or index or a transposed operand
in the oracle fails here.  CPU only."""
import math

import numpy as np
import pytest
import torch

import dckv_synth as S
import oracle as O
from conftest import golden


def bits_of(x):
    return x.view(torch.int16).numpy().view(np.uint16)


# ----------------------------------------------------------------------------- sizes
def test_sizes_printed_on_the_pages():
    g = golden("pages_sizes.json")
    assert O.ROW_DIM == g["row_dim"] == g["layers_full_attention"] * 2 * g["kv_heads"] * g["head_dim"]
    assert O.ROW_DIM * 2 == g["bytes_per_token_bf16"]
    assert 4096 * O.ROW_DIM * 2 == g["kv_cache_bytes_4k_tokens"] == 48 * 2 ** 20
    assert 131072 * O.ROW_DIM * 2 == g["kv_cache_bytes_128k_tokens"] == int(1.5 * 2 ** 30)
    kp = O.kept_positions(4096)
    assert len(kp) == g["kept_first_positions"] + g["kept_last_positions"]
    assert kp[:4] == [0, 1, 2, 3] and kp[4] == 4096 - 128 and kp[-1] == 4095
    assert round(len(kp) * O.ROW_DIM * 2 / 2 ** 20, 2) == g["kept_bytes_mib_rounded"]
    assert O.N_COEF == g["coefficients"] and O.N_HIDDEN == g["gelu_units"]
    assert O.ESC_LIMIT == g["escape_limit"] and O.B0_STEPS == g["drop_threshold_steps"]
    assert O.kept_positions(100) == list(range(100))


def test_blob_kept_section_is_132_rows(src, codec_literal):
    x, tok = S.prompt(src, 300, seed=3)
    blob = O.encode(bits_of(x), tok.numpy(), [0, 300], codec_literal)
    rep = O.byte_report(blob)
    assert rep["kept_rows"] == 132 * 12288 == 1622016


# ----------------------------------------------------------------------------- formats
def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    v = rng.standard_normal(100000).astype(np.float32) * np.exp(rng.uniform(-20, 20, 100000)).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.f64_to_bf16(v.astype(np.float64)), ref)
    # exact ties (round half to even) and a value just above a tie
    assert O.f64_to_bf16(np.array([1.0 + 2 ** -8]))[0] == 0x3F80  # tie -> even (1.0)
    assert O.f64_to_bf16(np.array([1.0 + 3 * 2 ** -8]))[0] == 0x3F82  # tie -> even (1.015625)
    assert O.f64_to_bf16(np.array([1.0 + 2 ** -8 + 2 ** -40]))[0] == 0x3F81
    assert np.array_equal(O.bf16_to_f64(np.array([0x3F80, 0xC000], np.uint16)), [1.0, -2.0])


# ----------------------------------------------------------------------------- transform
def test_gelu_matches_torch_library():
    h = np.linspace(-8, 8, 10001)
    ref = torch.nn.functional.gelu(torch.from_numpy(h), approximate="none").numpy()
    assert np.max(np.abs(O.gelu(h) - ref)) < 1e-14


def test_transform_is_pca_projection_when_correction_is_zero(src):
    """The pages initialise the correction to zero: then y = (x - mu) B, and for rows
    x = mu + z B^T the coefficients come back exactly (B has orthonormal columns)."""
    cod = S.codec(src, step_scale=1.0, zero_mlp=True)
    rng = np.random.default_rng(2)
    z = rng.standard_normal((7, O.N_COEF))
    x = cod.mu.astype(np.float64)[None, :] + z @ cod.basis.astype(np.float64).T
    y = O.transform(x, cod)
    bt = cod.basis.astype(np.float64)
    assert np.max(np.abs(y - z @ (bt.T @ bt))) < 1e-10  # exact identity for the stored basis
    assert np.max(np.abs(y - z)) < 1e-6  # the basis is fp32-orthonormal


def test_transform_correction_single_unit(src):
    """One hidden unit fed by one channel: y - (x - mu) B = GELU(a (x_i - mu_i)) * W2[h]."""
    cod = S.codec(src, step_scale=1.0)
    cod.w1 = np.zeros_like(cod.w1)
    cod.w2 = np.zeros_like(cod.w2)
    i, h, a = 1234, 77, 3.0
    cod.w1[i, h] = a
    rng = np.random.default_rng(3)
    cod.w2[h] = rng.standard_normal(O.N_COEF).astype(np.float32)
    x = rng.standard_normal((5, O.ROW_DIM))
    y = O.transform(x, cod)
    lin = (x - cod.mu.astype(np.float64)) @ cod.basis.astype(np.float64)
    hid = torch.nn.functional.gelu(torch.from_numpy(a * (x[:, i] - float(cod.mu[i])))).numpy()
    expect = hid[:, None] * cod.w2[h].astype(np.float64)[None, :]
    assert np.max(np.abs((y - lin) - expect)) < 1e-12
    # the correction must not leak into the linear part's channel mapping
    assert np.max(np.abs(expect)) > 0.1


def test_synthesis_correction_single_unit(src):
    """Decoder-side synthesis with one hidden unit fed by one coefficient: x_hat minus the
    linear reconstruction is GELU(a q_c Delta_c) * V2[h] (torch's GELU, fp64); without
    synthesis weights the reconstruction is the linear one."""
    cod = S.codec(src, step_scale=1.0, synthesis=True)
    c, h, a = 321, 45, 2.5
    cod.v1 = np.zeros_like(cod.v1)
    cod.v1[c, h] = a
    rng = np.random.default_rng(4)
    cod.v2 = np.zeros_like(cod.v2)
    cod.v2[h] = rng.standard_normal(O.ROW_DIM).astype(np.float32)
    q = rng.integers(-40, 41, (6, O.N_COEF))
    x = O.reconstruct(q, cod)
    lin = cod.mu.astype(np.float64)[None, :] + (q * cod.delta.astype(np.float64)) @ cod.basis.astype(np.float64).T
    u = a * q[:, c] * float(cod.delta[c])
    expect = torch.nn.functional.gelu(torch.from_numpy(u)).numpy()[:, None] * cod.v2[h].astype(np.float64)[None, :]
    assert np.max(np.abs((x - lin) - expect)) < 1e-12
    assert np.max(np.abs(expect)) > 0.01
    cod.v1 = cod.v2 = None
    assert np.array_equal(O.reconstruct(q, cod), lin)


# ----------------------------------------------------------------------------- quantiser
def test_quantise_hand_cases():
    delta = np.array([2.0, 0.5, 1.0, 1.0], np.float32)
    keep = np.array([True, True, True, False])
    y = np.array([[5.0, 1.75, -2.5, 9.0],     # 2.5 -> 2, 3.5 -> 4, -2.5 -> -2, dropped -> 0
                  [7.0, -0.25, 0.4999, 3.0],  # 3.5 -> 4, -0.5 -> 0 (even), 0.4999 -> 0
                  [255.0, 64.0, 127.5, 1.0]])  # 127.5 -> 128, 128 -> 128, 127.5 -> 128
    q, ratio = O.quantise(y, delta, keep)
    assert q.tolist() == [[2, 4, -2, 0], [4, 0, 0, 0], [128, 128, 128, 0]]
    assert ratio[0, 0] == 2.5


def test_scale_index_hand_cases():
    # beta = b / Delta in steps; s = clamp(round(8 log2(beta / 0.05)), 0, 63)
    delta = np.ones(7, np.float32)
    b = np.array([0.6, 0.05, 0.0499, 1000.0, 0.05 * 2 ** (10 / 8), 0.05 * 2 ** (10.49 / 8), 0.05 * 2 ** (10.51 / 8)],
                 np.float32)
    s, keep = O.scale_index(b, delta)
    # 8 log2(12) = 28.68 -> 29 (the literal small configuration b = 0.6 Delta)
    assert keep.tolist() == [True, True, False, True, True, True, True]
    assert s.tolist() == [29, 0, 0, 63, 10, 10, 11]


# ----------------------------------------------------------------------------- tables
def test_tables_against_scipy_laplace():
    from scipy.stats import laplace

    freq, cdf = O.laplace_tables()
    g = golden("rans_hand_cases.json")
    assert freq[0, 254] == g["scale0_freq_r0"]
    assert freq[0, 253] == freq[0, 255] == g["scale0_freq_r_pm1"]
    assert freq[0, 252] == g["scale0_freq_r_pm2"] and freq[0, 509] == g["scale0_freq_esc"]
    assert cdf[0, 254] == g["scale0_cdf_sym254"] and cdf[0, 253] == g["scale0_cdf_sym253"]
    r = np.arange(-254, 255)
    for s in range(64):
        beta = 0.05 * 2 ** (s / 8)
        p = laplace.cdf(r + 0.5, scale=beta) - laplace.cdf(r - 0.5, scale=beta)
        p_esc = 2 * laplace.sf(254.5, scale=beta)
        ideal = 1 + np.floor(np.append(p, p_esc) * (65536 - 510))
        diff = freq[s].astype(np.int64) - ideal.astype(np.int64)
        diff[254] = 0  # r = 0 also receives the remainder
        assert np.all(np.abs(diff) <= 1), s
        assert np.sum(np.abs(diff)) <= 2, s
        assert freq[s].sum() == 65536 and freq[s].min() >= 1
        assert np.array_equal(freq[s, :254], freq[s, 255:509][::-1])  # symmetric in r
        assert np.all(np.diff(freq[s, 254:509].astype(np.int64)) <= 0)  # falls with |r|
        assert cdf[s, 0] == 0 and cdf[s, -1] == 65536
        assert np.array_equal(np.diff(cdf[s].astype(np.int64)), freq[s].astype(np.int64))


# ----------------------------------------------------------------------------- rANS
def _hand_case_symbols(spec):
    if isinstance(spec, list):
        return np.array(spec)
    return np.array([253] + [254] * 31 + [253])


def test_rans_hand_worked_values():
    freq, cdf = O.laplace_tables()
    for case in golden("rans_hand_cases.json")["cases"]:
        sym = _hand_case_symbols(case["symbols"])
        scl = np.full(sym.size, case["scale"])
        states, words = O.rans_encode(sym, scl, freq, cdf)
        for lane in range(32):
            want = case["states"].get(str(lane), case["other_states"] if lane < sym.size else 65536)
            assert states[lane] == want, (case["_why"], lane)
        assert words.tolist() == case["words"]
        dec, used = O.rans_decode(states, words, scl, freq, cdf)
        assert np.array_equal(dec, sym) and used == len(case["words"])


@pytest.mark.parametrize("S_", [0, 1, 31, 32, 33, 1000, 4103])
@pytest.mark.parametrize("kind", ["laplace", "esc", "rare"])
def test_rans_round_trip_and_length_bound(S_, kind):
    freq, cdf = O.laplace_tables()
    rng = np.random.default_rng(S_ * 7 + len(kind))
    scl = rng.integers(0, 64, S_)
    if kind == "laplace":  # draw from the table itself
        sym = np.array([rng.choice(510, p=freq[s] / 65536.0) for s in scl], np.int64)
    elif kind == "esc":
        sym = np.full(S_, 509)
    else:  # the rarest symbols: one word per symbol
        sym = rng.choice([0, 508], S_)
        scl[:] = 0
    states, words = O.rans_encode(sym, scl, freq, cdf)
    dec, used = O.rans_decode(states, words, scl, freq, cdf)
    assert np.array_equal(dec, sym) and used == words.size
    ideal = -np.log2(freq[scl, sym] / 65536.0).sum()
    bits = 16 * words.size + 32 * 32
    assert bits >= ideal - 1e-6
    assert bits <= ideal + 32 * 32 + 16 * 32 + 1e-6
    assert words.size <= S_


def test_rans_detects_truncation():
    freq, cdf = O.laplace_tables()
    rng = np.random.default_rng(5)
    sym = rng.choice([0, 508], 200)
    scl = np.zeros(200, np.int64)
    states, words = O.rans_encode(sym, scl, freq, cdf)
    with pytest.raises(ValueError):
        O.rans_decode(states, words[:-3], scl, freq, cdf)


# ----------------------------------------------------------------------------- mean models
def test_mean_models_with_identity_weights():
    rng = np.random.default_rng(6)
    n = 5
    e = S.f32_to_bf16_bits(rng.standard_normal((n, 2048)))
    eye = S.f32_to_bf16_bits(np.eye(2048))
    zero = np.zeros((2048, 2048), np.uint16)
    assert np.array_equal(O.mean_even(e, eye), O.bf16_to_f64(e))
    ql = rng.integers(-300, 300, (n, 2048))
    qr = rng.integers(-300, 300, (n, 2048))
    w_left = np.concatenate([zero, eye, zero])
    w_right = np.concatenate([zero, zero, eye])
    w_emb = np.concatenate([eye, zero, zero])
    assert np.array_equal(O.mean_odd(e, ql, qr, w_emb), O.bf16_to_f64(e))
    left = O.mean_odd(e, ql, qr, w_left)
    right = O.mean_odd(e, ql, qr, w_right)
    small = np.abs(ql) <= 256
    assert np.array_equal(left[small], ql[small].astype(np.float64))  # exact in bf16
    assert np.array_equal(right[np.abs(qr) <= 256], qr[np.abs(qr) <= 256].astype(np.float64))
    big = ~small
    assert np.all(np.abs(left[big] - ql[big]) <= 1)  # bf16 spacing is 2 above 256
    assert np.array_equal(O.centres(np.array([-300.0, -126.5, 0.5, 1.5, 2.4999, 300.0])),
                          [-127, -126, 0, 2, 2, 127])


def test_checkerboard_dependencies(src, codec_centred):
    """Even centres depend on the token only; an odd row's centre depends on its two even
    neighbours (and a missing right neighbour is zero), never on odd codes."""
    x, tok = S.prompt(src, 132 + 9, seed=4)
    aux = {}
    O.encode(bits_of(x), tok.numpy(), [0, 141], codec_centred, chunk_rows=4, aux=aux)
    P = aux["per_prompt"][0]
    qe, qo = P["qe"], P["qo"]
    assert qe.shape[0] == 5 and qo.shape[0] == 4
    assert np.any(P["ce"] != 0) and np.any(P["co"] != 0)
    t_odd = tok.numpy()[4 + 1: 4 + 9: 2]
    # odd row 3 (coded row 7) has neighbours coded rows 6 and 8 = even rows 3 and 4
    base = O.mean_odd(codec_centred.embed[t_odd], qe[:4], qe[1:5], codec_centred.w_odd)
    assert np.allclose(base, P["mu_o"], rtol=0, atol=1e-9)
    bumped = qe.copy()
    bumped[4] += 50
    mu2 = O.mean_odd(codec_centred.embed[t_odd], bumped[:4], bumped[1:5], codec_centred.w_odd)
    changed = np.any(np.abs(mu2 - base) > 1e-12, axis=1)
    assert changed.tolist() == [False, False, False, True]
    # with an even number of coded rows the last odd row has no right neighbour
    x2, tok2 = S.prompt(src, 132 + 8, seed=5)
    aux2 = {}
    O.encode(bits_of(x2), tok2.numpy(), [0, 140], codec_centred, chunk_rows=4, aux=aux2)
    P2 = aux2["per_prompt"][0]
    t2 = tok2.numpy()[5:12:2]
    right = np.concatenate([P2["qe"][1:], np.zeros((1, 2048), np.int64)])
    ref = O.mean_odd(codec_centred.embed[t2], P2["qe"], right, codec_centred.w_odd)
    assert np.allclose(ref, P2["mu_o"], atol=1e-9)


# ----------------------------------------------------------------------------- RoPE
def test_rope_closed_forms():
    rng = np.random.default_rng(7)
    v = rng.standard_normal((3, 256))
    assert np.allclose(O.rope(v, [0, 0, 0]), v, atol=0)
    out = O.rope(v, [5, 1000, 131071])
    assert np.allclose(np.linalg.norm(out, axis=1), np.linalg.norm(v, axis=1), rtol=1e-13)
    e0 = np.zeros((1, 256))
    e0[0, 0] = 1.0
    r = O.rope(e0, [1])[0]
    assert abs(r[0] - math.cos(1.0)) < 1e-15 and abs(r[128] - math.sin(1.0)) < 1e-15
    e5 = np.zeros((1, 256))
    e5[0, 128 + 5] = 1.0  # second half of pair d = 5, theta = 1e7^(-10/256)
    th = 1e7 ** (-10 / 256)
    r = O.rope(e5, [3])[0]
    assert abs(r[5] + math.sin(3 * th)) < 1e-15 and abs(r[133] - math.cos(3 * th)) < 1e-15
    # rotating back by the negative position undoes it
    assert np.allclose(O.rope(out, [-5, -1000, -131071]), v, atol=1e-12)


def test_rope_touches_keys_only():
    rng = np.random.default_rng(8)
    rows = rng.standard_normal((4, O.ROW_DIM))
    out = O.output_rows(rows, np.array([0, 1, 2, 3]))
    r5 = rows.reshape(4, 6, 2, 2, 256)
    o5 = out.reshape(4, 6, 2, 2, 256)
    assert np.array_equal(o5[:, :, 1], r5[:, :, 1])
    assert np.array_equal(o5[0], r5[0])
    assert not np.allclose(o5[1, :, 0], r5[1, :, 0])


# ----------------------------------------------------------------------------- full codec
def test_lattice_rows_round_trip_exactly(src):
    """With the correction at zero and rows on the quantiser lattice, x = mu + (q Delta) B^T,
    encode recovers q exactly (escapes included) and decode returns bf16(RoPE(x))."""
    cod = S.codec(src, step_scale=None, target_bytes=220.0, zero_mlp=True)
    s_idx, keep = O.scale_index(cod.laplace_b, cod.delta)
    rng = np.random.default_rng(9)
    N = 132 + 11
    q = rng.integers(-3, 4, (N, 2048))
    q[:, :8] = rng.integers(-400, 400, (N, 8))  # escapes beyond +-127 and beyond bf16's 256
    q[:, ~keep] = 0
    x = O.reconstruct(q, cod)
    tok = rng.integers(0, 32768, N)
    aux = {}
    blob = O.encode(x, tok, [0, N], cod, chunk_rows=3, aux=aux)
    assert np.array_equal(aux["per_prompt"][0]["q"], q[4:4 + 11])
    assert aux["n_esc"] == int(np.sum(np.abs(q[4:15]) > 127))
    daux = {}
    k, v = O.decode(blob, tok, [0, N], cod, aux=daux)
    pos = np.arange(N)
    want = O.f64_to_bf16(O.output_rows(x, pos)).reshape(N, 6, 2, 2, 256)
    # coded rows: exact reconstruction; kept rows: bf16(x) stored, then RoPE
    got_k = np.transpose(k, (1, 0, 2, 3))
    got_v = np.transpose(v, (1, 0, 2, 3))
    coded = np.arange(4, 15)
    assert np.array_equal(got_k[coded], want[coded, :, 0])
    assert np.array_equal(got_v[coded], want[coded, :, 1])
    kept = O.f64_to_bf16(O.output_rows(O.bf16_to_f64(O.f64_to_bf16(x)), pos)).reshape(N, 6, 2, 2, 256)
    kp = np.array(O.kept_positions(N))
    assert np.array_equal(got_k[kp], kept[kp, :, 0]) and np.array_equal(got_v[kp], kept[kp, :, 1])


def test_linear_codec_projection_zero_centres_and_lattice_round_trip(src):
    """The linear codec ("Evidence": no correction, unconditional zero-mean tables): for
    rows x = mu + z B^T the transform returns z; every centre is 0, so a kept code's
    symbol is q + 254 (ESC beyond +-127); rows on the quantiser lattice encode to their
    codes exactly and decode to bf16(RoPE(x)).  The decoder never reads token ids."""
    cod = S.codec(src, step_scale=None, target_bytes=220.0, linear=True)
    assert cod.w1 is None and cod.embed is None
    rng = np.random.default_rng(12)
    z = rng.standard_normal((5, O.N_COEF))
    y = O.transform(cod.mu.astype(np.float64)[None, :] + z @ cod.basis.astype(np.float64).T, cod)
    assert np.max(np.abs(y - z)) < 1e-6
    s_idx, keep = O.scale_index(cod.laplace_b, cod.delta)
    N = 132 + 9
    q = rng.integers(-4, 5, (N, 2048))
    q[:, :6] = rng.integers(-300, 300, (N, 6))
    q[:, ~keep] = 0
    x = O.reconstruct(q, cod)
    aux = {}
    tok = rng.integers(0, 32768, N)
    blob = O.encode(x, tok, [0, N], cod, chunk_rows=4, aux=aux)
    P = aux["per_prompt"][0]
    assert np.array_equal(P["q"], q[4:4 + 9])
    assert not P["ce"].any() and not P["co"].any()
    sym, esc = O.symbols(P["qe"], P["ce"], keep)
    want_sym = np.where(np.abs(P["qe"][:, keep]) > 127, 509, P["qe"][:, keep] + 254)
    assert np.array_equal(sym, want_sym) and np.array_equal(esc, np.abs(P["qe"][:, keep]) > 127)
    other = rng.integers(0, 32768, N)  # different token ids: the same decode
    k, v = O.decode(blob, other, [0, N], cod)
    want = O.f64_to_bf16(O.output_rows(x, np.arange(N))).reshape(N, 6, 2, 2, 256)
    coded = np.arange(4, 13)
    assert np.array_equal(np.transpose(k, (1, 0, 2, 3))[coded], want[coded, :, 0])
    assert np.array_equal(np.transpose(v, (1, 0, 2, 3))[coded], want[coded, :, 1])


def test_batch_round_trip_payload_and_escapes(src, codec_centred):
    lens = [132 + 37, 50, 132, 132 + 64]
    x, tok, offs = S.batch(src, lens, seeds=[11, 12, 13, 14], student_t_frac=0.2)
    mu = torch.from_numpy(codec_centred.mu)
    boost = [10, 11, 175, 300]  # rows scaled far out: escapes, some beyond bf16's exact 256
    x[boost] = (mu + (x[boost].float() - mu) * 60.0).to(torch.bfloat16)
    xb = bits_of(x)
    aux = {}
    blob = O.encode(xb, tok.numpy(), offs, codec_centred, chunk_rows=8, aux=aux)
    assert aux["n_esc"] > 0
    daux = {}
    O.decode(blob, tok.numpy(), offs, codec_centred, aux=daux)
    for b, P in enumerate(aux["per_prompt"]):
        assert np.array_equal(daux["qe"][b], P["qe"]) and np.array_equal(daux["qo"][b], P["qo"])
    rep = O.byte_report(blob)
    assert rep["esc_values"] == 8 * aux["n_esc"]
    n_rows = sum(max(0, n - 132) for n in lens)
    assert rep["kept_rows"] == sum(len(O.kept_positions(n)) for n in lens) * 12288
    # stored payload vs model code length (sum -log2 f/2^16 + 64 per escape)
    n_ch = len(aux["chunks"])
    overhead = rep["header_tables"] + n_ch * (128 + 4) + rep["padding"]
    assert rep["payload"] * 8 >= aux["code_bits"]
    assert rep["payload"] * 8 <= aux["code_bits"] + 8 * overhead + 16 * 32 * n_ch
    assert n_rows == 101


def test_corrupt_blobs_are_rejected(src, codec_literal):
    x, tok = S.prompt(src, 140, seed=6)
    blob = bytearray(O.encode(bits_of(x), tok.numpy(), [0, 140], codec_literal, chunk_rows=2))
    with pytest.raises(ValueError):
        O.decode(bytes(blob[:40]), tok.numpy(), [0, 140], codec_literal)
    bad = bytearray(blob)
    bad[0] ^= 1
    with pytest.raises(ValueError):
        O.decode(bytes(bad), tok.numpy(), [0, 140], codec_literal)
    with pytest.raises(ValueError):
        O.decode(bytes(blob), tok.numpy(), [0, 141], codec_literal)
    hdr = O.parse_blob(blob)
    cut = hdr["off_streams"] + hdr["chunk_offsets"][1] - 6  # last words of chunk 0 gone
    bad = bytearray(blob)
    bad[hdr["off_streams"] + 4 * 32] = 0xFF  # an absurd escape count
    with pytest.raises(ValueError):
        O.decode(bytes(bad), tok.numpy(), [0, 140], codec_literal)
    assert cut > 0

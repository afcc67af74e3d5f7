"""GPU codec vs the CPU oracle, element by element, through the C ABI.

Parity rules (one GPU, seeded synthetic inputs):
  codes      bit-exact, except |dq| = 1 flips where the oracle's y / Delta lies within
             1e-3 of a half-step boundary, and such flips are at most 0.1% of codes;
  centres    equal to the oracle's centres computed from the same codes, except where the
             oracle's mean lies within 1e-4 of a half-step boundary (fp32 vs fp64 sums);
  bitstream  given the GPU's codes and centres, the oracle coder and container produce
             the GPU's blob byte for byte;
  rows       decoded K/V within 1e-3 relative Frobenius of the oracle's decode of the
             same blob (both rounded to bf16), and GPU decode reproduces the GPU encoder's
             codes exactly;
  determinism  repeated calls give identical blobs and rows.
"""
import copy

import numpy as np
import pytest
import torch

import dckv_synth as S
import learned_kv_cache_dckv_b200 as D
import oracle as O

pytestmark = pytest.mark.gpu

FLIP_WINDOW = 1e-3
FLIP_MAX_FRAC = 1e-3
CENTRE_WINDOW = 1e-4
ROW_TOL = 1e-3


class _CAI:
    def __init__(self, ptr, shape, typestr):
        self.__cuda_array_interface__ = dict(shape=shape, typestr=typestr, data=(ptr, False), version=3)


def bits(x):
    return x.detach().cpu().view(torch.int16).numpy().view(np.uint16)


_GPU_CODECS = {}


def gpu_codec(np_codec, chunk_rows=0):
    key = (id(np_codec), chunk_rows)
    if key not in _GPU_CODECS:
        _GPU_CODECS[key] = D.Codec(D.upload_params(np_codec), 0, chunk_rows)
    return _GPU_CODECS[key]


def make_batch(src, cod, lens, seeds, boost=(), boost_gain=60.0, student_t=0.0):
    x, tok, offs = S.batch(src, lens, seeds, student_t_frac=student_t, device="cuda")
    vocab = cod.embed.shape[0] if cod.embed is not None else 0
    if vocab > 1 << 16:  # every third token id from the vocabulary's rows at and past 2^16
        tok[::3] = (1 << 16) + tok[::3] % (vocab - (1 << 16))
    if boost:
        mu = torch.from_numpy(cod.mu).cuda()
        idx = torch.tensor(list(boost), device="cuda")
        x[idx] = (mu + (x[idx].float() - mu) * boost_gain).to(torch.bfloat16)
    return x, tok, offs


def encode_gpu(gc, x, tok, offs):
    blob = gc.encode(x, tok, offs)
    torch.cuda.synchronize()
    status = int(gc.status.item())
    size = int(gc.blob_size.item())
    v = D.dckv_ws_offsets(gc.handle, offs, 0)
    ws = gc._ws
    n, ne = v["n_rows"], v["ne_pad"]
    q32 = gc.workspace_codes(offs, 0)
    K = gc.k_eff
    cen8 = ws[v["cen8"]: v["cen8"] + n * K].view(torch.int8).reshape(n, K).cpu().numpy()
    row_slot = ws[v["row_slot"]: v["row_slot"] + 4 * n].view(torch.int32).cpu().numpy()
    cnt = ws[v["counters"]: v["counters"] + 8].view(torch.int32).cpu().numpy()
    return dict(blob_dev=blob, blob=blob[:size].cpu().numpy().tobytes(), size=size, status=status, q32=q32,
                cen=cen8[row_slot] if n else cen8, refined_codes=int(cnt[0]), refined_rows=int(cnt[1]))


def decode_gpu(gc, blob_dev, size, tok, offs):
    k, v = gc.decode(blob_dev, size, tok, offs)
    torch.cuda.synchronize()
    w = D.dckv_ws_offsets(gc.handle, offs, 1)
    n = w["n_rows"]
    q16 = gc.workspace_codes(offs, 1)
    return k, v, int(gc.status.item()), q16


def split_gpu_codes(gc, np_codec, res, tok, offs):
    """Per prompt: the GPU's codes and centres (centres of dropped components are 0; they
    are never used)."""
    lay = O.prompt_layout(np.diff(offs))
    keep = O.scale_index(np_codec.laplace_b, np_codec.delta)[1]
    out = []
    for L in lay:
        q = res["q32"][L["row_base"]: L["row_base"] + L["n"]].astype(np.int64)
        cen = np.zeros((L["n"], 2048), np.int64)
        cen[:, keep] = res["cen"][L["row_base"]: L["row_base"] + L["n"]]
        out.append(dict(q=q, qe=q[0::2], qo=q[1::2], ce=cen[0::2], co=cen[1::2]))
    return out


def near_half(v, window):
    f = np.abs(v - np.floor(v) - 0.5)
    return f < window


def check_codes(gpu_q, ora):
    d = gpu_q - ora["q"]
    bad = d != 0
    if bad.any():
        assert np.all(np.abs(d[bad]) == 1), "code differs by more than one step"
        assert np.all(near_half(ora["ratio"][bad], FLIP_WINDOW)), "flip away from a half-step boundary"
    assert bad.sum() <= FLIP_MAX_FRAC * max(1, gpu_q.size)
    return int(bad.sum())


def check_centres(gc_codes, np_codec, tok, offs):
    """Oracle centres from the GPU's own codes vs the GPU's centres."""
    lay = O.prompt_layout(np.diff(offs))
    tok_np = tok.cpu().numpy().astype(np.int64)
    mism = 0
    total = 0
    for L, G in zip(lay, gc_codes):
        t0 = L["tok_base"] + 4
        te = tok_np[t0: t0 + L["n"]: 2]
        to = tok_np[t0 + 1: t0 + L["n"]: 2]
        for par, toks in ((0, te), (1, to)):
            if toks.size == 0:
                continue
            if par == 0:
                mu = O.codec_means_even(np_codec, toks)
            else:
                qe = G["qe"]
                right = np.concatenate([qe[1:], np.zeros((1, 2048), np.int64)])[: toks.size]
                mu = O.codec_means_odd(np_codec, toks, qe[: toks.size], right)
            keep = O.scale_index(np_codec.laplace_b, np_codec.delta)[1]
            ora_c = O.centres(mu)[:, keep]
            gpu_c = (G["ce"] if par == 0 else G["co"])[:, keep]
            mu = mu[:, keep]
            bad = ora_c != gpu_c
            if bad.any():
                assert np.all(np.abs(ora_c[bad] - gpu_c[bad]) == 1)
                assert np.all(near_half(mu[bad], CENTRE_WINDOW)), "centre differs away from a boundary"
            mism += int(bad.sum())
            total += bad.size
    assert mism <= 1e-4 * max(total, 1)
    return mism


def rel_frob(a, b):
    a = a.astype(np.float64)
    b = b.astype(np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def token_rows(k_bits, v_bits, tok_idx):
    """Rows of the [6][T][2][256] K and V outputs at the given token indices, as fp64
    [rows][2 * 6,144] (K then V)."""
    kk = O.bf16_to_f64(k_bits[:, tok_idx]).transpose(1, 0, 2, 3).reshape(len(tok_idx), -1)
    vv = O.bf16_to_f64(v_bits[:, tok_idx]).transpose(1, 0, 2, 3).reshape(len(tok_idx), -1)
    return np.concatenate([kk, vv], axis=1)


def row_errors(got, want):
    """(relative Frobenius error over all the given rows, largest relative error of one
    row) for fp64 rows [rows][d]."""
    if got.shape[0] == 0:
        return 0.0, 0.0
    d = np.linalg.norm(got - want, axis=1)
    w = np.linalg.norm(want, axis=1)
    frob = float(np.sqrt(np.sum(d * d)) / max(np.sqrt(np.sum(w * w)), 1e-30))
    return frob, float(np.max(d / np.maximum(w, 1e-30)))


def coded_token_index(lay):
    """Token indices of every coded row of a batch (prompt order, row order)."""
    parts = [np.arange(L["tok_base"] + 4, L["tok_base"] + 4 + L["n"]) for L in lay]
    return np.concatenate(parts) if parts else np.zeros(0, np.int64)


def check_rows(k, v, k_o, v_o, lay, q_gpu, cod, dec_aux, centre_mismatches):
    """Decoded rows against the oracle.
    (1) The spec measure: relative Frobenius error against the oracle's decode of the
        same blob, within 1e-3, taken over the coded rows alone (kept rows are stored
        verbatim and would dilute it).
    (2) The oracle's decoder computes its own centres; where one differs by one from the
        centre the GPU encoder coded with (the 1e-4 rule of check_centres), the oracle
        decodes that code one off.  So its codes must equal the GPU's except for at most
        that many +-1 differences.
    (3) Every coded row on its own: the oracle's reconstruction of the GPU's codes (RoPE,
        bf16) against the GPU's row, relative error within 1e-3 for the worst row.
    (4) Kept rows on their own, row by row, against the oracle's decode.
    Returns (Frobenius error, worst row error)."""
    kg, vg = bits(k), bits(v)
    idx = coded_token_index(lay)
    got = token_rows(kg, vg, idx)
    frob, _ = row_errors(got, token_rows(k_o, v_o, idx))
    assert frob <= ROW_TOL, frob
    n_diff = 0
    for L, qe, qo in zip(lay, dec_aux["qe"], dec_aux["qo"]):
        q = np.zeros((L["n"], 2048), np.int64)
        q[0::2], q[1::2] = qe, qo
        d = q - q_gpu[L["row_base"]: L["row_base"] + L["n"]]
        assert np.all(np.abs(d) <= 1), "oracle decode differs from the GPU's codes by more than one step"
        n_diff += int(np.count_nonzero(d))
    assert n_diff <= centre_mismatches, (n_diff, centre_mismatches)
    if idx.size:
        pos = np.concatenate([np.arange(4, 4 + L["n"]) for L in lay])
        want = O.f64_to_bf16(O.output_rows(O.reconstruct(q_gpu.astype(np.int64), cod), pos)).reshape(-1, 6, 2, 2, 256)
        want = np.concatenate([O.bf16_to_f64(want[:, :, 0]).reshape(idx.size, -1),
                               O.bf16_to_f64(want[:, :, 1]).reshape(idx.size, -1)], axis=1)
        _, worst = row_errors(got, want)
        assert worst <= ROW_TOL, worst
    else:
        worst = 0.0
    kept = np.setdiff1d(np.arange(kg.shape[1]), idx)
    kf, kw = row_errors(token_rows(kg, vg, kept), token_rows(k_o, v_o, kept))
    assert kf <= ROW_TOL and kw <= ROW_TOL, (kf, kw)
    return frob, worst


def full_check(src, np_codec, lens, seeds, chunk_rows=0, boost=(), boost_gain=60.0, student_t=0.0,
               expect_escapes=False, expect_big=False):
    gc = gpu_codec(np_codec, chunk_rows)
    G = gc.handle
    x, tok, offs = make_batch(src, np_codec, lens, seeds, boost, boost_gain, student_t)
    res = encode_gpu(gc, x, tok, offs)
    assert res["status"] == D.DCKV_OK, D.STATUS_NAMES[res["status"]]
    xb = bits(x)
    ora = O.analyse(xb, tok.cpu().numpy(), offs, np_codec)
    codes = split_gpu_codes(gc, np_codec, res, tok, offs)
    flips = sum(check_codes(c["q"], o) for c, o in zip(codes, ora))
    mism = check_centres(codes, np_codec, tok, offs)
    # bitstream: the oracle's coder and container on the GPU's codes and centres
    aux = {}
    G = D.dckv_codec_info(gc.handle)["chunk_rows"]
    assert G == (chunk_rows or 16)
    ora_blob = O.assemble_blob(xb, offs, codes, np_codec.laplace_b, np_codec.delta, G, aux=aux)
    assert len(ora_blob) == res["size"]
    if ora_blob != res["blob"]:
        hdr = O.parse_blob(ora_blob)
        first = next(i for i in range(len(ora_blob)) if ora_blob[i] != res["blob"][i])
        pytest.fail(f"blob differs first at byte {first} (streams start at {hdr['off_streams']})")
    if expect_escapes:
        assert aux["n_esc"] > 0
    if boost:
        assert res["refined_rows"] >= 1  # far-out rows are recomputed whole
    # decode on the GPU, and the oracle's decode of the same blob
    k, v, st, q16 = decode_gpu(gc, res["blob_dev"], res["size"], tok, offs)
    assert st == D.DCKV_OK, D.STATUS_NAMES[st]
    small = np.abs(res["q32"]) < 2048
    assert np.array_equal(q16[small], res["q32"][small].astype(np.float32))
    if expect_big:
        assert (~small).any()
    dec_aux = {}
    k_o, v_o = O.decode(res["blob"], tok.cpu().numpy(), offs, np_codec, aux=dec_aux)
    row_frob, row_worst = check_rows(k, v, k_o, v_o, O.prompt_layout(np.diff(offs)), res["q32"], np_codec,
                                     dec_aux, mism)
    return dict(row_frob=row_frob, row_worst=row_worst, gc=gc, x=x, tok=tok, offs=offs, res=res, flips=flips, centre_mismatch=mism, k=k, v=v, aux=aux)


# ------------------------------------------------------------------------------------ tests
def test_tables_scale_and_mask_identical(codec_55, codec_literal):
    freq, cdf = O.laplace_tables()
    for cod in (codec_55, codec_literal):
        gc = gpu_codec(cod)
        g_cdf, g_scale, g_keep, exps = D.dckv_codec_export(gc.handle)
        assert np.array_equal(g_cdf.astype(np.int64), cdf[:, :510].astype(np.int64))
        s, keep = O.scale_index(cod.laplace_b, cod.delta)
        assert np.array_equal(g_keep.astype(bool), keep)
        assert np.array_equal(g_scale.astype(np.int64), s)
        assert gc.k_eff == int(keep.sum())


def test_compacted_gemm_shapes_and_inverse_lo_cut(src, codec_55):
    """The GEMMs run on kept components only: K_eff rounded up to 64 (code arrays, K of the
    GEMMs reading codes) and to 256 (M of the transform and the odd mean model).  The
    inverse adds the lo half of its split operand Delta_c B[:, c] 2^p for the first
    inv_lo_k kept components only: the smallest multiple of 64 past which the lo halves
    carry at most 2^-30 of the expected signal energy sum E[q_m^2] |A_m|^2, with
    E[q^2] = 2 beta^2 + 1/12 under each component's Laplace scale beta (in steps).  The
    rule is recomputed here from the codec's parameters in fp64."""
    gc = gpu_codec(codec_55)
    shp = D.dckv_codec_gemm_shape(gc.handle)
    k = gc.k_eff
    assert shp["k_eff"] == k and shp["kw"] == max(64, -(-k // 64) * 64) and shp["mp"] == max(256, -(-k // 256) * 256)
    keep = O.scale_index(codec_55.laplace_b, codec_55.delta)[1]
    kl = np.nonzero(keep)[0]
    p_inv = int(D.dckv_codec_export(gc.handle)[3][2])
    a = (codec_55.delta.astype(np.float64)[kl, None] * codec_55.basis.astype(np.float64).T[kl]) * 2.0 ** p_inv
    hi = a.astype(np.float16).astype(np.float64)
    lo = (a - hi).astype(np.float16).astype(np.float64)
    beta = (codec_55.laplace_b.astype(np.float64) / codec_55.delta.astype(np.float64))[kl]
    eq2 = 2.0 * beta ** 2 + 1.0 / 12.0
    total = np.sum(eq2 * ((hi + lo) ** 2).sum(axis=1))
    tail = np.cumsum((eq2 * (lo ** 2).sum(axis=1))[::-1])[::-1]
    ok = np.nonzero(tail <= total / 2.0 ** 30)[0]
    cut = int(ok[0]) if ok.size else k
    assert shp["inv_lo_k"] == min(shp["kw"], -(-cut // 64) * 64)
    assert 0 < shp["inv_lo_k"] < shp["kw"]  # the cut is in use on this codec


def test_vocabulary_tables_kept_components(codec_55, codec_centred):
    """The per-vocabulary tables hold the kept components only, column kc = compact index,
    row stride kw: the even table is the even rows' centres themselves (int8), equal to
    the oracle's centres of mu = e(token) W_e except where mu lies within 1e-4 of a
    half-step boundary (fp32 vs fp64 sums); the odd table is e(token) W_oE within fp32
    accumulation error (2^-12 of sum |e||W|); pad columns are zero.  Checked on 2,048
    sampled vocabulary rows plus the first and last."""
    for cod in (codec_55, codec_centred):
        gc = gpu_codec(cod)
        shp = D.dckv_codec_gemm_shape(gc.handle)
        k, kw = shp["k_eff"], shp["kw"]
        V = cod.embed.shape[0]
        te_p, to_p = D.dckv_codec_tables(gc.handle)
        te = torch.as_tensor(_CAI(te_p, (V, kw), "|i1"), device="cuda").cpu().numpy()
        to = torch.as_tensor(_CAI(to_p, (V, kw), "<f4"), device="cuda").cpu().numpy()
        kl = np.nonzero(O.scale_index(cod.laplace_b, cod.delta)[1])[0]
        rows = np.unique(np.concatenate([[0, V - 1], np.random.default_rng(7).choice(V, 2048, replace=False)]))
        e = O.bf16_to_f64(cod.embed[rows])
        w_e = O.bf16_to_f64(cod.w_even)[:, kl]
        w_o = O.bf16_to_f64(cod.w_odd[:2048])[:, kl]
        mu_e = e @ w_e
        near = np.abs(np.abs(mu_e - np.floor(mu_e)) - 0.5) < CENTRE_WINDOW
        ce = O.centres(mu_e)
        got = te[rows, :k].astype(np.int64)
        assert np.array_equal(got[~near], ce[~near])
        assert np.all(np.abs(got[near] - ce[near]) <= 1)
        assert np.all(te[:, k:] == 0) and np.all(to[:, k:] == 0)
        mu_o = e @ w_o
        bound = 2.0 ** -12 * (np.abs(e) @ np.abs(w_o)) + 1e-30
        assert np.all(np.abs(to[rows, :k].astype(np.float64) - mu_o) <= bound)
    assert np.count_nonzero(got) > got.size // 4  # codec_centred: the even centres are not all 0


def test_hidden_layer_identical_across_batch_sizes(src, codec_55):
    """A batch with at least as many 256-token tiles as SMs sums the correction layer's four
    K parts in registers; a small batch writes the parts and sums them in a second kernel.
    Both add the same fp32 partials in the same order, so the hidden units (hi/lo fp16) and
    the codes of a prompt are bit-identical whichever batch it is coded in."""
    gc = gpu_codec(codec_55)
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    n_big = -(-n_sm * 256 // (4096 - 132)) + 1  # prompts of 4,096 tokens: tiles >= SMs
    got = {}
    for lens in ([4096], [4096] * n_big):
        x, tok, offs = S.batch(src, lens, list(range(100, 100 + len(lens))), device="cuda")
        gc.encode(x, tok, offs)
        torch.cuda.synchronize()
        assert int(gc.status.item()) == 0
        v = D.dckv_ws_offsets(gc.handle, offs, 0)
        assert -(-v["n_rows"] // 256) >= n_sm or len(lens) == 1
        n0 = 4096 - 132  # the first prompt's coded rows come first in either batch
        g = gc._ws[v["g16"]: v["g16"] + 2 * 512 * n0].view(torch.int16).cpu().numpy()
        got[len(lens)] = (g, gc.workspace_codes(offs, 0, rows=np.arange(n0)))
        del x
    (g1, q1), (g2, q2) = got[1], got[n_big]
    assert np.array_equal(g1, g2)
    assert np.array_equal(q1, q2)
    assert np.count_nonzero(g1) > g1.size // 2


def test_parity_literal_small_config(src, codec_literal):
    # one prompt of 256 tokens (124 coded rows) plus ragged neighbours and degenerate prompts
    full_check(src, codec_literal, [256, 700, 50, 132, 133, 134], seeds=[0, 1, 2, 3, 4, 5])


def test_parity_fitted_rate_several_tiles(src, codec_55):
    r = full_check(src, codec_55, [132 + 600, 132 + 301], seeds=[7, 8])
    assert r["flips"] <= 0.001 * 901 * 2048


def test_parity_centres_escapes_and_big_codes(src, codec_centred):
    # rows pushed far out: escapes beyond +-127 and codes beyond the fp16-exact 2048
    full_check(src, codec_centred, [132 + 90, 132 + 41, 140], seeds=[11, 12, 13], chunk_rows=8,
               boost=(4, 9, 30, 60, 223 + 4, 223 + 50), boost_gain=400.0, expect_escapes=True, expect_big=True)


def test_parity_token_ids_past_2_16(src, codec_centred):
    """A vocabulary of 70,000 rows, every third token id at or above 2^16: the even-centre
    and odd tables are indexed by token id times their row stride, so these ids take the
    tables' upper rows (and 64-bit offsets at the largest vocabularies)."""
    import copy

    cod = copy.copy(codec_centred)
    extra = np.random.default_rng(99).standard_normal((70000 - S.VOCAB, cod.embed.shape[1])).astype(np.float32)
    cod.embed = np.concatenate([cod.embed, S.f32_to_bf16_bits(extra)], axis=0)
    r = full_check(src, cod, [132 + 300, 132 + 77], seeds=[21, 22], chunk_rows=8)
    assert (r["tok"].cpu().numpy() >= 1 << 16).sum() > 100


def test_parity_student_t_rows(src, codec_55):
    full_check(src, codec_55, [132 + 256], seeds=[21], chunk_rows=16, student_t=0.25)


_FEW_KEPT = {}


@pytest.mark.parametrize("step_scale,chunk_rows,k_range", [(60.0, 0, (8, 31)), (120.0, 5, (1, 7)), (200.0, 0, (0, 0))])
def test_parity_fewer_than_32_kept_components(src, step_scale, chunk_rows, k_range):
    # coarse steps drop most components: a lane's component wraps several times per step,
    # and with none kept the streams hold only their final states
    if step_scale not in _FEW_KEPT:
        _FEW_KEPT[step_scale] = S.codec(src, step_scale=step_scale)
    cod = _FEW_KEPT[step_scale]
    k = int(O.scale_index(cod.laplace_b, cod.delta)[1].sum())
    assert k_range[0] <= k <= k_range[1]
    full_check(src, cod, [132 + 200, 140, 132 + 37], seeds=[41, 42, 43], chunk_rows=chunk_rows)


_LINEAR = {}


@pytest.mark.parametrize("variant", ["literal", "fitted"])
def test_parity_linear_codec(src, variant):
    # the linear codec: no correction, unconditional zero-mean tables (all centres 0)
    if variant not in _LINEAR:
        _LINEAR[variant] = (S.codec(src, step_scale=1.0, literal_b=True, linear=True) if variant == "literal"
                            else S.codec(src, step_scale=None, target_bytes=220.0, linear=True))
    cod = _LINEAR[variant]
    r = full_check(src, cod, [132 + 300, 140, 132 + 77], seeds=[71, 72, 73])
    assert not r["res"]["cen"].any()
    # without mean models the token ids are not needed: NULL gives the same blob and rows
    gc = r["gc"]
    blob2 = gc.encode(r["x"], None, r["offs"])
    torch.cuda.synchronize()
    assert int(gc.status.item()) == D.DCKV_OK
    size = int(gc.blob_size.item())
    assert blob2[:size].cpu().numpy().tobytes() == r["res"]["blob"]
    k2, v2 = gc.decode(blob2, size, None, r["offs"])
    torch.cuda.synchronize()
    assert int(gc.status.item()) == D.DCKV_OK
    assert torch.equal(k2, r["k"]) and torch.equal(v2, r["v"])


_SYNTH = {}


@pytest.mark.parametrize("big", [False, True])
def test_parity_decoder_side_synthesis(src, big):
    # decode adds GELU((q Delta) V1) V2 to the linear synthesis; rows pushed far out reach
    # codes beyond 2048, which the fix-up recomputes with the synthesis term included
    if "c" not in _SYNTH:
        _SYNTH["c"] = S.codec(src, step_scale=None, target_bytes=220.0, embed_std=1.0, mean_gain=1.0,
                              neigh_gain=40.0, synthesis=True, synthesis_gain=10.0)
    cod = _SYNTH["c"]
    if big:
        r = full_check(src, cod, [132 + 90, 140, 132 + 41], seeds=[81, 82, 83], chunk_rows=8,
                       boost=(4, 30, 60, 90 + 8), boost_gain=400.0, expect_big=True)
    else:
        r = full_check(src, cod, [132 + 300, 132 + 77], seeds=[84, 85])
    # the synthesis term is not negligible: the oracle's linear decode of the same blob
    # lies well outside the row tolerance
    lin = copy.copy(cod)
    lin.v1 = lin.v2 = None
    k_l, v_l = O.decode(r["res"]["blob"], r["tok"].cpu().numpy(), r["offs"], lin)
    assert rel_frob(O.bf16_to_f64(bits(r["k"])), O.bf16_to_f64(k_l)) > 20 * ROW_TOL


def test_determinism(src, codec_55):
    gc = gpu_codec(codec_55)
    x, tok, offs = make_batch(src, codec_55, [132 + 500, 300], [31, 32])
    a = encode_gpu(gc, x, tok, offs)
    b = encode_gpu(gc, x, tok, offs)
    assert a["blob"] == b["blob"]
    k1, v1, _, _ = decode_gpu(gc, a["blob_dev"], a["size"], tok, offs)
    k1, v1 = k1.clone(), v1.clone()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        k2, v2 = gc.decode(a["blob_dev"], a["size"], tok, offs, stream=s)
    s.synchronize()
    assert torch.equal(k1, k2) and torch.equal(v1, v2)


def test_corrupt_blobs_report_status(src, codec_55):
    gc = gpu_codec(codec_55)
    x, tok, offs = make_batch(src, codec_55, [132 + 200], [41])
    res = encode_gpu(gc, x, tok, offs)
    blob = res["blob_dev"]
    hdr = O.parse_blob(res["blob"])
    # 1: truncated blob
    _, _, st, _ = decode_gpu(gc, blob, res["size"] - 10, tok, offs)
    assert st == D.DCKV_ECORRUPT
    # 2: wrong prompt length
    _, _, st, _ = decode_gpu(gc, blob, res["size"], tok, np.array([0, 331]))
    assert st in (D.DCKV_ECORRUPT,)
    # 3: words of a chunk overwritten
    bad = blob.clone()
    p = hdr["off_streams"] + hdr["chunk_offsets"][0] + 140
    bad[p: p + 64] = 0xA5
    _, _, st, _ = decode_gpu(gc, bad, res["size"], tok, offs)
    assert st == D.DCKV_ECORRUPT
    # 4: escape count inflated
    bad = blob.clone()
    bad[hdr["off_streams"] + hdr["chunk_offsets"][1] + 128] = 200
    _, _, st, _ = decode_gpu(gc, bad, res["size"], tok, offs)
    assert st == D.DCKV_ECORRUPT
    # a clean decode still works afterwards
    _, _, st, _ = decode_gpu(gc, blob, res["size"], tok, offs)
    assert st == D.DCKV_OK


def test_capacity_error(src, codec_55):
    gc = gpu_codec(codec_55)
    x, tok, offs = make_batch(src, codec_55, [132 + 64], [51])
    small = torch.empty(1024 * 1024, dtype=torch.uint8, device="cuda")  # below the kept rows' 1.55 MiB
    gc.encode(x, tok, offs, blob=small)
    torch.cuda.synchronize()
    assert int(gc.status.item()) == D.DCKV_ECAPACITY
    with pytest.raises(D.DckvError):
        D.dckv_encode(gc.handle, x, tok, offs, small, gc.blob_size, gc.status,
                      torch.empty(1024, dtype=torch.uint8, device="cuda"))


def sample_rows(lay, rng, n_random, chunk_rows):
    """Coded rows (batch-wide indices) for the full-size checks: n_random drawn at random,
    plus in every prompt its first three and last three coded rows (both parities at both
    ends, the last odd row's missing right neighbour included), the rows on both sides of
    the first chunk boundary of each parity, and the rows around every multiple of 2^16
    of the prompt's own and of the batch-wide coded-row index."""
    n = sum(L["n"] for L in lay)
    picks = set(int(r) for r in rng.choice(n, min(n_random, n), replace=False)) if n else set()
    for L in lay:
        m, b = L["n"], L["row_base"]
        rel = {0, 1, 2, m - 3, m - 2, m - 1}
        g = 2 * chunk_rows  # first row of the second chunk of each parity: 2G (even), 2G + 1 (odd)
        rel |= {g - 2, g - 1, g, g + 1}
        for mark in range(1 << 16, m + 2, 1 << 16):
            rel |= {mark - 2, mark - 1, mark, mark + 1}
        picks |= {b + j for j in rel if 0 <= j < m}
    for mark in range(1 << 16, n + 2, 1 << 16):
        picks |= {r for r in (mark - 2, mark - 1, mark, mark + 1) if 0 <= r < n}
    return np.array(sorted(picks), np.int64)


def check_sampled(gc, cod, res, x, tok, offs, rows, k, v):
    """Full-size parity on selected coded rows (batch-wide indices):
    codes     the oracle's transform and quantiser on the rows' inputs (flip rule);
    centres   the oracle's mean models on the rows' tokens and, for odd rows, the GPU's
              own codes of both even neighbours (zero past a prompt's last even row),
              against the GPU encoder's centres (1e-4 rule); encoder and decoder share
              the tables, so this is what catches a centre both would get wrong;
    rows      the oracle's reconstruction of the GPU's codes, RoPE'd at each row's
              position, against the decoded K and V: relative Frobenius over the rows and
              the largest single-row error, both within 1e-3.
    Returns (flips, centre mismatches, row Frobenius error, worst row error)."""
    lay = O.prompt_layout(np.diff(offs))
    starts = np.array([L["row_base"] for L in lay])
    pidx = np.searchsorted(starts, rows, side="right") - 1
    rel = rows - starts[pidx]
    tbase = np.array([L["tok_base"] for L in lay])[pidx]
    tok_rows = tbase + 4 + rel
    xb = bits(x)
    keep = O.scale_index(cod.laplace_b, cod.delta)[1]
    q_o, ratio = O.quantise(O.transform(xb[tok_rows], cod), cod.delta, keep)
    q_gpu = res["q32"][rows].astype(np.int64)
    flips = check_codes(q_gpu, dict(q=q_o, ratio=ratio))
    # centres
    tok_np = tok.cpu().numpy().astype(np.int64)
    n_rel = np.array([L["n"] for L in lay])[pidx]
    mism = 0
    for par in (0, 1):
        sel = np.nonzero((rel & 1) == par)[0]
        if sel.size == 0:
            continue
        toks = tok_np[tok_rows[sel]]
        if par == 0:
            mu = O.codec_means_even(cod, toks)
        else:
            left = res["q32"][rows[sel] - 1].astype(np.int64)
            has_right = rel[sel] + 1 < n_rel[sel]
            right = np.zeros((sel.size, 2048), np.int64)
            right[has_right] = res["q32"][rows[sel][has_right] + 1]
            mu = O.codec_means_odd(cod, toks, left, right)
        ora_c = O.centres(mu)[:, keep]
        gpu_c = res["cen"][rows[sel]].astype(np.int64)
        bad = ora_c != gpu_c
        if bad.any():
            assert np.all(np.abs(ora_c[bad] - gpu_c[bad]) == 1)
            assert np.all(near_half(mu[:, keep][bad], CENTRE_WINDOW)), "centre differs away from a boundary"
        mism += int(bad.sum())
    assert mism <= 1e-4 * max(1, rows.size * int(keep.sum()))
    # decoded rows
    xh = O.reconstruct(q_gpu, cod)
    want = O.output_rows(xh, 4 + rel)
    want = O.bf16_to_f64(O.f64_to_bf16(want)).reshape(-1, 6, 2, 2, 256)
    want = np.concatenate([want[:, :, 0].reshape(rows.size, -1), want[:, :, 1].reshape(rows.size, -1)], axis=1)
    frob, worst = row_errors(token_rows(bits(k), bits(v), tok_rows), want)
    assert frob <= ROW_TOL, frob
    assert worst <= ROW_TOL, worst
    return flips, mism, frob, worst


def full_size_check(src, cod, lens, seeds, chunk_rows, student_t=0.0, n_random=320):
    """One full-size configuration: sampled rows against the oracle (check_sampled), the
    whole blob re-coded by the oracle coder from the GPU's codes and centres, the payload
    against the model code length, and the exact code round trip through the GPU decoder."""
    gc = gpu_codec(cod, chunk_rows)
    x, tok, offs = make_batch(src, cod, lens, seeds, student_t=student_t)
    res = encode_gpu(gc, x, tok, offs)
    assert res["status"] == D.DCKV_OK, D.STATUS_NAMES[res["status"]]
    lay = O.prompt_layout(np.diff(offs))
    G = D.dckv_codec_info(gc.handle)["chunk_rows"]
    assert G == (chunk_rows or 16)
    codes = split_gpu_codes(gc, cod, res, tok, offs)
    aux = {}
    ora_blob = O.assemble_blob(bits(x), offs, codes, cod.laplace_b, cod.delta, G, aux=aux)
    assert len(ora_blob) == res["size"] and ora_blob == res["blob"]
    kept = sum(L["N"] - L["n"] for L in lay)
    payload = res["size"] - kept * 12288
    assert payload <= 1.05 * aux["code_bits"] / 8, (payload, aux["code_bits"] / 8)
    if student_t > 0:
        assert aux["n_esc"] > 0  # heavy-tailed rows force escapes
    k, v, status, q16 = decode_gpu(gc, res["blob_dev"], res["size"], tok, offs)
    assert status == D.DCKV_OK
    small = np.abs(res["q32"]) < 2048
    assert np.array_equal(q16[small], res["q32"][small].astype(np.float32))
    rows = sample_rows(lay, np.random.default_rng(sum(seeds)), n_random, G)
    flips, mism, frob, worst = check_sampled(gc, cod, res, x, tok, offs, rows, k, v)
    n = sum(L["n"] for L in lay)
    print(f"{len(lens)} x {lens[0]}: {rows.size} sampled rows, {flips} flips, {mism} centre mismatches, "
          f"rows {frob:.2e} (worst {worst:.2e}), payload {payload / n:.1f} B/row, {aux['n_esc']} escapes")
    return dict(res=res, aux=aux, payload=payload, n=n, rows=rows)


def test_full_size_4k_prompt_sampled(src, codec_55):
    """4,096-token prompt at about 220 B/token: sampled and boundary rows against the
    oracle (codes, centres, decoded rows), every chunk re-coded by the oracle coder, and
    the payload against the model code length."""
    r = full_size_check(src, codec_55, [4096], [100], 0)
    assert 150 <= r["payload"] / r["n"] <= 300


_FULL_CODECS = {}


def _full_codec(src, target, chunk_rows, student_t):
    key = (target, chunk_rows, student_t)
    if key not in _FULL_CODECS:
        _FULL_CODECS[key] = S.calibrated_codec(src, target, chunk_rows, student_t)
    return _FULL_CODECS[key]


# the larger configurations: (prompt lengths, target bytes per coded row, Student-t fraction,
# rows per rANS chunk), each with the step scale calibrated for its rate.  At ~110 B per row a
# chunk's fixed 136 bytes need 32 rows to stay within the 5% payload bound.
FULL_CONFIGS = {
    "32k_220B": ([32768], 220.0, 0.0, 16),
    "32k_110B": ([32768], 110.0, 0.0, 32),
    "131k_220B": ([131072], 220.0, 0.0, 16),
    "64x4k_220B_student_t": ([4096] * 64, 220.0, 0.01, 16),
}


@pytest.mark.parametrize("name", sorted(FULL_CONFIGS))
def test_full_size_configs_sampled(src, name):
    """Full-size configurations: sampled rows plus every prompt's boundary rows and the
    rows around each 2^16 mark against the oracle (codes, centres, decoded rows), the whole
    blob re-coded by the oracle coder, the payload against the model code length, and the
    exact code round trip through the GPU decoder."""
    lens, target, st, chunk_rows = FULL_CONFIGS[name]
    cod = _full_codec(src, target, chunk_rows, st)
    seeds = [200 + 7 * i for i in range(len(lens))]
    r = full_size_check(src, cod, lens, seeds, chunk_rows, student_t=st)
    # the calibrated step scale puts the payload near the configuration's rate
    assert abs(r["payload"] / r["n"] / target - 1.0) <= 0.05, r["payload"] / r["n"]


@pytest.mark.parametrize("which", ["literal", "fitted"])
def test_guard_band_bounds_fp32_error(src, codec_literal, codec_55, which):
    """The fp32 transform ratio y / Delta (before exact recomputation) stays within the
    guard band the encoder uses to pick codes for fp64 recomputation,
    5e-7 * |x|_2 / Delta + 2e-5, so every code outside the band is decided correctly."""
    cod = codec_literal if which == "literal" else codec_55
    gc = gpu_codec(cod)
    lens = [132 + 400, 300] if which == "literal" else [132 + 700]
    x, tok, offs = make_batch(src, cod, lens, seeds=[61, 62][: len(lens)])
    n = sum(max(0, L - 132) for L in lens)
    ratio = torch.full((n, 2048), float("nan"), dtype=torch.float32, device="cuda")
    D.dckv_debug_ratio(gc.handle, ratio)
    try:
        encode_gpu(gc, x, tok, offs)
    finally:
        D.dckv_debug_ratio(gc.handle, None)
    g = ratio.cpu().numpy().astype(np.float64)
    xb = bits(x)
    ora = O.analyse(xb, tok.cpu().numpy(), offs, cod)
    r_o = np.concatenate([P["ratio"] for P in ora])
    lay = O.prompt_layout(np.diff(offs))
    rows = np.concatenate([np.arange(L["tok_base"] + 4, L["tok_base"] + 4 + L["n"]) for L in lay])
    xn = np.linalg.norm(O.bf16_to_f64(xb[rows]), axis=1)
    keep = O.scale_index(cod.laplace_b, cod.delta)[1]
    d = cod.delta.astype(np.float64)
    err = np.abs(g - r_o)[:, keep]
    band = (5e-7 * xn[:, None] / d[None, keep]) + 2e-5
    kappa = np.max(err * d[None, keep] / xn[:, None])
    print(f"{which}: max fp32 ratio error {err.max():.3e} steps, effective kappa {kappa:.3e}")
    assert np.all(err < band), (err.max(), kappa)

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
    q32 = ws[v["q32"]: v["q32"] + 4 * n * 2048].view(torch.int32).reshape(n, 2048).cpu().numpy()
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
    q16 = gc._ws[w["q16"]: w["q16"] + 2 * n * 2048].view(torch.float16).reshape(n, 2048).float().cpu().numpy()
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
    k_o, v_o = O.decode(res["blob"], tok.cpu().numpy(), offs, np_codec)
    kg, vg = bits(k), bits(v)
    for g, o in ((kg, k_o), (vg, v_o)):
        e = rel_frob(O.bf16_to_f64(g), O.bf16_to_f64(o))
        assert e <= ROW_TOL, e
    return dict(gc=gc, x=x, tok=tok, offs=offs, res=res, flips=flips, centre_mismatch=mism, k=k, v=v, aux=aux)


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


def test_full_size_4k_prompt_sampled(src, codec_55):
    """4,096-token prompt at about 220 B/token, in the configuration the benchmark times:
    sampled rows against the oracle, every chunk's section re-coded by the oracle coder,
    and the payload against the model code length."""
    gc = gpu_codec(codec_55)
    x, tok, offs = make_batch(src, codec_55, [4096], [100])
    res = encode_gpu(gc, x, tok, offs)
    assert res["status"] == D.DCKV_OK
    n = 4096 - 132
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(n, 48, replace=False))
    xb = bits(x)
    y = O.transform(xb[4 + rows], codec_55)
    q_o, ratio = O.quantise(y, codec_55.delta, O.scale_index(codec_55.laplace_b, codec_55.delta)[1])
    check_codes(res["q32"][rows].astype(np.int64), dict(q=q_o, ratio=ratio))
    codes = split_gpu_codes(gc, codec_55, res, tok, offs)
    # the whole blob from the GPU's codes and centres through the oracle coder
    aux = {}
    G = D.dckv_codec_info(gc.handle)["chunk_rows"]
    ora_blob = O.assemble_blob(xb, offs, codes, codec_55.laplace_b, codec_55.delta, G, aux=aux)
    assert ora_blob == res["blob"]
    payload = res["size"] - 132 * 12288
    model_bytes = aux["code_bits"] / 8
    assert payload <= 1.05 * model_bytes, (payload, model_bytes)
    assert 150 <= payload / n <= 300
    k, v, st, q16 = decode_gpu(gc, res["blob_dev"], res["size"], tok, offs)
    assert st == D.DCKV_OK
    assert np.array_equal(q16, res["q32"].astype(np.float32))
    # sampled decoded rows against the oracle's reconstruction of the same codes
    xh = O.reconstruct(res["q32"][rows].astype(np.int64), codec_55)
    want = O.f64_to_bf16(O.output_rows(xh, 4 + rows)).reshape(-1, 6, 2, 2, 256)
    kg = bits(k)[:, 4 + rows].transpose(1, 0, 2, 3)
    vg = bits(v)[:, 4 + rows].transpose(1, 0, 2, 3)
    assert rel_frob(O.bf16_to_f64(kg), O.bf16_to_f64(want[:, :, 0])) <= ROW_TOL
    assert rel_frob(O.bf16_to_f64(vg), O.bf16_to_f64(want[:, :, 1])) <= ROW_TOL


_FULL_CODECS = {}


def _full_codec(src, target):
    if target not in _FULL_CODECS:
        _FULL_CODECS[target] = S.codec(src, step_scale=None, target_bytes=target)
    return _FULL_CODECS[target]


# the larger configurations: (prompt lengths, target bytes per coded row, Student-t fraction,
# rows per rANS chunk).  At ~110 B per row a chunk's fixed 136 bytes need 32 rows to stay
# within the 5% payload bound.
FULL_CONFIGS = {
    "32k_220B": ([32768], 220.0, 0.0, 16),
    "32k_110B": ([32768], 110.0, 0.0, 32),
    "131k_220B": ([131072], 220.0, 0.0, 16),
    "64x4k_220B_student_t": ([4096] * 64, 220.0, 0.01, 16),
}


@pytest.mark.parametrize("name", sorted(FULL_CONFIGS))
def test_full_size_configs_sampled(src, name):
    """Full-size configurations: sampled rows' codes against the oracle, the whole blob
    re-coded by the oracle coder from the GPU's codes and centres, the payload against the
    model code length, exact code round trip through the GPU decoder, and sampled decoded
    rows against the oracle's reconstruction."""
    lens, target, st, chunk_rows = FULL_CONFIGS[name]
    cod = _full_codec(src, target)
    gc = gpu_codec(cod, chunk_rows)
    seeds = [200 + 7 * i for i in range(len(lens))]
    x, tok, offs = make_batch(src, cod, lens, seeds, student_t=st)
    res = encode_gpu(gc, x, tok, offs)
    assert res["status"] == D.DCKV_OK, D.STATUS_NAMES[res["status"]]
    lay = O.prompt_layout(np.diff(offs))
    n = sum(L["n"] for L in lay)
    rng = np.random.default_rng(1)
    rows = np.sort(rng.choice(n, 48, replace=False))  # coded-row indices over the batch
    starts = np.array([L["row_base"] for L in lay])
    pidx = np.searchsorted(starts, rows, side="right") - 1
    tok_rows = np.array([lay[p]["tok_base"] + 4 + (r - lay[p]["row_base"]) for p, r in zip(pidx, rows)])
    pos = np.array([4 + (r - lay[p]["row_base"]) for p, r in zip(pidx, rows)])
    xb = bits(x)
    keep = O.scale_index(cod.laplace_b, cod.delta)[1]
    q_o, ratio = O.quantise(O.transform(xb[tok_rows], cod), cod.delta, keep)
    check_codes(res["q32"][rows].astype(np.int64), dict(q=q_o, ratio=ratio))
    codes = split_gpu_codes(gc, cod, res, tok, offs)
    aux = {}
    G = D.dckv_codec_info(gc.handle)["chunk_rows"]
    ora_blob = O.assemble_blob(xb, offs, codes, cod.laplace_b, cod.delta, G, aux=aux)
    assert len(ora_blob) == res["size"] and ora_blob == res["blob"]
    kept = sum(L["N"] - L["n"] for L in lay)
    payload = res["size"] - kept * 12288
    assert payload <= 1.05 * aux["code_bits"] / 8, (payload, aux["code_bits"] / 8)
    if st > 0:
        assert aux["n_esc"] > 0  # heavy-tailed rows force escapes
    k, v, status, q16 = decode_gpu(gc, res["blob_dev"], res["size"], tok, offs)
    assert status == D.DCKV_OK
    small = np.abs(res["q32"]) < 2048
    assert np.array_equal(q16[small], res["q32"][small].astype(np.float32))
    xh = O.reconstruct(res["q32"][rows].astype(np.int64), cod)
    want = O.f64_to_bf16(O.output_rows(xh, pos)).reshape(-1, 6, 2, 2, 256)
    kg = bits(k)[:, tok_rows].transpose(1, 0, 2, 3)
    vg = bits(v)[:, tok_rows].transpose(1, 0, 2, 3)
    assert rel_frob(O.bf16_to_f64(kg), O.bf16_to_f64(want[:, :, 0])) <= ROW_TOL
    assert rel_frob(O.bf16_to_f64(vg), O.bf16_to_f64(want[:, :, 1])) <= ROW_TOL


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

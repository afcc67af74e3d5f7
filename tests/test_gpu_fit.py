"""GPU parity of the closed-form fit of the conditional models (include/dckv_fit.h)
against the oracle (oracle/fit.py), through the C ABI.

  * sums: X^T X and X^T Y of both parities from the GPU's own codes, element by element
    within a bound derived from the arithmetic (bf16 products are exact in fp32; each
    4,096-row slice is summed in fp32 on the tensor core, slices in fp64):
    |G_gpu - G| <= 2^-14 (|X|^T |X|) elementwise (256 truncating fp32 additions per slice);
  * solve: the GPU's fp64 Cholesky solution against numpy's on the same sums
    (backward error at fp64 level, and the two solutions' difference), bf16 export
    bit-exact against the oracle's rounding of the same values, and the singular case;
  * scales: integer residual sums bit-exact against the oracle's sums over the same
    codes and centres, fitted scales bit-exact;
  * end to end: a codec whose means are refit on 16 calibration prompts of 4,096 tokens
    and whose scales are refit on 4 others codes held-out prompts in fewer bytes than the
    trained codec and than a scale-only refit, and its blob and rows pass the codec parity
    checks.
"""
import numpy as np
import pytest
import torch

import dckv_synth as S
import learned_kv_cache_dckv_b200 as D
import oracle as O

pytestmark = pytest.mark.gpu

RIDGE = 1e-3


def _embed_dev(cod):
    return torch.from_numpy(np.ascontiguousarray(cod.embed).view(np.int16)).cuda()


def _codes_from_ws(handle, ws, offs, k_eff, keep):
    """Per prompt: the GPU's final codes (and, after the symbol kernel, centres)."""
    v = D.dckv_ws_offsets(handle, offs, 0)
    n = v["n_rows"]
    q32 = np.zeros((n, 2048), np.int64)
    if n:
        qc = ws[v["q32"]: v["q32"] + 4 * n * 2048].view(torch.int32).reshape(n, 2048).cpu().numpy()
        q32[:, keep] = qc[:, :k_eff]  # the library keeps kept components only, compact
    cen8 = ws[v["cen8"]: v["cen8"] + n * k_eff].view(torch.int8).reshape(n, k_eff).cpu().numpy()
    slot = ws[v["row_slot"]: v["row_slot"] + 4 * n].view(torch.int32).cpu().numpy()
    cen = np.zeros((n, 2048), np.int64)
    if n:
        cen[:, keep] = cen8[slot]
    out = []
    for L in O.prompt_layout(np.diff(offs)):
        q = q32[L["row_base"]: L["row_base"] + L["n"]]
        c = cen[L["row_base"]: L["row_base"] + L["n"]]
        out.append(dict(qe=q[0::2], qo=q[1::2], ce=c[0::2], co=c[1::2]))
    return out


def _accumulate(gc, cod, x, tok, offs, stats=None):
    if stats is None:
        stats = torch.zeros(D.FIT_STATS_DOUBLES, dtype=torch.float64, device="cuda")
    ws = torch.empty(D.dckv_fit_workspace_bytes(gc.handle, offs), dtype=torch.uint8, device="cuda")
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    D.dckv_fit_accumulate(gc.handle, _embed_dev(cod), x, tok, offs, stats, st, ws)
    torch.cuda.synchronize()
    assert int(st.item()) == D.DCKV_OK, D.STATUS_NAMES[int(st.item())]
    return stats, ws


def _stats_np(stats):
    s = stats.cpu().numpy()
    return dict(g_e=s[D.FIT_OFF_GE: D.FIT_OFF_CE].reshape(2048, 2048),
                c_e=s[D.FIT_OFF_CE: D.FIT_OFF_GO].reshape(2048, 2048),
                g_o=s[D.FIT_OFF_GO: D.FIT_OFF_CO].reshape(6144, 6144),
                c_o=s[D.FIT_OFF_CO: D.FIT_OFF_N].reshape(6144, 2048),
                n_e=int(s[D.FIT_OFF_N]), n_o=int(s[D.FIT_OFF_N + 1]))


def _solve(stats_dev, ridge=RIDGE):
    w_e = torch.empty((2048, 2048), dtype=torch.float64, device="cuda")
    w_o = torch.empty((6144, 2048), dtype=torch.float64, device="cuda")
    ws = torch.empty(D.dckv_fit_solve_workspace_bytes(), dtype=torch.uint8, device="cuda")
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    D.dckv_fit_solve(stats_dev, ridge, w_e, w_o, st, ws)
    torch.cuda.synchronize()
    return w_e, w_o, int(st.item())


_CASE = {}


def _small_case(src, codec_55):
    if "c" not in _CASE:
        x, tok, offs = S.structured_batch(src, codec_55.embed, [132 + 300, 132 + 201, 90], [61, 62, 63],
                                          token_gain=0.6, ar=0.8, device="cuda")
        gc = D.Codec(D.upload_params(codec_55), 0, 0)
        stats, ws = _accumulate(gc, codec_55, x, tok, offs)
        keep = O.scale_index(codec_55.laplace_b, codec_55.delta)[1]
        codes = _codes_from_ws(gc.handle, ws, offs, gc.k_eff, keep)
        _CASE["c"] = dict(x=x, tok=tok, offs=offs, gc=gc, stats=stats, codes=codes)
    return _CASE["c"]


def test_fit_sums_match_the_oracle(src, codec_55):
    c = _small_case(src, codec_55)
    g = _stats_np(c["stats"])
    tok = c["tok"].cpu().numpy()
    ora = O.fit_statistics_from_codes(c["codes"], tok, c["offs"], codec_55.embed)
    assert g["n_e"] == ora["n_e"] == 150 + 101 and g["n_o"] == ora["n_o"] == 150 + 100
    # |X|^T |X| and |X|^T |Y| bound the accumulation error
    ab = dict(g_e=0, c_e=0, g_o=0, c_o=0)
    for L, P in zip(O.prompt_layout(np.diff(c["offs"])), c["codes"]):
        if L["n"] == 0:
            continue
        t0 = L["tok_base"] + O.HEAD_KEPT
        xe, ye, xo, yo = O.fit_regressors(P["qe"], P["qo"], tok[t0: t0 + L["n"]: 2], tok[t0 + 1: t0 + L["n"]: 2],
                                          codec_55.embed)
        ab["g_e"] = ab["g_e"] + np.abs(xe).T @ np.abs(xe)
        ab["c_e"] = ab["c_e"] + np.abs(xe).T @ np.abs(ye)
        ab["g_o"] = ab["g_o"] + np.abs(xo).T @ np.abs(xo)
        ab["c_o"] = ab["c_o"] + np.abs(xo).T @ np.abs(yo)
    for k in ("g_e", "c_e", "g_o", "c_o"):
        err = np.abs(g[k] - ora[k])
        bound = 2.0 ** -14 * ab[k] + 1e-30
        assert np.all(err <= bound), (k, float((err / bound).max()))
        assert np.any(ora[k] != 0)


def test_fit_solve_matches_the_oracle(src, codec_55):
    c = _small_case(src, codec_55)
    ora = O.fit_statistics_from_codes(c["codes"], c["tok"].cpu().numpy(), c["offs"], codec_55.embed)
    # the GPU solve on the oracle's own sums, so that only the solve is compared
    s = np.zeros(D.FIT_STATS_DOUBLES)
    s[D.FIT_OFF_GE: D.FIT_OFF_CE] = ora["g_e"].ravel()
    s[D.FIT_OFF_CE: D.FIT_OFF_GO] = ora["c_e"].ravel()
    s[D.FIT_OFF_GO: D.FIT_OFF_CO] = ora["g_o"].ravel()
    s[D.FIT_OFF_CO: D.FIT_OFF_N] = ora["c_o"].ravel()
    w_e, w_o, st = _solve(torch.from_numpy(s).cuda())
    assert st == D.DCKV_OK
    we_o, wo_o = O.fit_mean_models(ora, RIDGE)
    for w_gpu, w_ora, gname, cname in ((w_e, we_o, "g_e", "c_e"), (w_o, wo_o, "g_o", "c_o")):
        w = w_gpu.cpu().numpy()
        a = ora[gname].copy()
        i = np.arange(a.shape[0])
        a[i, i] += RIDGE * (a[i, i] + 1.0)
        # backward error of a Cholesky solve: ||A W - C|| <= c n eps ||A|| ||W||
        res = np.linalg.norm(a @ w - ora[cname]) / (np.linalg.norm(a) * np.linalg.norm(w))
        assert res <= 64 * a.shape[0] * 2.0 ** -53, res
        diff = np.linalg.norm(w - w_ora) / np.linalg.norm(w_ora)
        assert diff <= 1e-6, diff
        # bf16 export: one RNE step, as the oracle rounds the same values
        bits = torch.empty(w_gpu.shape, dtype=torch.int16, device="cuda")
        D.dckv_fit_to_bf16(w_gpu, bits)
        torch.cuda.synchronize()
        assert np.array_equal(bits.cpu().numpy().view(np.uint16), O.f64_to_bf16(w))


def test_fit_solve_reports_a_singular_system():
    s = torch.zeros(D.FIT_STATS_DOUBLES, dtype=torch.float64, device="cuda")
    # G_e = -2 I: with the ridge term the first pivot is -2 + 1e-3 (-2 + 1) < 0
    s[D.FIT_OFF_GE: D.FIT_OFF_CE].view(2048, 2048).diagonal().fill_(-2.0)
    _, _, st = _solve(s)
    assert st == D.DCKV_ESINGULAR


def test_fit_scales_match_the_oracle(src, codec_55):
    c = _small_case(src, codec_55)
    w_e, w_o, st = _solve(c["stats"])
    assert st == D.DCKV_OK
    refit = O.refit_codec(codec_55, w_e.cpu().numpy(), w_o.cpu().numpy())
    gr = D.Codec(D.upload_params(refit), 0, 0)
    ws = torch.empty(D.dckv_fit_workspace_bytes(gr.handle, c["offs"]), dtype=torch.uint8, device="cuda")
    acc = torch.zeros(2049, dtype=torch.int64, device="cuda")
    stt = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    D.dckv_fit_scales_accumulate(gr.handle, c["x"], c["tok"], c["offs"], acc, stt, ws)
    torch.cuda.synchronize()
    assert int(stt.item()) == D.DCKV_OK
    keep = O.scale_index(refit.laplace_b, refit.delta)[1]
    codes = _codes_from_ws(gr.handle, ws, c["offs"], gr.k_eff, keep)
    total, rows = O.fit_scales_from_codes(codes, refit.laplace_b, refit.delta)
    a = acc.cpu().numpy()
    assert int(a[2048]) == rows == 501
    assert np.array_equal(a[:2048], total)
    # the refit codec's centres are the oracle's (fp32 vs fp64 means: flips only at .5)
    ana = O.analyse(c["x"].view(torch.int16).cpu().numpy().view(np.uint16), c["tok"].cpu().numpy(), c["offs"], refit)
    n_diff = sum(int((P["ce"][:, keep] != A["ce"][:, keep]).sum() + (P["co"][:, keep] != A["co"][:, keep]).sum())
                 for P, A in zip(codes, ana))
    assert n_diff <= 1e-3 * rows * int(keep.sum())
    b = torch.empty(2048, dtype=torch.float32, device="cuda")
    D.dckv_fit_scales_finish(gr.handle, acc, b)
    torch.cuda.synchronize()
    b_ora = O.scales_from_sums(a[:2048], int(a[2048]), refit.laplace_b, refit.delta)
    assert np.array_equal(b.cpu().numpy().view(np.uint32), b_ora.view(np.uint32))
    assert np.array_equal(O.scale_index(b_ora, refit.delta)[1], keep)
    gr.close()


def test_refit_codec_codes_held_out_prompts_in_fewer_bytes(src, codec_55):
    # rows with strong token and neighbour structure; means fitted on 16 calibration prompts
    # of 4,096 tokens, scales on 4 others (in-sample residuals of a least-squares fit are
    # biased low), bytes measured on 2 held-out prompts
    cod = codec_55
    tg, ar = 0.8, 0.95
    gc = D.Codec(D.upload_params(cod), 0, 0)
    stats = torch.zeros(D.FIT_STATS_DOUBLES, dtype=torch.float64, device="cuda")
    for i in range(4):
        x, tok, offs = S.structured_batch(src, cod.embed, [4096] * 4, [500 + 4 * i + j for j in range(4)],
                                          token_gain=tg, ar=ar, device="cuda")
        _accumulate(gc, cod, x, tok, offs, stats)
    w_e, w_o, st = _solve(stats, ridge=0.1)
    assert st == D.DCKV_OK
    we_b = torch.empty((2048, 2048), dtype=torch.int16, device="cuda")
    wo_b = torch.empty((6144, 2048), dtype=torch.int16, device="cuda")
    D.dckv_fit_to_bf16(w_e, we_b)
    D.dckv_fit_to_bf16(w_o, wo_b)
    means = O.refit_codec(cod, w_e.cpu().numpy(), w_o.cpu().numpy())
    assert np.array_equal(means.w_even, we_b.cpu().numpy().view(np.uint16))
    assert np.array_equal(means.w_odd, wo_b.cpu().numpy().view(np.uint16))
    gm = D.Codec(D.upload_params(means), 0, 0)
    xs, ts, os_ = S.structured_batch(src, cod.embed, [4096] * 4, [700, 701, 702, 703], token_gain=tg, ar=ar,
                                     device="cuda")
    ws = torch.empty(D.dckv_fit_workspace_bytes(gm.handle, os_), dtype=torch.uint8, device="cuda")
    scales = []
    for g in (gm, gc):  # fitted means; trained means (a scale-only refit, for comparison)
        acc = torch.zeros(2049, dtype=torch.int64, device="cuda")
        stt = torch.zeros(1, dtype=torch.int32, device="cuda")
        D.dckv_fit_scales_accumulate(g.handle, xs, ts, os_, acc, stt, ws)
        b = torch.empty(2048, dtype=torch.float32, device="cuda")
        D.dckv_fit_scales_finish(g.handle, acc, b)
        torch.cuda.synchronize()
        assert int(stt.item()) == D.DCKV_OK
        scales.append(b.cpu().numpy())
    refit = O.refit_codec(cod, w_e.cpu().numpy(), w_o.cpu().numpy(), scales[0])
    scale_only = O.refit_codec(cod, O.bf16_to_f64(cod.w_even), O.bf16_to_f64(cod.w_odd), scales[1])
    gr, gs = D.Codec(D.upload_params(refit), 0, 0), D.Codec(D.upload_params(scale_only), 0, 0)
    x, tok, offs = S.structured_batch(src, cod.embed, [4096, 4096], [900, 901], token_gain=tg, ar=ar, device="cuda")
    sizes = []
    for g in (gc, gs, gr):
        blob = g.encode(x, tok, offs)
        torch.cuda.synchronize()
        assert int(g.status.item()) == D.DCKV_OK
        sizes.append(D.dckv_bytes(blob[: int(g.blob_size.item())].cpu().numpy().tobytes())["payload"])
    assert sizes[2] < 0.97 * sizes[1] and sizes[2] < 0.93 * sizes[0], sizes
    # the refit codec's blob and rows pass the codec's own parity checks
    xs, ts, os_ = S.structured_batch(src, cod.embed, [132 + 300], [902], token_gain=tg, ar=ar, device="cuda")
    blob = gr.encode(xs, ts, os_)
    torch.cuda.synchronize()
    assert int(gr.status.item()) == D.DCKV_OK
    size = int(gr.blob_size.item())
    xb = xs.view(torch.int16).cpu().numpy().view(np.uint16)
    keep = O.scale_index(refit.laplace_b, refit.delta)[1]
    ana = O.analyse(xb, ts.cpu().numpy(), os_, refit)
    ws_codes = _codes_from_ws_encode(gr, os_, keep)
    ora_blob = O.assemble_blob(xb, os_, ws_codes, refit.laplace_b, refit.delta, 16)
    assert ora_blob == blob[:size].cpu().numpy().tobytes()
    n_diff = sum(int((P["qe"] != A["qe"]).sum() + (P["qo"] != A["qo"]).sum()) for P, A in zip(ws_codes, ana))
    n_cen = sum(int((P["ce"][:, keep] != A["ce"][:, keep]).sum() + (P["co"][:, keep] != A["co"][:, keep]).sum())
                for P, A in zip(ws_codes, ana))
    assert n_diff <= 1e-3 * 300 * 2048 and n_cen <= 1e-3 * 300 * int(keep.sum())
    k, v = gr.decode(blob, size, ts, os_)
    torch.cuda.synchronize()
    assert int(gr.status.item()) == D.DCKV_OK
    k_o, v_o = O.decode(blob[:size].cpu().numpy().tobytes(), ts.cpu().numpy(), os_, refit)
    for g_, o_ in ((k, k_o), (v, v_o)):
        a = O.bf16_to_f64(g_.view(torch.int16).cpu().numpy().view(np.uint16))
        bb = O.bf16_to_f64(o_)
        assert np.linalg.norm(a - bb) / np.linalg.norm(bb) <= 1e-3
    for g in (gc, gm, gr, gs):
        g.close()


def _codes_from_ws_encode(gc, offs, keep):
    return _codes_from_ws(gc.handle, gc._ws, offs, gc.k_eff, keep)

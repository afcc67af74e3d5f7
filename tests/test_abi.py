"""The C-ABI library builds for sm_100a, loads without a GPU, exports every function the
headers declare, and its host-only entry points agree with the oracle.  CPU only."""
import ctypes

import numpy as np
import pytest
import torch

import dckv_synth as S
import learned_kv_cache_dckv_b200 as D
import oracle as O
from learned_kv_cache_dckv_b200 import build as B


@pytest.fixture(scope="module")
def lib():
    B.build()
    return D.lib()


def test_library_exports_every_declared_function(lib):
    names = D.header_functions()
    assert {"dckv_encode", "dckv_decode", "dckv_bytes", "dckv_codec_create"} <= set(names)
    raw = ctypes.CDLL(D.LIB_PATH)
    missing = [n for n in names if not hasattr(raw, n)]
    assert not missing, missing


def test_dckv_bytes_matches_oracle_report(lib, src):
    cod = S.codec(src, step_scale=None, target_bytes=220.0)
    x, tok, offs = S.batch(src, [300, 60, 140], seeds=[1, 2, 3])
    xb = x.view(torch.int16).numpy().view(np.uint16)
    mu = torch.from_numpy(cod.mu)
    x[10] = (mu + (x[10].float() - mu) * 80).to(torch.bfloat16)  # force escapes
    xb = x.view(torch.int16).numpy().view(np.uint16)
    blob = O.encode(xb, tok.numpy(), offs, cod, chunk_rows=8)
    rep = D.dckv_bytes(blob)
    ora = O.byte_report(blob)
    hdr = O.parse_blob(blob)
    assert rep["total"] == ora["total"] == len(blob)
    assert rep["kept_rows"] == ora["kept_rows"] == (4 + 128 + 60 + 132) * 12288
    assert rep["states"] == ora["states"] and rep["esc_values"] == ora["esc_values"]
    assert rep["words"] == ora["words"] + ora["padding"] - (ora["header_tables"] - hdr["off_kept"])
    assert rep["payload"] == ora["payload"]
    assert rep["n_coded_rows"] == 168 + 8 and rep["k_eff"] == hdr["k_eff"] and rep["chunk_rows"] == 8
    assert rep["n_escapes"] * 8 == ora["esc_values"] and rep["n_escapes"] > 0


def test_dckv_bytes_rejects_corrupt_blobs(lib, src, codec_literal):
    x, tok = S.prompt(src, 140, seed=9)
    blob = bytearray(O.encode(x.view(torch.int16).numpy().view(np.uint16), tok.numpy(), [0, 140], codec_literal))
    with pytest.raises(D.DckvError):
        D.dckv_bytes(bytes(blob[:100]))
    bad = bytearray(blob)
    bad[0] ^= 0x40
    with pytest.raises(D.DckvError):
        D.dckv_bytes(bytes(bad))
    bad = bytearray(blob)
    bad[40] ^= 1  # stream offset
    with pytest.raises(D.DckvError):
        D.dckv_bytes(bytes(bad))


def test_host_argument_errors_need_no_gpu(lib):
    L = D.lib()
    offs = np.array([0, 300], np.int64)
    r = L.dckv_encode(None, None, None, offs.ctypes.data_as(ctypes.c_void_p), 1, None, 0, None, None, None, 0, None)
    assert r == D.DCKV_EINVAL
    r = L.dckv_decode(None, None, 0, None, offs.ctypes.data_as(ctypes.c_void_p), 1, None, None, None, None, 0, None)
    assert r == D.DCKV_EINVAL
    assert L.dckv_workspace_bytes(None, offs.ctypes.data_as(ctypes.c_void_p), 1) == 0
    assert "NULL" in D.last_error() or D.last_error() == ""


def test_fit_host_argument_errors_need_no_gpu(lib):
    L = D.lib()
    offs = np.array([0, 300], np.int64)
    po = offs.ctypes.data_as(ctypes.c_void_p)
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: every call below fails its host checks first
    assert L.dckv_fit_workspace_bytes(None, po, 1) == 0
    assert L.dckv_fit_accumulate(None, fake, 8, fake, fake, po, 1, fake, fake, fake, 1 << 30, None) == D.DCKV_EINVAL
    assert L.dckv_fit_solve_workspace_bytes() == 8 * 6144 * 6144
    assert L.dckv_fit_solve(None, 1e-3, fake, fake, fake, fake, 1 << 30, None) == D.DCKV_EINVAL
    assert L.dckv_fit_solve(fake, 0.0, fake, fake, fake, fake, 1 << 30, None) == D.DCKV_EINVAL
    assert "ridge" in D.last_error()
    assert L.dckv_fit_solve(fake, float("nan"), fake, fake, fake, fake, 1 << 30, None) == D.DCKV_EINVAL
    assert L.dckv_fit_solve(fake, 1e-3, fake, fake, fake, fake, 1024, None) == D.DCKV_ECAPACITY
    assert L.dckv_fit_to_bf16(None, 4, fake, None) == D.DCKV_EINVAL
    assert L.dckv_fit_to_bf16(fake, -1, fake, None) == D.DCKV_EINVAL
    assert L.dckv_fit_to_bf16(fake, 0, fake, None) == D.DCKV_OK  # nothing to convert, no device work
    assert L.dckv_fit_scales_accumulate(None, fake, fake, po, 1, fake, fake, fake, 1 << 30, None) == D.DCKV_EINVAL
    assert L.dckv_fit_scales_finish(None, fake, fake, None) == D.DCKV_EINVAL


def test_fit_rejects_misaligned_fp64_buffers(lib):
    L = D.lib()
    odd = ctypes.c_void_p(0x1004)  # 4-byte but not 8-byte aligned
    ok = ctypes.c_void_p(0x1000)
    assert L.dckv_fit_solve(odd, 1e-3, ok, ok, ok, ok, 1 << 30, None) == D.DCKV_EINVAL
    assert "aligned" in D.last_error()
    assert L.dckv_fit_to_bf16(odd, 4, ok, None) == D.DCKV_EINVAL

"""dckv_decode_static (decode on the library's static per-device scratch) against
dckv_decode with a caller workspace, through the C ABI.

Both run the same kernels on the same blob, so the rows must agree exactly (well inside the
1e-3 relative Frobenius tolerance of the decode parity tests), on consecutive calls of
different batches: each call finds the previous call's contents in the shared scratch.
"""
import numpy as np
import pytest
import torch

import dckv_synth as S
import learned_kv_cache_dckv_b200 as D

pytestmark = pytest.mark.gpu

STATIC_BYTES = 16 << 20  # DCKV_STATIC_SCRATCH_BYTES


def _rel_frob(a, b):
    a = a.double()
    b = b.double()
    return float((a - b).norm() / max(float(b.norm()), 1e-30))


def _encode(gc, src, lens, seeds):
    x, tok, offs = S.batch(src, lens, seeds, device="cuda")
    blob = gc.encode(x, tok, offs)
    torch.cuda.synchronize()
    assert int(gc.status.item()) == D.DCKV_OK
    size = int(gc.blob_size.item())
    blob = blob[:size].clone()
    k_ref, v_ref = gc.decode(blob, size, tok, offs)
    torch.cuda.synchronize()
    assert int(gc.status.item()) == D.DCKV_OK
    return blob, size, tok, offs, k_ref.clone(), v_ref.clone()


def _decode_static(gc, blob, size, tok, offs):
    n_tok = int(np.asarray(offs)[-1])
    k = torch.full((6, n_tok, 2, 256), float("nan"), dtype=torch.bfloat16, device="cuda")
    v = torch.full_like(k, float("nan"))
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    D.dckv_decode_static(gc.handle, blob, size, tok, offs, k, v, st)
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    assert int(st.item()) == D.DCKV_OK
    return k, v, free0, free1


def test_static_scratch_decode_matches_workspace_decode(src, codec_literal):
    """A large batch (near the scratch's size) first, then a smaller one with other
    lengths, token ids and chunk counts, twice: each call must initialise what it reads
    of the shared scratch, so every result equals the workspace decode of the same blob
    exactly; and after the first call (which looks the array up) a call allocates no
    device memory."""
    gc = D.Codec(D.upload_params(codec_literal), 0, 0)
    big = _encode(gc, src, [132 + 650, 132 + 50], [61, 62])
    small = _encode(gc, src, [132 + 300, 140, 132 + 77, 90], [51, 52, 53, 54])
    assert D.dckv_ws_offsets(gc.handle, big[3], 1)["total"] <= STATIC_BYTES
    assert D.dckv_ws_offsets(gc.handle, small[3], 1)["total"] < D.dckv_ws_offsets(gc.handle, big[3], 1)["total"]
    for call, (blob, size, tok, offs, k_ref, v_ref) in enumerate((big, small, small, big)):
        k, v, free0, free1 = _decode_static(gc, blob, size, tok, offs)
        assert _rel_frob(k, k_ref) <= 1e-3 and _rel_frob(v, v_ref) <= 1e-3, f"call {call}"
        assert torch.equal(k, k_ref) and torch.equal(v, v_ref), f"call {call}"
        if call > 0:
            assert free1 == free0, f"call {call} changed free device memory by {free0 - free1} bytes"
    gc.close()


def test_static_scratch_rejects_batches_beyond_its_size(src, codec_literal):
    gc = D.Codec(D.upload_params(codec_literal), 0, 0)
    offs = np.array([0, 132 + 1200], np.int64)  # 1,200 coded rows at K_eff = 2048
    assert D.dckv_ws_offsets(gc.handle, offs, 1)["total"] > STATIC_BYTES
    tok = torch.zeros(int(offs[-1]), dtype=torch.int32, device="cuda")
    blob = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    k = torch.empty((6, int(offs[-1]), 2, 256), dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(D.DckvError) as e:
        D.dckv_decode_static(gc.handle, blob, blob.numel(), tok, offs, k, k.clone(), st)
    assert e.value.code == D.DCKV_ECAPACITY
    assert "static scratch" in D.last_error()
    gc.close()

"""The tcgen05 GEMM core (TMA -> swizzled smem -> tcgen05.mma -> TMEM -> tcgen05.ld)
against an fp64 product of the same fp16/bf16 operands."""
import pytest
import torch

import learned_kv_cache_dckv_b200 as D

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("slabs", [1, 2])
@pytest.mark.parametrize("M,N,K,bn", [(128, 256, 64, 256), (256, 300, 512, 256), (384, 1000, 2048, 128),
                                      (128, 1, 64, 256), (128, 77, 192, 64), (256, 513, 6144, 256)])
def test_gemm_matches_fp64(bf16, slabs, M, N, K, bn):
    _check_gemm(bf16, slabs, M, N, K, bn, False)


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("slabs", [1, 2])
@pytest.mark.parametrize("M,N,K,bn", [(256, 256, 64, 256), (256, 300, 512, 256), (512, 1000, 2048, 224),
                                      (256, 1, 64, 32), (256, 77, 192, 64), (768, 513, 6144, 256),
                                      (2048, 700, 1024, 128)])
def test_pair_gemm_matches_fp64(bf16, slabs, M, N, K, bn):
    # CTA pairs (cta_group::2): 256-row tiles, each CTA staging half of the B tile
    _check_gemm(bf16, slabs, M, N, K, bn, True)


def _check_gemm(bf16, slabs, M, N, K, bn, pair):
    g = torch.Generator(device="cuda")
    g.manual_seed(M * 7 + N * 13 + K + slabs + int(bf16))
    dt = torch.bfloat16 if bf16 else torch.float16
    A = torch.randn((slabs, M, K), generator=g, device="cuda").to(dt)
    B = torch.randn((N, K), generator=g, device="cuda").to(dt)
    Dm = torch.full((N, M), float("nan"), dtype=torch.float32, device="cuda")
    D.dckv_debug_gemm(bf16, A, slabs, B, M, N, K, Dm, bn, pair)
    torch.cuda.synchronize()
    ref = sum(B.double() @ A[s].double().T for s in range(slabs))
    err = (Dm.double() - ref).abs().max().item()
    scale = (B.double().abs() @ A.double().abs().sum(0).T).max().item()
    assert err <= 4e-6 * scale, (err, scale)

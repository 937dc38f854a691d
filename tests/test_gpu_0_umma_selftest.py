"""tcgen05 building blocks (TMA 128-byte swizzle, shared-memory descriptors
for K-major and MN-major operands, tcgen05.mma, TMEM read-back) on one GEMM
tile, against torch.matmul in fp32."""
import pytest
import torch

from gpu_helpers import lib_ready

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N", [64, 128, 256])
@pytest.mark.parametrize("Kd", [64, 128, 256])
@pytest.mark.parametrize("mn_major", [False, True])
@pytest.mark.parametrize("a_tmem", [False, True])
def test_umma_tile(N, Kd, mn_major, a_tmem):
    lib_ready()
    from block_sparse_long_05_b200 import msa
    g = torch.Generator(device="cuda").manual_seed(N * 1000 + Kd + mn_major)
    A = torch.randn(128, Kd, generator=g, device="cuda").to(torch.bfloat16)
    Bm = torch.randn(Kd, N, generator=g, device="cuda").to(torch.bfloat16)  # logical [Kd, N]
    B = Bm.contiguous() if mn_major else Bm.t().contiguous()
    C, status = msa.selftest_umma(A, B, mn_major, a_tmem)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = A.float() @ Bm.float()
    err = (C - ref).abs().max().item()
    assert err < 1e-3 * max(1.0, ref.abs().max().item()), err

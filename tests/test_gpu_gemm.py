"""The persistent tcgen05 GEMM against a float64 product of the same bf16/f16
inputs (several tiles, ragged M, many waves)."""
import pytest
import torch

from tests.gpu_helpers import ensure_built

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("m,n,k,dtype,tile_n", [
    (128, 256, 64, torch.bfloat16, 256),
    (300, 512, 192, torch.bfloat16, 256),
    (1000, 768, 4096, torch.float16, 256),
    (2048, 6144, 4096, torch.bfloat16, 256),
    (300, 384, 192, torch.float16, 128),
])
def test_gemm_matches_float64(cuda_ready, m, n, k, dtype, tile_n):
    ensure_built()
    from mot_flow_matching_b200.layer import mot_dev_gemm
    g = torch.Generator(device="cpu").manual_seed(m * 7 + n)
    a = torch.randn(m, k, generator=g).to(dtype).cuda()
    b = torch.randn(n, k, generator=g).to(dtype).cuda()
    d = torch.full((m, n), float("nan"), device="cuda")
    mot_dev_gemm(a, b, d, tile_n)
    torch.cuda.synchronize()
    ref = a.double() @ b.double().T
    err = (d.double() - ref).abs().max().item()
    assert err <= 2e-5 * k ** 0.5 * ref.abs().max().item(), err

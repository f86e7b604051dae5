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


def _operands(m, n, k, dtype, seed, two=False):
    g = torch.Generator(device="cpu").manual_seed(seed)
    a = torch.randn(m, k, generator=g).to(dtype).cuda()
    b = torch.randn(n, k, generator=g).to(dtype).cuda()
    b2 = torch.randn(n, k, generator=g).to(dtype).cuda() if two else None
    return a, b, b2


@pytest.mark.parametrize("m,n,k,dtype", [
    (256, 256, 64, torch.bfloat16),
    (300, 512, 192, torch.float16),     # ragged rows: the odd CTA of the last pair is past M
    (2048, 1024, 4096, torch.bfloat16),
])
def test_pair_gemm_matches_float64(cuda_ready, m, n, k, dtype):
    # CTA-pair (cta_group::2) kernel, 256 x 256 tiles
    ensure_built()
    from mot_flow_matching_b200.layer import mot_dev_gemm_variant
    a, b, _ = _operands(m, n, k, dtype, m + 3 * n)
    d = torch.full((m, n), float("nan"), device="cuda")
    mot_dev_gemm_variant(a, b, d, 1)
    torch.cuda.synchronize()
    ref = a.double() @ b.double().T
    assert (d.double() - ref).abs().max().item() <= 2e-5 * k ** 0.5 * ref.abs().max().item()


@pytest.mark.parametrize("m,k,dtype", [
    (128, 128, torch.bfloat16),   # one tile, two k-blocks: at most one block per split
    (300, 640, torch.float16),    # ragged rows
    (4096, 4096, torch.bfloat16),
])
def test_split_k_gemm_matches_float64_and_is_deterministic(cuda_ready, m, k, dtype):
    # 64-wide tiles split along K; the tile's last CTA sums the partials in split order
    ensure_built()
    from mot_flow_matching_b200.layer import mot_dev_gemm_variant
    a, b, _ = _operands(m, 64, k, dtype, 11 * m + k)
    d1 = torch.full((m, 64), float("nan"), device="cuda")
    d2 = torch.full((m, 64), float("nan"), device="cuda")
    mot_dev_gemm_variant(a, b, d1, 2)
    mot_dev_gemm_variant(a, b, d2, 2)
    ref = a.double() @ b.double().T
    assert (d1.double() - ref).abs().max().item() <= 2e-5 * k ** 0.5 * ref.abs().max().item()
    assert torch.equal(d1.view(torch.int32), d2.view(torch.int32))


@pytest.mark.parametrize("m,k,dtype", [(200, 256, torch.bfloat16), (4096, 4096, torch.float16)])
def test_dual_b_gemm_matches_float64(cuda_ready, m, k, dtype):
    # two B operands per A tile accumulate into one D: A B^T + A B2^T
    ensure_built()
    from mot_flow_matching_b200.layer import mot_dev_gemm_variant
    a, b, b2 = _operands(m, 64, k, dtype, 5 * m + k, two=True)
    d = torch.full((m, 64), float("nan"), device="cuda")
    mot_dev_gemm_variant(a, b, d, 3, b2=b2)
    torch.cuda.synchronize()
    ref = a.double() @ b.double().T + a.double() @ b2.double().T
    assert (d.double() - ref).abs().max().item() <= 4e-5 * k ** 0.5 * ref.abs().max().item()


@pytest.mark.parametrize("m,n,k,dtype", [(300, 256, 128, torch.float16), (2048, 1024, 4096, torch.bfloat16)])
def test_pair_gemm_mn_major_b_matches_float64(cuda_ready, m, n, k, dtype):
    # CTA pairs with B loaded as an MN-major operand (B given as [k, n])
    ensure_built()
    from mot_flow_matching_b200.layer import mot_dev_gemm_variant
    g = torch.Generator(device="cpu").manual_seed(m + n + k)
    a = torch.randn(m, k, generator=g).to(dtype).cuda()
    b = torch.randn(k, n, generator=g).to(dtype).cuda()
    d = torch.full((m, n), float("nan"), device="cuda")
    mot_dev_gemm_variant(a, b, d, 4)
    torch.cuda.synchronize()
    ref = a.double() @ b.double()
    assert (d.double() - ref).abs().max().item() <= 2e-5 * k ** 0.5 * ref.abs().max().item()

"""The FMA-pipe exponential of the attention softmax (range reduction plus a
degree-3 minimax polynomial for 2^f, f in [-1/2, 1/2]).

CPU: the polynomial, evaluated in float32 exactly as the kernel does, stays
within its fitted relative-error bound against float64 2^f. GPU: the device
routine (including the exponent-field step) against float64 exp2 on a dense
grid of the softmax's argument range, and against CUDA's exp2f."""
import numpy as np
import pytest
import torch

C = np.array([9.999280735e-01, 6.932609855e-01, 2.426111222e-01, 5.517166906e-02], dtype=np.float32)
BOUND = 7.6e-5  # fitted minimax relative error of the coefficients


def horner_f32(f):
    q = np.float32(C[3])
    for k in (2, 1, 0):
        q = (q * f + C[k]).astype(np.float32)
    return q


def test_polynomial_error_bound_cpu():
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    rel = np.abs(horner_f32(f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)
    assert rel.max() < BOUND
    # the bound is tight (equioscillation), so a wrong coefficient shows
    assert rel.max() > 0.5 * BOUND


@pytest.mark.gpu
def test_device_exp2_poly_matches_exp2(cuda_ready):
    from tests.gpu_helpers import ensure_built
    from mot_flow_matching_b200.layer import mot_dev_exp2_poly
    ensure_built()
    x = torch.linspace(-125.0, 8.0, 1 << 20, dtype=torch.float32, device="cuda")
    y = torch.empty_like(x)
    mot_dev_exp2_poly(x, y)
    torch.cuda.synchronize()
    ref = torch.exp2(x.double())
    rel = (y.double() / ref - 1.0).abs()
    assert rel.max().item() < BOUND + 4e-7
    assert torch.all(torch.isfinite(y)) and torch.all(y > 0)
    # CUDA's own exp2f within the same bound of ours
    assert ((y.double() - torch.exp2(x).double()).abs() / ref).max().item() < BOUND + 1e-6

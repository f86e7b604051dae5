"""Host-only checks of the MLP, mixture-of-experts and denoise-step C ABIs
(include/mot_mlp.h, include/mot_moe.h, include/mot_step.h): sizing and
argument validation answer on the host, before any CUDA call (no GPU
needed)."""
import ctypes
from ctypes import POINTER, byref, c_size_t, c_void_p

import pytest

from mot_flow_matching_b200 import _abi
from mot_flow_matching_b200 import build as build_mod


@pytest.fixture(scope="module")
def L():
    build_mod.build()
    return _abi.lib()


def mlp_cfg(**kw):
    c = _abi.MotMlpConfig(hidden=4096, intermediate=12288, lora_rank=32, lora_alpha=32.0, max_tokens=8192,
                          enable_backward=1)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def moe_cfg(**kw):
    c = _abi.MotMoeConfig(hidden=2048, intermediate=768, experts=32, top_k=8, max_tokens=8192)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def test_mlp_query_sizes(L):
    ws, sv = c_size_t(), c_size_t()
    T, I = 4096, 12288
    assert L.mot_mlp_query_sizes(byref(mlp_cfg()), T, byref(ws), byref(sv)) == _abi.MOT_OK
    # the training forward keeps g, u and h (f16 [T, I] each)
    assert sv.value >= 3 * T * I * 2
    # inference needs at least h (f16 [T, I]) in the workspace
    assert ws.value >= T * I * 2
    assert L.mot_mlp_query_sizes(byref(mlp_cfg()), 0, byref(ws), byref(sv)) == _abi.MOT_ERR_INVALID_ARGUMENT
    assert L.mot_mlp_query_sizes(byref(mlp_cfg()), 8193, byref(ws), byref(sv)) == _abi.MOT_ERR_UNSUPPORTED_SHAPE
    # either output may be NULL
    assert L.mot_mlp_query_sizes(byref(mlp_cfg()), T, None, byref(sv)) == _abi.MOT_OK


@pytest.mark.parametrize("field,value,status", [
    ("hidden", 4000, _abi.MOT_ERR_UNSUPPORTED_SHAPE),
    ("intermediate", 12300, _abi.MOT_ERR_UNSUPPORTED_SHAPE),
    ("lora_rank", 12, _abi.MOT_ERR_UNSUPPORTED_SHAPE),
    ("lora_rank", 136, _abi.MOT_ERR_UNSUPPORTED_SHAPE),
    ("lora_rank", -8, _abi.MOT_ERR_INVALID_ARGUMENT),
    ("hidden", -256, _abi.MOT_ERR_INVALID_ARGUMENT),
    ("max_tokens", 0, _abi.MOT_ERR_INVALID_ARGUMENT),
    ("lora_alpha", float("nan"), _abi.MOT_ERR_INVALID_ARGUMENT),
])
def test_mlp_config_validation(L, field, value, status):
    ws = c_size_t()
    assert L.mot_mlp_query_sizes(byref(mlp_cfg(**{field: value})), 16, byref(ws), None) == status


def test_mlp_create_rejects_bad_arguments_before_cuda(L):
    out = c_void_p(1)
    w = _abi.MotMlpWeights()
    assert L.mot_mlp_create(byref(mlp_cfg()), byref(w), None, byref(out)) == _abi.MOT_ERR_INVALID_ARGUMENT
    assert out.value is None
    # base weights present but the adapters missing at rank 32
    w.w_gate, w.w_up, w.w_down = 4096, 8192, 12288
    assert L.mot_mlp_create(byref(mlp_cfg()), byref(w), None, byref(out)) == _abi.MOT_ERR_INVALID_ARGUMENT
    # misaligned base weight
    w2 = _abi.MotMlpWeights(w_gate=4097, w_up=8192, w_down=12288)
    assert L.mot_mlp_create(byref(mlp_cfg(lora_rank=0)), byref(w2), None, byref(out)) == _abi.MOT_ERR_ALIGNMENT
    assert L.mot_mlp_create(byref(mlp_cfg()), byref(w), None, None) == _abi.MOT_ERR_INVALID_ARGUMENT


def test_moe_query_workspace(L):
    ws = c_size_t()
    T, K, d, I = 8192, 8, 2048, 768
    assert L.mot_moe_query_workspace(byref(moe_cfg()), T, byref(ws)) == _abi.MOT_OK
    # at least the permuted token copies (bf16 [T K, d]), the experts'
    # activations and outputs (f16 [T K, I] and [T K, d])
    assert ws.value >= T * K * (2 * d + 2 * I + 2 * d)
    small = c_size_t()
    assert L.mot_moe_query_workspace(byref(moe_cfg()), 1, byref(small)) == _abi.MOT_OK
    assert 0 < small.value < ws.value
    assert L.mot_moe_query_workspace(byref(moe_cfg()), 0, byref(ws)) == _abi.MOT_ERR_INVALID_ARGUMENT
    assert L.mot_moe_query_workspace(byref(moe_cfg()), T + 1, byref(ws)) == _abi.MOT_ERR_UNSUPPORTED_SHAPE
    assert L.mot_moe_query_workspace(byref(moe_cfg()), T, None) == _abi.MOT_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("field,value,status", [
    ("experts", 33, _abi.MOT_ERR_UNSUPPORTED_SHAPE),
    ("top_k", 9, _abi.MOT_ERR_UNSUPPORTED_SHAPE),
    ("hidden", 2000, _abi.MOT_ERR_UNSUPPORTED_SHAPE),
    ("intermediate", 700, _abi.MOT_ERR_UNSUPPORTED_SHAPE),
    ("experts", 0, _abi.MOT_ERR_INVALID_ARGUMENT),
    ("top_k", 0, _abi.MOT_ERR_INVALID_ARGUMENT),
    ("max_tokens", -1, _abi.MOT_ERR_INVALID_ARGUMENT),
])
def test_moe_config_validation(L, field, value, status):
    ws = c_size_t()
    assert L.mot_moe_query_workspace(byref(moe_cfg(**{field: value})), 16, byref(ws)) == status


def test_moe_top_k_above_experts_is_refused(L):
    ws = c_size_t()
    assert L.mot_moe_query_workspace(byref(moe_cfg(experts=4, top_k=6)), 16, byref(ws)) == \
        _abi.MOT_ERR_UNSUPPORTED_SHAPE


def test_moe_create_rejects_bad_arguments_before_cuda(L):
    out = c_void_p(1)
    w = _abi.MotMoeWeights()
    assert L.mot_moe_create(byref(moe_cfg()), byref(w), None, byref(out)) == _abi.MOT_ERR_INVALID_ARGUMENT
    assert out.value is None
    w = _abi.MotMoeWeights(w_router=4096, w_gate=8192, w_up=12288, w_down=16392)
    assert L.mot_moe_create(byref(moe_cfg()), byref(w), None, byref(out)) == _abi.MOT_ERR_ALIGNMENT


def test_step_create_rejects_bad_arguments_before_cuda(L):
    out = c_void_p(1)
    cfg = _abi.MotStepConfig(n_layers=1, hidden=4096, patch_dim=3072, rms_eps=1e-6)
    handles = (c_void_p * 1)(None)
    norms = (c_void_p * 1)(4096)
    model = _abi.MotStepModel(attn=ctypes.cast(handles, POINTER(c_void_p)), mlp=ctypes.cast(handles, POINTER(c_void_p)),
                              norm_in=ctypes.cast(norms, POINTER(c_void_p)),
                              norm_post=ctypes.cast(norms, POINTER(c_void_p)), w_in=8192, norm_out=12288,
                              w_out=16384)
    # a layer without its attention / MLP handle
    assert L.mot_step_create(byref(cfg), byref(model), None, byref(out)) == _abi.MOT_ERR_INVALID_ARGUMENT
    assert out.value is None
    # shapes the kernels do not take, refused before any handle is read
    bad = _abi.MotStepConfig(n_layers=1, hidden=4000, patch_dim=3072, rms_eps=1e-6)
    assert L.mot_step_create(byref(bad), byref(model), None, byref(out)) == _abi.MOT_ERR_UNSUPPORTED_SHAPE
    bad = _abi.MotStepConfig(n_layers=1, hidden=4096, patch_dim=3000, rms_eps=1e-6)
    assert L.mot_step_create(byref(bad), byref(model), None, byref(out)) == _abi.MOT_ERR_UNSUPPORTED_SHAPE
    for bad in (_abi.MotStepConfig(n_layers=0, hidden=4096, patch_dim=3072, rms_eps=1e-6),
                _abi.MotStepConfig(n_layers=1, hidden=4096, patch_dim=3072, rms_eps=-1.0)):
        assert L.mot_step_create(byref(bad), byref(model), None, byref(out)) == _abi.MOT_ERR_INVALID_ARGUMENT
    assert L.mot_step_create(byref(cfg), None, None, byref(out)) == _abi.MOT_ERR_INVALID_ARGUMENT


def test_bindings_refuse_host_tensors_and_wrong_dtypes():
    # a host tensor where the C call takes a device pointer would hand the
    # kernels a host address: refused in the binding, before the call
    import torch
    from mot_flow_matching_b200.layer import _dptr, mot_attn_forward
    from mot_flow_matching_b200.moe import mot_moe_forward
    with pytest.raises(ValueError, match="CUDA"):
        _dptr(torch.zeros(4, dtype=torch.bfloat16), torch.bfloat16, "x")
    with pytest.raises(ValueError, match="CUDA"):
        mot_attn_forward(c_void_p(1), torch.zeros(1, 16, 512, dtype=torch.bfloat16), 1, 16, None, None, [0], 0,
                         torch.zeros(1, 16, 512, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="CUDA"):
        mot_moe_forward(c_void_p(1), torch.zeros(4, 256, dtype=torch.bfloat16), 4,
                        torch.zeros(4, 256, dtype=torch.bfloat16))
    assert _dptr(None, torch.float32) is None

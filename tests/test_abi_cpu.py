"""Host-only checks of the C ABI: the library builds, loads and exports every
function the headers declare; sizing and argument validation run on the host
before any CUDA call (no GPU needed)."""
import ctypes
import os
import re
from ctypes import byref, c_size_t, c_void_p

import pytest

from mot_flow_matching_b200 import build as build_mod
from mot_flow_matching_b200 import _abi
from mot_flow_matching_b200.layer import make_config

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build_mod.build()
    return _abi.lib()


def header_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(mot_\w+)\s*\(", text))
    return names


def test_every_declared_symbol_is_exported(L):
    names = header_functions()
    assert {"mot_attn_create", "mot_attn_forward", "mot_attn_backward", "mot_attn_merge_lora"} <= names
    cdll = ctypes.CDLL(_abi.LIB_PATH)
    for n in sorted(names):
        assert hasattr(cdll, n), n
    assert names == set(_abi.SIGNATURES), "binding and headers disagree"


def test_status_strings(L):
    for s in range(9):
        assert L.mot_status_string(s).decode()
    assert L.mot_status_string(99).decode() == "unknown status"


def test_query_sizes_host_only(L):
    cfg = make_config(lora_rank=32, lora_alpha=32, max_batch=2, max_img_tokens=4096, max_prefix=400)
    ws, sv = c_size_t(), c_size_t()
    assert L.mot_attn_query_sizes(byref(cfg), 2, 4096, 400, byref(ws), byref(sv)) == _abi.MOT_OK
    # activations at least: q^ (2*32*4096*128*2) + K,V (2*8*4608*128*2 each) + o (8192*4096*2)
    assert sv.value >= 2 * 32 * 4096 * 256 + 2 * 2 * 8 * 4608 * 256 + 8192 * 4096 * 2
    assert ws.value >= 2 * 32 * 4096 * 256
    assert L.mot_attn_query_sizes(byref(cfg), 3, 4096, 400, byref(ws), byref(sv)) == _abi.MOT_ERR_UNSUPPORTED_SHAPE
    assert L.mot_attn_query_sizes(byref(cfg), 0, 4096, 400, byref(ws), byref(sv)) == _abi.MOT_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("field,value,status", [
    ("head_dim", 64, _abi.MOT_ERR_UNSUPPORTED_SHAPE),
    ("n_kv_heads", 5, _abi.MOT_ERR_UNSUPPORTED_SHAPE),
    ("lora_rank", 12, _abi.MOT_ERR_UNSUPPORTED_SHAPE),
    ("lora_rank", 256, _abi.MOT_ERR_UNSUPPORTED_SHAPE),
    ("max_batch", 65, _abi.MOT_ERR_UNSUPPORTED_SHAPE),
    ("hidden", -1, _abi.MOT_ERR_INVALID_ARGUMENT),
    ("rope_theta", 0.0, _abi.MOT_ERR_INVALID_ARGUMENT),
])
def test_config_validation(L, field, value, status):
    cfg = make_config(lora_rank=16, lora_alpha=16)
    setattr(cfg, field, value)
    ws, sv = c_size_t(), c_size_t()
    assert L.mot_attn_query_sizes(byref(cfg), 1, 16, 0, byref(ws), byref(sv)) == status


def test_create_rejects_bad_arguments_before_cuda(L):
    cfg = make_config(lora_rank=16, lora_alpha=16)
    out = c_void_p(1)
    w = _abi.MotAttnWeights()
    assert L.mot_attn_create(byref(cfg), byref(w), None, byref(out)) == _abi.MOT_ERR_INVALID_ARGUMENT
    assert out.value is None
    # misaligned weight pointers are refused on the host
    vals = [0x1000 * (i + 1) for i in range(14)]
    vals[3] += 2
    w = _abi.MotAttnWeights(*[c_void_p(v) for v in vals])
    assert L.mot_attn_create(byref(cfg), byref(w), None, byref(out)) == _abi.MOT_ERR_ALIGNMENT
    assert L.mot_attn_create(None, byref(w), None, byref(out)) == _abi.MOT_ERR_INVALID_ARGUMENT


def test_forward_backward_reject_null_handle(L):
    assert L.mot_attn_forward(None, None, 1, 1, None, None, None, 0, None, None, None, 0, None, 0, None) \
        == _abi.MOT_ERR_INVALID_ARGUMENT
    assert L.mot_attn_backward(None, None, None, 1, 1, None, None, None, 0, None, 0, None, None, None, None, 0,
                               None, 0, None) == _abi.MOT_ERR_INVALID_ARGUMENT
    assert L.mot_attn_merge_lora(None, None, None, None, None, None) == _abi.MOT_ERR_INVALID_ARGUMENT
    assert L.mot_attn_last_launch_count(None) == 0
    L.mot_attn_destroy(None)


def test_host_staging_size_host_only(L):
    cfg = make_config(lora_rank=32, lora_alpha=32, max_batch=2, max_img_tokens=4096, max_prefix=400)
    n = c_size_t()
    assert L.mot_attn_query_host_staging(byref(cfg), 2, 4096, 400, byref(n)) == _abi.MOT_OK
    # two slots of x and y (2*4096*4096 bf16 each) and the two caches (2*8*400*128 bf16 each)
    x = 2 * 4096 * 4096 * 2
    kv = 2 * 8 * 400 * 128 * 2
    assert n.value == 2 * (2 * x + 2 * kv)
    assert L.mot_attn_query_host_staging(byref(cfg), 2, 4096, 0, byref(n)) == _abi.MOT_OK
    assert n.value == 2 * 2 * x
    assert L.mot_attn_query_host_staging(byref(cfg), 3, 4096, 400, byref(n)) == _abi.MOT_ERR_UNSUPPORTED_SHAPE
    assert L.mot_attn_query_host_staging(byref(cfg), 2, 4096, 400, None) == _abi.MOT_ERR_INVALID_ARGUMENT


def test_forward_host_rejects_bad_arguments_before_cuda(L):
    one = (c_void_p * 1)(None)
    pl = (ctypes.c_int32 * 1)(0)
    # no handle, no calls, null buffer arrays: rejected on the host
    assert L.mot_attn_forward_host(None, 1, one, 1, 16, None, None, pl, 0, one, None, 0, None, 0, None) \
        == _abi.MOT_ERR_INVALID_ARGUMENT
    assert L.mot_attn_forward_host(None, 0, one, 1, 16, None, None, pl, 0, one, None, 0, None, 0, None) \
        == _abi.MOT_ERR_INVALID_ARGUMENT

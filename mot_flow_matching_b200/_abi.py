"""ctypes declarations of the C ABI in include/mot_attn.h and include/mot_attn_dev.h.

Loading fails loudly (ImportError) when libmotattn.so is missing: there is no
fallback path. Build it with ``python -m mot_flow_matching_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_double, c_float, c_int32, c_size_t, c_void_p

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmotattn.so")

# status codes (mot_status)
MOT_OK = 0
MOT_ERR_INVALID_ARGUMENT = 1
MOT_ERR_UNSUPPORTED_SHAPE = 2
MOT_ERR_ALIGNMENT = 3
MOT_ERR_WORKSPACE_TOO_SMALL = 4
MOT_ERR_NO_SAVED_STATE = 5
MOT_ERR_CUDA = 6
MOT_ERR_NUMERIC = 7
MOT_ERR_TIMEOUT = 8


class MotAttnConfig(ctypes.Structure):
    _fields_ = [
        ("hidden", c_int32), ("n_q_heads", c_int32), ("n_kv_heads", c_int32), ("head_dim", c_int32),
        ("lora_rank", c_int32), ("lora_alpha", c_float), ("rms_eps", c_float), ("rope_theta", c_double),
        ("max_batch", c_int32), ("max_img_tokens", c_int32), ("max_prefix", c_int32),
        ("enable_backward", c_int32),
    ]


class MotAttnWeights(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in ("w_q", "w_k", "w_v", "w_o", "q_norm", "k_norm", "a_q", "a_k", "a_v",
                                        "a_o", "b_q", "b_k", "b_v", "b_o")]


class MotMlpConfig(ctypes.Structure):
    _fields_ = [("hidden", c_int32), ("intermediate", c_int32), ("lora_rank", c_int32), ("lora_alpha", c_float),
                ("max_tokens", c_int32), ("enable_backward", c_int32)]


class MotMlpWeights(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in ("w_gate", "w_up", "w_down", "a_gate", "a_up", "a_down", "b_gate", "b_up",
                                        "b_down")]


class MotStepConfig(ctypes.Structure):
    _fields_ = [("n_layers", c_int32), ("hidden", c_int32), ("patch_dim", c_int32), ("rms_eps", c_float)]


class MotStepModel(ctypes.Structure):
    _fields_ = [("attn", POINTER(c_void_p)), ("mlp", POINTER(c_void_p)), ("norm_in", POINTER(c_void_p)),
                ("norm_post", POINTER(c_void_p)), ("w_in", c_void_p), ("norm_out", c_void_p), ("w_out", c_void_p)]


class MotMoeConfig(ctypes.Structure):
    _fields_ = [("hidden", c_int32), ("intermediate", c_int32), ("experts", c_int32), ("top_k", c_int32),
                ("max_tokens", c_int32)]


class MotMoeWeights(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in ("w_router", "w_gate", "w_up", "w_down")]


# name -> (restype, argtypes); every symbol the headers declare
SIGNATURES = {
    "mot_attn_query_sizes": (c_int32, [POINTER(MotAttnConfig), c_int32, c_int32, c_int32, POINTER(c_size_t),
                                       POINTER(c_size_t)]),
    "mot_attn_create": (c_int32, [POINTER(MotAttnConfig), POINTER(MotAttnWeights), c_void_p, POINTER(c_void_p)]),
    "mot_attn_forward": (c_int32, [c_void_p, c_void_p, c_int32, c_int32, c_void_p, c_void_p, POINTER(c_int32),
                                   c_int32, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p, c_size_t, c_void_p]),
    "mot_attn_backward": (c_int32, [c_void_p, c_void_p, c_void_p, c_int32, c_int32, c_void_p, c_void_p,
                                    POINTER(c_int32), c_int32, c_void_p, c_size_t, c_void_p, c_void_p,
                                    POINTER(c_void_p), POINTER(c_void_p), c_int32, c_void_p, c_size_t, c_void_p]),
    "mot_attn_prefix_forward": (c_int32, [c_void_p, c_void_p, c_int32, c_int32, POINTER(c_int32), c_void_p,
                                          c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "mot_attn_forward_noalloc": (c_int32, [c_void_p, c_void_p, c_int32, c_int32, c_void_p, c_void_p,
                                           POINTER(c_int32), c_int32, c_void_p, c_void_p, c_void_p]),
    "mot_attn_query_host_staging": (c_int32, [POINTER(MotAttnConfig), c_int32, c_int32, c_int32,
                                              POINTER(c_size_t)]),
    "mot_attn_forward_host": (c_int32, [c_void_p, c_int32, POINTER(c_void_p), c_int32, c_int32, POINTER(c_void_p),
                                        POINTER(c_void_p), POINTER(c_int32), c_int32, POINTER(c_void_p), c_void_p,
                                        c_size_t, c_void_p, c_size_t, c_void_p]),
    "mot_attn_merge_lora": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "mot_attn_get_device_status": (c_int32, [c_void_p, c_void_p]),
    "mot_attn_destroy": (None, [c_void_p]),
    "mot_status_string": (c_char_p, [c_int32]),
    "mot_attn_last_launch_count": (c_int32, [c_void_p]),
    "mot_dev_gemm": (c_int32, [c_void_p, c_void_p, c_void_p, c_int32, c_int32, c_int32, c_int32, c_int32, c_void_p]),
    "mot_dev_gemm_variant": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_int32, c_int32, c_int32, c_int32,
                                       c_int32, c_void_p]),
    "mot_dev_exp2_poly": (c_int32, [c_void_p, c_void_p, c_int32, c_void_p]),
    "mot_dev_profile": (c_int32, [c_void_p, c_int32]),
    "mot_dev_stage_times": (c_int32, [c_void_p, POINTER(c_int32), POINTER(c_float), c_int32, POINTER(c_int32)]),
    "mot_dev_stage_name": (c_char_p, [c_int32]),
    "mot_dev_wait_probe": (c_int32, [c_void_p, c_void_p]),
    "mot_dev_set_attn_splits": (c_int32, [c_void_p, c_int32]),
    "mot_dev_last_attn_splits": (c_int32, [c_void_p]),
    "mot_dev_last_attn_full_units": (c_int32, [c_void_p]),
    "mot_dev_stage_timeline": (c_int32, [c_void_p, POINTER(c_int32), POINTER(c_float), POINTER(c_float), c_int32,
                                         POINTER(c_int32)]),
    "mot_dev_saved_layout": (c_int32, [POINTER(MotAttnConfig), c_int32, c_int32, c_int32, POINTER(c_size_t),
                                       POINTER(c_int32)]),
    "mot_mlp_query_sizes": (c_int32, [POINTER(MotMlpConfig), c_int32, POINTER(c_size_t), POINTER(c_size_t)]),
    "mot_mlp_create": (c_int32, [POINTER(MotMlpConfig), POINTER(MotMlpWeights), c_void_p, POINTER(c_void_p)]),
    "mot_mlp_forward": (c_int32, [c_void_p, c_void_p, c_int32, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p,
                                  c_size_t, c_void_p]),
    "mot_mlp_backward": (c_int32, [c_void_p, c_void_p, c_void_p, c_int32, c_void_p, c_size_t, c_void_p, c_void_p,
                                   POINTER(c_void_p), POINTER(c_void_p), c_int32, c_void_p, c_size_t, c_void_p]),
    "mot_mlp_get_device_status": (c_int32, [c_void_p, c_void_p]),
    "mot_mlp_last_launch_count": (c_int32, [c_void_p]),
    "mot_mlp_destroy": (None, [c_void_p]),
    "mot_dev_mlp_profile": (c_int32, [c_void_p, c_int32]),
    "mot_dev_mlp_stage_times": (c_int32, [c_void_p, POINTER(c_int32), POINTER(c_float), c_int32, POINTER(c_int32)]),
    "mot_dev_mlp_stage_name": (c_char_p, [c_int32]),
    "mot_step_create": (c_int32, [POINTER(MotStepConfig), POINTER(MotStepModel), c_void_p, POINTER(c_void_p)]),
    "mot_step_query_workspace": (c_int32, [c_void_p, c_int32, c_int32, c_int32, POINTER(c_size_t)]),
    "mot_step_forward": (c_int32, [c_void_p, c_void_p, c_int32, c_int32, POINTER(c_void_p), POINTER(c_void_p),
                                   POINTER(c_int32), c_int32, c_float, c_float, c_float, c_float, c_float, c_void_p,
                                   c_void_p, c_void_p, c_size_t, c_void_p]),
    "mot_step_destroy": (None, [c_void_p]),
    "mot_moe_query_workspace": (c_int32, [POINTER(MotMoeConfig), c_int32, POINTER(c_size_t)]),
    "mot_moe_create": (c_int32, [POINTER(MotMoeConfig), POINTER(MotMoeWeights), c_void_p, POINTER(c_void_p)]),
    "mot_moe_forward": (c_int32, [c_void_p, c_void_p, c_int32, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                  c_void_p]),
    "mot_moe_get_device_status": (c_int32, [c_void_p, c_void_p]),
    "mot_moe_destroy": (None, [c_void_p]),
}

_lib = None


def lib():
    """The loaded library with prototypes set (ImportError if not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with python -m mot_flow_matching_b200.build")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


class MotError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib().mot_status_string(status).decode()
        super().__init__(f"{where}: {msg} (status {status})")


def check(status: int, where: str) -> None:
    if status != MOT_OK:
        raise MotError(status, where)

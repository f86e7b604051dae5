"""Python binding of the MLP half of the C ABI (include/mot_mlp.h):
argument marshalling only; every step runs in libmotattn.so.

The functions carry the C names and take torch tensors where the C call
takes device pointers. ``MotMlp`` bundles a handle with the buffers a caller
needs.
"""
from __future__ import annotations

import ctypes
from ctypes import byref, c_int32, c_size_t, c_void_p
from typing import Dict, Optional, Tuple

import torch

from ._abi import MotMlpConfig, MotMlpWeights, check, lib
from .layer import _BF16, _F32, _dptr, _stream

MLP_WEIGHT_NAMES = ("w_gate", "w_up", "w_down", "a_gate", "a_up", "a_down", "b_gate", "b_up", "b_down")


def make_mlp_config(hidden=4096, intermediate=12288, lora_rank=0, lora_alpha=0.0, max_tokens=256,
                    enable_backward=False) -> MotMlpConfig:
    return MotMlpConfig(hidden, intermediate, lora_rank, float(lora_alpha), max_tokens, int(bool(enable_backward)))


def mot_mlp_query_sizes(cfg: MotMlpConfig, tokens: int) -> Tuple[int, int]:
    ws, sv = c_size_t(0), c_size_t(0)
    check(lib().mot_mlp_query_sizes(byref(cfg), tokens, byref(ws), byref(sv)), "mot_mlp_query_sizes")
    return ws.value, sv.value


def mot_mlp_create(cfg: MotMlpConfig, weights: Dict[str, torch.Tensor], stream=None) -> c_void_p:
    w = MotMlpWeights(*[_dptr(weights.get(n), _BF16, n) for n in MLP_WEIGHT_NAMES])
    h = c_void_p()
    check(lib().mot_mlp_create(byref(cfg), byref(w), _stream(stream), byref(h)), "mot_mlp_create")
    return h


def mot_mlp_forward(h, x, tokens, y, y_f32=None, saved=None, workspace=None, stream=None) -> None:
    check(lib().mot_mlp_forward(h, _dptr(x, _BF16, "x"), tokens, _dptr(y, _BF16, "y"), _dptr(y_f32, _F32, "y_f32"),
                                _dptr(saved, None, "saved"), saved.numel() if saved is not None else 0,
                                _dptr(workspace, None, "workspace"),
                                workspace.numel() if workspace is not None else 0, _stream(stream)),
          "mot_mlp_forward")


def mot_mlp_backward(h, dy, x, tokens, saved, dx, dx_f32=None, d_a=None, d_b=None, accumulate=False,
                     workspace=None, stream=None) -> None:
    da = (c_void_p * 3)(*[_dptr(t, _F32, "d_a") for t in (d_a or [None] * 3)])
    db = (c_void_p * 3)(*[_dptr(t, _F32, "d_b") for t in (d_b or [None] * 3)])
    check(lib().mot_mlp_backward(h, _dptr(dy, _BF16, "dy"), _dptr(x, _BF16, "x"), tokens, _dptr(saved, None, "saved"),
                                 saved.numel(), _dptr(dx, _BF16, "dx"), _dptr(dx_f32, _F32, "dx_f32"),
                                 da, db, int(bool(accumulate)), _dptr(workspace, None, "workspace"),
                                 workspace.numel() if workspace is not None else 0, _stream(stream)),
          "mot_mlp_backward")


def mot_mlp_get_device_status(h, stream=None) -> int:
    return int(lib().mot_mlp_get_device_status(h, _stream(stream)))


def mot_mlp_last_launch_count(h) -> int:
    return int(lib().mot_mlp_last_launch_count(h))


def mot_mlp_destroy(h) -> None:
    lib().mot_mlp_destroy(h)


def mot_dev_mlp_profile(h, enable: bool) -> None:
    check(lib().mot_dev_mlp_profile(h, int(bool(enable))), "mot_dev_mlp_profile")


def mot_dev_mlp_stage_times(h, max_stages: int = 32):
    ids = (c_int32 * max_stages)()
    ms = (ctypes.c_float * max_stages)()
    count = c_int32(0)
    check(lib().mot_dev_mlp_stage_times(h, ids, ms, max_stages, byref(count)), "mot_dev_mlp_stage_times")
    return [(lib().mot_dev_mlp_stage_name(ids[i]).decode(), ms[i]) for i in range(min(count.value, max_stages))]


class MotMlp:
    """An MLP handle plus the caller-owned buffers of one call shape."""

    def __init__(self, weights: Dict[str, torch.Tensor], lora_rank: int = 0, lora_alpha: float = 0.0,
                 max_tokens: int = 256, enable_backward: bool = False, hidden: int = 4096,
                 intermediate: int = 12288, stream=None):
        self.cfg = make_mlp_config(hidden, intermediate, lora_rank, lora_alpha, max_tokens, enable_backward)
        self.weights = dict(weights)
        self.handle = mot_mlp_create(self.cfg, self.weights, stream)
        self._ws = None

    def sizes(self, tokens):
        return mot_mlp_query_sizes(self.cfg, tokens)

    def workspace(self, tokens, device="cuda"):
        ws, _ = self.sizes(tokens)
        if self._ws is None or self._ws.numel() < ws:
            self._ws = torch.empty(ws, dtype=torch.uint8, device=device)
        return self._ws

    def new_saved(self, tokens, device="cuda"):
        _, sv = self.sizes(tokens)
        return torch.empty(sv, dtype=torch.uint8, device=device)

    def forward(self, x, y=None, y_f32=None, saved=None, workspace=None, stream=None):
        T = x.shape[0]
        if y is None:
            y = torch.empty_like(x)
        if workspace is None:
            workspace = self.workspace(T, x.device)
        mot_mlp_forward(self.handle, x, T, y, y_f32, saved, workspace, stream)
        return y

    def backward(self, dy, x, saved, dx=None, dx_f32=None, d_a=None, d_b=None, accumulate=False, workspace=None,
                 stream=None):
        T = x.shape[0]
        if dx is None:
            dx = torch.empty_like(x)
        if workspace is None:
            workspace = self.workspace(T, x.device)
        mot_mlp_backward(self.handle, dy, x, T, saved, dx, dx_f32, d_a, d_b, accumulate, workspace, stream)
        return dx

    def device_status(self, stream=None) -> int:
        return mot_mlp_get_device_status(self.handle, stream)

    def last_launch_count(self) -> int:
        return mot_mlp_last_launch_count(self.handle)

    def close(self):
        if self.handle is not None:
            mot_mlp_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

"""Python binding of the mixture-of-experts part of the C ABI
(include/mot_moe.h): argument marshalling only; routing, dispatch, the
expert GEMMs and the combine run in libmotattn.so."""
from __future__ import annotations

from ctypes import byref, c_size_t, c_void_p
from typing import Dict

import torch

from ._abi import MotMoeConfig, MotMoeWeights, check, lib
from .layer import _BF16, _F32, _I32, _dptr, _stream


def mot_moe_query_workspace(cfg: MotMoeConfig, tokens: int) -> int:
    n = c_size_t(0)
    check(lib().mot_moe_query_workspace(byref(cfg), tokens, byref(n)), "mot_moe_query_workspace")
    return n.value


def mot_moe_create(cfg: MotMoeConfig, weights: Dict[str, torch.Tensor], stream=None) -> c_void_p:
    w = MotMoeWeights(*[_dptr(weights[n], _BF16, n) for n in ("w_router", "w_gate", "w_up", "w_down")])
    h = c_void_p()
    check(lib().mot_moe_create(byref(cfg), byref(w), _stream(stream), byref(h)), "mot_moe_create")
    return h


def mot_moe_forward(h, x, tokens, y, y_f32=None, experts_out=None, workspace=None, stream=None) -> None:
    check(lib().mot_moe_forward(h, _dptr(x, _BF16, "x"), tokens, _dptr(y, _BF16, "y"), _dptr(y_f32, _F32, "y_f32"),
                                _dptr(experts_out, _I32, "experts_out"), _dptr(workspace, None, "workspace"),
                                workspace.numel() if workspace is not None else 0, _stream(stream)),
          "mot_moe_forward")


class MotMoe:
    """A MoE MLP handle plus its workspace."""

    def __init__(self, weights: Dict[str, torch.Tensor], top_k: int = 8, max_tokens: int = 256, stream=None):
        E, I, d = weights["w_gate"].shape
        self.cfg = MotMoeConfig(d, I, E, top_k, max_tokens)
        self.weights = dict(weights)
        self.handle = mot_moe_create(self.cfg, self.weights, stream)
        self._ws = None

    def workspace(self, tokens, device="cuda"):
        n = mot_moe_query_workspace(self.cfg, tokens)
        if self._ws is None or self._ws.numel() < n:
            self._ws = torch.empty(n, dtype=torch.uint8, device=device)
        return self._ws

    def forward(self, x, y=None, y_f32=None, experts_out=None, workspace=None, stream=None):
        T = x.shape[0]
        if y is None:
            y = torch.empty_like(x)
        if workspace is None:
            workspace = self.workspace(T, x.device)
        mot_moe_forward(self.handle, x, T, y, y_f32, experts_out, workspace, stream)
        return y

    def device_status(self, stream=None) -> int:
        return int(lib().mot_moe_get_device_status(self.handle, _stream(stream)))

    def close(self):
        if self.handle is not None:
            lib().mot_moe_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

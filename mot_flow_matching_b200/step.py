"""Python binding of the denoise-step part of the C ABI (include/mot_step.h):
argument marshalling only; every step of the tower runs in libmotattn.so.

``MotStep`` ties a stack of attention (``layer.MotAttnLayer``) and MLP
(``mlp.MotMlp``) handles, one pair per decoder layer, to the step handle.
"""
from __future__ import annotations

from ctypes import byref, c_int32, c_size_t, c_void_p
from typing import Sequence

import torch

from ._abi import MotStepConfig, MotStepModel, check, lib
from .layer import _BF16, _F32, _dptr, _stream


def mot_step_create(cfg: MotStepConfig, attn_handles, mlp_handles, norm_in, norm_post, w_in, norm_out, w_out,
                    stream=None) -> c_void_p:
    n = cfg.n_layers
    arr = lambda xs: (c_void_p * n)(*[x.value if isinstance(x, c_void_p) else x for x in xs])
    model = MotStepModel(arr(attn_handles), arr(mlp_handles), arr([_dptr(t, _BF16, "norm_in") for t in norm_in]),
                         arr([_dptr(t, _BF16, "norm_post") for t in norm_post]), _dptr(w_in, _BF16, "w_in"),
                         _dptr(norm_out, _BF16, "norm_out"), _dptr(w_out, _BF16, "w_out"))
    h = c_void_p()
    check(lib().mot_step_create(byref(cfg), byref(model), _stream(stream), byref(h)), "mot_step_create")
    return h


def mot_step_query_workspace(h, batch, img_tokens, prefix_max) -> int:
    n = c_size_t(0)
    check(lib().mot_step_query_workspace(h, batch, img_tokens, prefix_max, byref(n)), "mot_step_query_workspace")
    return n.value


def mot_step_forward(h, z, batch, img_tokens, k_caches, v_caches, prefix_len: Sequence[int], prefix_max, sigma,
                     sigma_next, cfg_scale, img_cfg_scale, t_eps, z_next, z_next_bf16=None, workspace=None,
                     stream=None) -> None:
    n = len(k_caches)
    kc = (c_void_p * n)(*[_dptr(t, _BF16, "k_cache") for t in k_caches])
    vc = (c_void_p * n)(*[_dptr(t, _BF16, "v_cache") for t in v_caches])
    pl = (c_int32 * batch)(*[int(v) for v in prefix_len])
    check(lib().mot_step_forward(h, _dptr(z, _F32, "z"), batch, img_tokens, kc, vc, pl, prefix_max, float(sigma),
                                 float(sigma_next), float(cfg_scale), float(img_cfg_scale), float(t_eps),
                                 _dptr(z_next, _F32, "z_next"), _dptr(z_next_bf16, _BF16, "z_next_bf16"),
                                 _dptr(workspace, None, "workspace"),
                                 workspace.numel() if workspace is not None else 0, _stream(stream)),
          "mot_step_forward")


def mot_step_destroy(h) -> None:
    lib().mot_step_destroy(h)


class MotStep:
    """A denoise-step handle over per-layer attention and MLP objects (kept
    alive here), with its workspace."""

    def __init__(self, attn_layers, mlps, norm_in, norm_post, w_in, norm_out, w_out, rms_eps=1e-6, stream=None):
        self.attn_layers, self.mlps = list(attn_layers), list(mlps)
        self.tensors = [list(norm_in), list(norm_post), w_in, norm_out, w_out]
        hidden, patch = w_in.shape
        self.cfg = MotStepConfig(len(self.attn_layers), hidden, patch, float(rms_eps))
        self.handle = mot_step_create(self.cfg, [a.handle for a in self.attn_layers], [m.handle for m in self.mlps],
                                      norm_in, norm_post, w_in, norm_out, w_out, stream)
        self._ws = None

    def workspace(self, batch, img_tokens, prefix_max, device="cuda"):
        n = mot_step_query_workspace(self.handle, batch, img_tokens, prefix_max)
        if self._ws is None or self._ws.numel() < n:
            self._ws = torch.empty(n, dtype=torch.uint8, device=device)
        return self._ws

    def forward(self, z, k_caches, v_caches, prefix_len, sigma, sigma_next, cfg_scale=4.0, img_cfg_scale=1.0,
                t_eps=0.02, z_next=None, z_next_bf16=None, workspace=None, stream=None):
        N = z.shape[0]
        B = len(prefix_len)
        P = k_caches[0].shape[2] if k_caches else 0
        if z_next is None:
            z_next = torch.empty_like(z)
        if workspace is None:
            workspace = self.workspace(B, N, P, z.device)
        mot_step_forward(self.handle, z, B, N, k_caches, v_caches, prefix_len, P, sigma, sigma_next, cfg_scale,
                         img_cfg_scale, t_eps, z_next, z_next_bf16, workspace, stream)
        return z_next

    def close(self):
        if self.handle is not None:
            mot_step_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

"""Python binding of the C ABI: argument marshalling only.

The module-level functions carry the C names (``mot_attn_create``,
``mot_attn_forward``, ...) and take torch tensors where the C call takes
device pointers; every step of the layer runs in libmotattn.so.
``MotAttnLayer`` bundles a handle with the buffers a caller needs.
"""
from __future__ import annotations

import ctypes
from ctypes import byref, c_int32, c_size_t, c_void_p
from typing import Dict, Optional, Sequence, Tuple

import torch

from ._abi import MotAttnConfig, MotAttnWeights, check, lib

WEIGHT_NAMES = ("w_q", "w_k", "w_v", "w_o", "q_norm", "k_norm", "a_q", "a_k", "a_v", "a_o",
                "b_q", "b_k", "b_v", "b_o")


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libmotattn must be contiguous")
    return c_void_p(t.data_ptr())


_BF16, _F32, _I32 = torch.bfloat16, torch.float32, torch.int32


def _dptr(t: Optional[torch.Tensor], dtype: Optional[torch.dtype] = None, name: str = "tensor"):
    """Pointer of a device argument: a contiguous CUDA tensor (of `dtype`
    when given). A host tensor here would hand the kernels a host address."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (got {t.device})")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype} (got {t.dtype})")
    return _ptr(t)


def _stream(stream) -> c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def make_config(hidden=4096, n_q_heads=32, n_kv_heads=8, head_dim=128, lora_rank=0, lora_alpha=0.0,
                rms_eps=1e-6, rope_theta=1e6, max_batch=1, max_img_tokens=256, max_prefix=0,
                enable_backward=False) -> MotAttnConfig:
    return MotAttnConfig(hidden, n_q_heads, n_kv_heads, head_dim, lora_rank, float(lora_alpha), float(rms_eps),
                         float(rope_theta), max_batch, max_img_tokens, max_prefix, int(bool(enable_backward)))


def mot_attn_query_sizes(cfg: MotAttnConfig, batch: int, img_tokens: int, prefix_max: int) -> Tuple[int, int]:
    ws, sv = c_size_t(0), c_size_t(0)
    check(lib().mot_attn_query_sizes(byref(cfg), batch, img_tokens, prefix_max, byref(ws), byref(sv)),
          "mot_attn_query_sizes")
    return ws.value, sv.value


def mot_attn_create(cfg: MotAttnConfig, weights: Dict[str, torch.Tensor], stream=None) -> c_void_p:
    w = MotAttnWeights(*[_dptr(weights.get(n), _BF16, n) for n in WEIGHT_NAMES])
    h = c_void_p()
    check(lib().mot_attn_create(byref(cfg), byref(w), _stream(stream), byref(h)), "mot_attn_create")
    return h


def mot_attn_forward(h, x, batch, img_tokens, k_cache, v_cache, prefix_len: Sequence[int], prefix_max, y,
                     y_f32=None, saved=None, workspace=None, stream=None) -> None:
    pl = (c_int32 * batch)(*[int(v) for v in prefix_len])
    check(lib().mot_attn_forward(h, _dptr(x, _BF16, "x"), batch, img_tokens, _dptr(k_cache, _BF16, "k_cache"),
                                 _dptr(v_cache, _BF16, "v_cache"), pl, prefix_max, _dptr(y, _BF16, "y"),
                                 _dptr(y_f32, _F32, "y_f32"), _dptr(saved, None, "saved"),
                                 saved.numel() if saved is not None else 0, _dptr(workspace, None, "workspace"),
                                 workspace.numel() if workspace is not None else 0,
                                 _stream(stream)), "mot_attn_forward")


def mot_attn_prefix_forward(h, x, batch, tokens, lengths: Sequence[int], y, k_cache_out, v_cache_out, y_f32=None,
                            workspace=None, stream=None) -> None:
    """The prefix tower's layer over the prompt (causal), writing the layer's
    bf16 cache entry; see include/mot_attn.h."""
    ln = (c_int32 * batch)(*[int(v) for v in lengths])
    check(lib().mot_attn_prefix_forward(h, _dptr(x, _BF16, "x"), batch, tokens, ln, _dptr(y, _BF16, "y"),
                                        _dptr(y_f32, _F32, "y_f32"), _dptr(k_cache_out, _BF16, "k_cache_out"),
                                        _dptr(v_cache_out, _BF16, "v_cache_out"), _dptr(workspace, None, "workspace"),
                                        workspace.numel() if workspace is not None else 0, _stream(stream)),
          "mot_attn_prefix_forward")


def mot_attn_forward_noalloc(h, x, batch, img_tokens, k_cache, v_cache, prefix_len: Sequence[int], prefix_max,
                             y, y_f32=None, stream=None) -> None:
    """Forward whose scratch is the library's own fixed device array (no
    workspace argument, no allocation); see include/mot_attn.h."""
    pl = (c_int32 * batch)(*[int(v) for v in prefix_len])
    check(lib().mot_attn_forward_noalloc(h, _dptr(x, _BF16, "x"), batch, img_tokens,
                                         _dptr(k_cache, _BF16, "k_cache"), _dptr(v_cache, _BF16, "v_cache"), pl,
                                         prefix_max, _dptr(y, _BF16, "y"), _dptr(y_f32, _F32, "y_f32"),
                                         _stream(stream)),
          "mot_attn_forward_noalloc")


def mot_attn_backward(h, dy, x, batch, img_tokens, k_cache, v_cache, prefix_len: Sequence[int], prefix_max,
                      saved, dx, dx_f32=None, d_a=None, d_b=None, accumulate=False, workspace=None,
                      stream=None) -> None:
    pl = (c_int32 * batch)(*[int(v) for v in prefix_len])
    da = (c_void_p * 4)(*[_dptr(t, _F32, "d_a") for t in (d_a or [None] * 4)])
    db = (c_void_p * 4)(*[_dptr(t, _F32, "d_b") for t in (d_b or [None] * 4)])
    check(lib().mot_attn_backward(h, _dptr(dy, _BF16, "dy"), _dptr(x, _BF16, "x"), batch, img_tokens,
                                  _dptr(k_cache, _BF16, "k_cache"), _dptr(v_cache, _BF16, "v_cache"), pl,
                                  prefix_max, _dptr(saved, None, "saved"), saved.numel() if saved is not None else 0,
                                  _dptr(dx, _BF16, "dx"), _dptr(dx_f32, _F32, "dx_f32"), da, db,
                                  int(bool(accumulate)), _dptr(workspace, None, "workspace"),
                                  workspace.numel() if workspace is not None else 0, _stream(stream)),
          "mot_attn_backward")


def mot_attn_query_host_staging(cfg: MotAttnConfig, batch: int, img_tokens: int, prefix_max: int) -> int:
    n = c_size_t(0)
    check(lib().mot_attn_query_host_staging(byref(cfg), batch, img_tokens, prefix_max, byref(n)),
          "mot_attn_query_host_staging")
    return n.value


def _host_ptrs(ts: Sequence[Optional[torch.Tensor]]):
    for t in ts:
        if t is not None and (t.is_cuda or not t.is_contiguous()):
            raise ValueError("host buffers must be contiguous CPU tensors")
    return (c_void_p * len(ts))(*[t.data_ptr() if t is not None else None for t in ts])


def mot_attn_forward_host(h, xs, batch, img_tokens, k_caches, v_caches, prefix_len: Sequence[int], prefix_max,
                          ys, staging, workspace, stream=None) -> None:
    steps = len(xs)
    if len(ys) != steps or (k_caches is not None and len(k_caches) != steps) or \
            (v_caches is not None and len(v_caches) != steps):
        raise ValueError("one x, y (and cache) buffer per call")
    pl = (c_int32 * batch)(*[int(v) for v in prefix_len])
    kc = _host_ptrs(k_caches) if k_caches is not None else None
    vc = _host_ptrs(v_caches) if v_caches is not None else None
    check(lib().mot_attn_forward_host(h, steps, _host_ptrs(xs), batch, img_tokens, kc, vc, pl, prefix_max,
                                      _host_ptrs(ys), _dptr(staging, None, "staging"), staging.numel(),
                                      _dptr(workspace, None, "workspace"),
                                      workspace.numel(), _stream(stream)), "mot_attn_forward_host")


def mot_attn_merge_lora(h, w_q_out, w_k_out, w_v_out, w_o_out, stream=None) -> None:
    check(lib().mot_attn_merge_lora(h, _dptr(w_q_out, _BF16, "w_q_out"), _dptr(w_k_out, _BF16, "w_k_out"),
                                    _dptr(w_v_out, _BF16, "w_v_out"), _dptr(w_o_out, _BF16, "w_o_out"),
                                    _stream(stream)), "mot_attn_merge_lora")


def mot_attn_get_device_status(h, stream=None) -> int:
    return lib().mot_attn_get_device_status(h, _stream(stream))


def mot_attn_destroy(h) -> None:
    lib().mot_attn_destroy(h)


def mot_attn_last_launch_count(h) -> int:
    return lib().mot_attn_last_launch_count(h)


def mot_status_string(status: int) -> str:
    return lib().mot_status_string(status).decode()


def mot_dev_gemm(a, b, d, tile_n=256, stream=None) -> None:
    m, k = a.shape
    n = b.shape[0]
    check(lib().mot_dev_gemm(_ptr(a), _ptr(b), _ptr(d), m, n, k, int(a.dtype == torch.bfloat16), tile_n,
                             _stream(stream)), "mot_dev_gemm")


def mot_dev_gemm_variant(a, b, d, variant, b2=None, stream=None) -> None:
    """D = A B^T (+ A B2^T for variant 3; A B with B [k, n] for variant 4)
    through the pair (1, 4), split-K (2) or dual-B split-K (3) GEMM path;
    see include/mot_attn_dev.h."""
    m, k = a.shape
    n = b.shape[1] if variant == 4 else b.shape[0]
    check(lib().mot_dev_gemm_variant(_ptr(a), _ptr(b), _ptr(b2) if b2 is not None else None, _ptr(d), m, n, k,
                                     int(a.dtype == torch.bfloat16), variant, _stream(stream)),
          "mot_dev_gemm_variant")


def mot_dev_saved_layout(cfg: MotAttnConfig, batch, img_tokens, prefix_max):
    offs = (c_size_t * 9)()
    lcap = c_int32(0)
    check(lib().mot_dev_saved_layout(byref(cfg), batch, img_tokens, prefix_max, offs, byref(lcap)),
          "mot_dev_saved_layout")
    return list(offs), lcap.value


def mot_dev_exp2_poly(x, y, stream=None) -> None:
    check(lib().mot_dev_exp2_poly(_ptr(x), _ptr(y), x.numel(), _stream(stream)), "mot_dev_exp2_poly")


def mot_dev_wait_probe(h, stream=None) -> None:
    check(lib().mot_dev_wait_probe(h, _stream(stream)), "mot_dev_wait_probe")


def mot_dev_set_attn_splits(h, splits: int) -> None:
    """0: split-KV count planned per call; 1..8: forced (tests, measurements)."""
    check(lib().mot_dev_set_attn_splits(h, int(splits)), "mot_dev_set_attn_splits")


def mot_dev_last_attn_splits(h) -> int:
    return int(lib().mot_dev_last_attn_splits(h))


def mot_dev_last_attn_full_units(h) -> int:
    return int(lib().mot_dev_last_attn_full_units(h))


def mot_dev_profile(h, enable: bool) -> None:
    check(lib().mot_dev_profile(h, int(bool(enable))), "mot_dev_profile")


def mot_dev_stage_times(h, max_stages: int = 32):
    ids = (c_int32 * max_stages)()
    ms = (ctypes.c_float * max_stages)()
    count = c_int32(0)
    check(lib().mot_dev_stage_times(h, ids, ms, max_stages, byref(count)), "mot_dev_stage_times")
    return [(lib().mot_dev_stage_name(ids[i]).decode(), ms[i]) for i in range(min(count.value, max_stages))]


def mot_dev_stage_timeline(h, max_stages: int = 32):
    """[(stage name, start ms, end ms)] of the last call's launches on one clock
    (milliseconds after the first launch's start)."""
    ids = (c_int32 * max_stages)()
    t0 = (ctypes.c_float * max_stages)()
    t1 = (ctypes.c_float * max_stages)()
    count = c_int32(0)
    check(lib().mot_dev_stage_timeline(h, ids, t0, t1, max_stages, byref(count)), "mot_dev_stage_timeline")
    return [(lib().mot_dev_stage_name(ids[i]).decode(), t0[i], t1[i]) for i in range(min(count.value, max_stages))]


class MotAttnLayer:
    """A handle plus the caller-owned buffers of one call shape."""

    def __init__(self, weights: Dict[str, torch.Tensor], lora_rank: int = 0, lora_alpha: float = 0.0,
                 max_batch: int = 1, max_img_tokens: int = 256, max_prefix: int = 0,
                 enable_backward: bool = False, hidden: int = 4096, n_q_heads: int = 32, n_kv_heads: int = 8,
                 head_dim: int = 128, rms_eps: float = 1e-6, rope_theta: float = 1e6, stream=None):
        self.cfg = make_config(hidden, n_q_heads, n_kv_heads, head_dim, lora_rank, lora_alpha, rms_eps,
                               rope_theta, max_batch, max_img_tokens, max_prefix, enable_backward)
        self.weights = dict(weights)  # keep the tensors alive
        self.handle = mot_attn_create(self.cfg, self.weights, stream)
        self._ws = None

    def sizes(self, batch, img_tokens, prefix_max):
        return mot_attn_query_sizes(self.cfg, batch, img_tokens, prefix_max)

    def workspace(self, batch, img_tokens, prefix_max, device="cuda"):
        ws, _ = self.sizes(batch, img_tokens, prefix_max)
        if self._ws is None or self._ws.numel() < ws:
            self._ws = torch.empty(ws, dtype=torch.uint8, device=device)
        return self._ws

    def new_saved(self, batch, img_tokens, prefix_max, device="cuda"):
        _, sv = self.sizes(batch, img_tokens, prefix_max)
        return torch.empty(sv, dtype=torch.uint8, device=device)

    def forward(self, x, k_cache, v_cache, prefix_len, y=None, y_f32=None, saved=None, workspace=None,
                stream=None):
        B, N, d = x.shape
        P = k_cache.shape[2] if k_cache is not None else 0
        if y is None:
            y = torch.empty_like(x)
        if workspace is None:
            workspace = self.workspace(B, N, P, x.device)
        mot_attn_forward(self.handle, x, B, N, k_cache, v_cache, prefix_len, P, y, y_f32, saved, workspace, stream)
        return y

    def prefix_forward(self, x, lengths, y=None, y_f32=None, k_cache_out=None, v_cache_out=None, workspace=None,
                       stream=None):
        """Prefix-tower layer over the prompt x [B, N, d]: returns (y, k_cache, v_cache)."""
        B, N, d = x.shape
        c = self.cfg
        if y is None:
            y = torch.empty_like(x)
        shape = (B, c.n_kv_heads, N, c.head_dim)
        if k_cache_out is None:
            k_cache_out = torch.empty(shape, dtype=torch.bfloat16, device=x.device)
        if v_cache_out is None:
            v_cache_out = torch.empty(shape, dtype=torch.bfloat16, device=x.device)
        if workspace is None:
            workspace = self.workspace(B, N, 0, x.device)
        mot_attn_prefix_forward(self.handle, x, B, N, lengths, y, k_cache_out, v_cache_out, y_f32, workspace, stream)
        return y, k_cache_out, v_cache_out

    def host_staging(self, batch, img_tokens, prefix_max, device="cuda"):
        n = mot_attn_query_host_staging(self.cfg, batch, img_tokens, prefix_max)
        return torch.empty(n, dtype=torch.uint8, device=device)

    def forward_host(self, xs, k_caches, v_caches, prefix_len, ys, staging=None, workspace=None, stream=None):
        """Inference forwards over host buffers (one x, k_cache, v_cache, y
        per call; pinned for overlap): copies in, layer and copies out are
        pipelined over two device staging slots. Asynchronous: the y buffers
        are complete once `stream` has finished the enqueued work."""
        B, N, d = xs[0].shape
        P = k_caches[0].shape[2] if k_caches is not None else 0
        if staging is None:
            staging = self.host_staging(B, N, P)
        if workspace is None:
            workspace = self.workspace(B, N, P)
        mot_attn_forward_host(self.handle, xs, B, N, k_caches, v_caches, prefix_len, P, ys, staging, workspace,
                              stream)

    def backward(self, dy, x, k_cache, v_cache, prefix_len, saved, dx=None, dx_f32=None, d_a=None, d_b=None,
                 accumulate=False, workspace=None, stream=None):
        B, N, d = x.shape
        P = k_cache.shape[2] if k_cache is not None else 0
        if dx is None:
            dx = torch.empty_like(x)
        if workspace is None:
            workspace = self.workspace(B, N, P, x.device)
        mot_attn_backward(self.handle, dy, x, B, N, k_cache, v_cache, prefix_len, P, saved, dx, dx_f32, d_a, d_b,
                          accumulate, workspace, stream)
        return dx

    def merge_lora(self, w_q_out, w_k_out, w_v_out, w_o_out, stream=None):
        mot_attn_merge_lora(self.handle, w_q_out, w_k_out, w_v_out, w_o_out, stream)
        self.weights.update(w_q=w_q_out, w_k=w_k_out, w_v=w_v_out, w_o=w_o_out)

    def device_status(self, stream=None) -> int:
        return mot_attn_get_device_status(self.handle, stream)

    def last_launch_count(self) -> int:
        return mot_attn_last_launch_count(self.handle)

    def close(self):
        if self.handle is not None:
            mot_attn_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

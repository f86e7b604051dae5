"""Seeded synthetic inputs for the gen-tower attention layer.

This module only draws random tensors; it holds none of the layer's arithmetic.
It is the one piece shared by the CUDA path's callers (tests, bench) and the
oracle's callers: both receive the very same bf16 tensors from here.

Workload shapes follow the pages' workloads (DiffSynth-Studio "SenseNova-U1"
page, quick-start and inference parameters: 2048x2048 default output, sides a
multiple of 32; same page, architecture note: prompt encoded once into
``past_key_values``; "Setup notes" page, "Why bf16 base on CPU + tower
offload?": a static prefix-KV cache of a few hundred tokens per sample).
Image tokens are 32-pixel patches, so 512^2 -> 256, 1024^2 -> 1024 and
2048^2 -> 4096 tokens. Layer dimensions (hidden 4096, 32 query / 8 KV heads,
head_dim 128) are those of the Qwen3-8B-class backbone the vLLM-Omni
"SenseNova-U1" recipe names (Summary); the pages print no dims themselves.

Distributions: hidden states, cached K/V and the upstream gradient N(0, 1);
base weights N(0, 0.02); LoRA down (A) N(0, 1/16); LoRA up (B) N(0, 0.01);
RMSNorm gains 1 + 0.1 N(0, 1). Each tensor is drawn in fp32 from its own CPU
``torch.Generator`` seeded ``1000 * config + tensor_index`` and rounded to bf16.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch

HIDDEN = 4096
N_Q_HEADS = 32
N_KV_HEADS = 8
HEAD_DIM = 128
RMS_EPS = 1e-6
ROPE_THETA = 1e6


@dataclasses.dataclass(frozen=True)
class LayerDims:
    hidden: int = HIDDEN
    n_q_heads: int = N_Q_HEADS
    n_kv_heads: int = N_KV_HEADS
    head_dim: int = HEAD_DIM
    rms_eps: float = RMS_EPS
    rope_theta: float = ROPE_THETA


@dataclasses.dataclass(frozen=True)
class Workload:
    """One layer call: B CFG branches of N image tokens over P cached keys."""
    name: str
    batch: int          # CFG branches (cond / uncond / image-uncond)
    img_tokens: int     # N = (H/32) * (W/32)
    prefix: int         # P = cached prefix keys per branch
    lora_rank: int      # r (0 = no adapters)
    lora_alpha: float
    merged: bool = False   # LoRA folded into the base weights before the call
    train: bool = False    # forward + LoRA backward
    dims: LayerDims = LayerDims()


# The five workloads: a 512^2 single-branch check, 1024^2 and 2048^2
# text-to-image CFG (cond + fixed uncond), the 2048^2 dual-CFG edit with an
# image prefix (400 text + 4096 image tokens) and merged LoRA, and the 2048^2
# LoRA training step.
WORKLOADS = {
    0: Workload("fwd_512sq_b1", 1, 256, 64, 16, 16.0),
    1: Workload("fwd_1024sq_cfg2", 2, 1024, 400, 32, 32.0),
    2: Workload("fwd_2048sq_cfg2", 2, 4096, 400, 32, 32.0),
    3: Workload("fwd_2048sq_edit_cfg3_merged", 3, 4096, 4496, 32, 32.0, merged=True),
    4: Workload("train_2048sq_b1", 1, 4096, 400, 32, 32.0, train=True),
}

# tensor_index of each named tensor (seed = 1000 * config + tensor_index)
_TENSOR_INDEX = {
    "x": 0, "w_q": 1, "w_k": 2, "w_v": 3, "w_o": 4, "q_norm": 5, "k_norm": 6,
    "a_q": 7, "a_k": 8, "a_v": 9, "a_o": 10, "b_q": 11, "b_k": 12, "b_v": 13,
    "b_o": 14, "k_cache": 15, "v_cache": 16, "dy": 17,
}


def _draw(shape, std: float, mean: float, seed: int) -> torch.Tensor:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    t = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    if mean != 0.0:
        t.add_(mean)
    return t.to(torch.bfloat16)


# data tensors of data-parallel shard k draw from seed + k * SHARD_STRIDE
SHARD_STRIDE = 100_000
_DATA = ("x", "k_cache", "v_cache", "dy")


def make_inputs(wl: Workload, seed_base: int, with_dy: Optional[bool] = None,
                shard: int = 0) -> Dict[str, torch.Tensor]:
    """Return CPU bf16 tensors for one layer call plus ``prefix_len`` (int32).

    Shapes: x, dy [B, N, hidden]; w_q [Hq*dh, hidden]; w_k, w_v [Hkv*dh, hidden];
    w_o [hidden, Hq*dh]; q_norm, k_norm [dh]; a_* [r, in]; b_* [out, r];
    k_cache, v_cache [B, Hkv, P, dh] (keys already normalised and rotated).
    ``shard`` selects a data-parallel shard: the weights are the same for
    every shard (replicas), x, the cache and dy are drawn independently;
    shard 0 is the unsharded call.
    """
    d = wl.dims
    B, N, P, r = wl.batch, wl.img_tokens, wl.prefix, wl.lora_rank
    qd, kvd = d.n_q_heads * d.head_dim, d.n_kv_heads * d.head_dim
    s = lambda name: seed_base + _TENSOR_INDEX[name] + (shard * SHARD_STRIDE if name in _DATA else 0)
    out = {
        "x": _draw((B, N, d.hidden), 1.0, 0.0, s("x")),
        "w_q": _draw((qd, d.hidden), 0.02, 0.0, s("w_q")),
        "w_k": _draw((kvd, d.hidden), 0.02, 0.0, s("w_k")),
        "w_v": _draw((kvd, d.hidden), 0.02, 0.0, s("w_v")),
        "w_o": _draw((d.hidden, qd), 0.02, 0.0, s("w_o")),
        "q_norm": _draw((d.head_dim,), 0.1, 1.0, s("q_norm")),
        "k_norm": _draw((d.head_dim,), 0.1, 1.0, s("k_norm")),
        "k_cache": _draw((B, d.n_kv_heads, P, d.head_dim), 1.0, 0.0, s("k_cache")),
        "v_cache": _draw((B, d.n_kv_heads, P, d.head_dim), 1.0, 0.0, s("v_cache")),
    }
    if r > 0:
        for name, (rows, cols) in {
            "a_q": (r, d.hidden), "a_k": (r, d.hidden), "a_v": (r, d.hidden), "a_o": (r, qd),
            "b_q": (qd, r), "b_k": (kvd, r), "b_v": (kvd, r), "b_o": (d.hidden, r),
        }.items():
            std = 1.0 / 16.0 if name.startswith("a_") else 0.01
            out[name] = _draw((rows, cols), std, 0.0, s(name))
    if wl.train if with_dy is None else with_dy:
        out["dy"] = _draw((B, N, d.hidden), 1.0, 0.0, s("dy"))
    out["prefix_len"] = torch.full((B,), P, dtype=torch.int32)
    return out


# the gen-tower MLP's tensors (the next block of the same decoder layer);
# indices apart from the attention layer's
_MLP_TENSOR_INDEX = {
    "x": 40, "w_gate": 41, "w_up": 42, "w_down": 43, "a_gate": 44, "a_up": 45, "a_down": 46,
    "b_gate": 47, "b_up": 48, "b_down": 49, "dy": 50,
}


def make_mlp_inputs(tokens: int, hidden: int, inter: int, lora_rank: int, seed_base: int,
                    with_dy: bool = False) -> Dict[str, torch.Tensor]:
    """CPU bf16 tensors for one gen-tower SwiGLU MLP call, with the same
    distributions as the attention layer's: x, dy [tokens, hidden];
    w_gate, w_up [inter, hidden]; w_down [hidden, inter]; a_gate, a_up
    [r, hidden]; a_down [r, inter]; b_gate, b_up [inter, r]; b_down [hidden, r]."""
    s = lambda name: seed_base + _MLP_TENSOR_INDEX[name]
    r = lora_rank
    out = {
        "x": _draw((tokens, hidden), 1.0, 0.0, s("x")),
        "w_gate": _draw((inter, hidden), 0.02, 0.0, s("w_gate")),
        "w_up": _draw((inter, hidden), 0.02, 0.0, s("w_up")),
        "w_down": _draw((hidden, inter), 0.02, 0.0, s("w_down")),
    }
    if r > 0:
        for name, shape in {"a_gate": (r, hidden), "a_up": (r, hidden), "a_down": (r, inter),
                            "b_gate": (inter, r), "b_up": (inter, r), "b_down": (hidden, r)}.items():
            out[name] = _draw(shape, 1.0 / 16.0 if name.startswith("a_") else 0.01, 0.0, s(name))
    if with_dy:
        out["dy"] = _draw((tokens, hidden), 1.0, 0.0, s("dy"))
    return out


# MLP workloads: the same calls as the attention workloads (tokens = all CFG
# branches' image tokens), intermediate width 12288 (3 x hidden; the pages
# give no dense width), the same LoRA ranks
MLP_INTER = 3 * HIDDEN


@dataclasses.dataclass(frozen=True)
class MlpWorkload:
    name: str
    tokens: int
    lora_rank: int
    lora_alpha: float
    train: bool = False
    hidden: int = HIDDEN
    inter: int = MLP_INTER


MLP_WORKLOADS = {
    0: MlpWorkload("mlp_512sq_b1", 256, 16, 16.0),
    1: MlpWorkload("mlp_1024sq_cfg2", 2048, 32, 32.0),
    2: MlpWorkload("mlp_2048sq_cfg2", 8192, 32, 32.0),
    4: MlpWorkload("mlp_train_2048sq_b1", 4096, 32, 32.0, train=True),
}


def mlp_workload_inputs(index: int, with_dy: Optional[bool] = None) -> Dict[str, torch.Tensor]:
    wl = MLP_WORKLOADS[index]
    return make_mlp_inputs(wl.tokens, wl.hidden, wl.inter, wl.lora_rank, 1000 * index,
                           wl.train if with_dy is None else with_dy)


# the denoise step's own tensors (patch embedding, norms, head) and the
# noisy image; indices apart from the layers' tensors
_STEP_TENSOR_INDEX = {"w_in": 60, "norm_out": 61, "w_out": 62, "z": 63, "norm_in": 64, "norm_post": 65}


def make_step_inputs(n_layers: int, wl: Workload, inter: int, patch_dim: int, seed_base: int):
    """CPU tensors for one denoise step over ``n_layers`` gen-tower layers:
    per layer the attention layer's tensors (``make_inputs``, seed
    seed_base + 100 l) with its prefix cache, the MLP's (``make_mlp_inputs``)
    and the two norm gains (1 + 0.1 N(0, 1)); the tower's w_in [d, C] and
    w_out [C, d] (N(0, 0.02)), norm_out; the image's patch tokens z [N, C]
    (f32, N(0, 1))."""
    d = wl.dims.hidden
    s = lambda name, l=0: seed_base + _STEP_TENSOR_INDEX[name] + 100 * l
    layers = []
    for l in range(n_layers):
        t = make_inputs(wl, seed_base + 100 * l, with_dy=False)
        m = make_mlp_inputs(wl.batch * wl.img_tokens, d, inter, wl.lora_rank, seed_base + 100 * l + 50)
        t.update({"mlp_" + k: v for k, v in m.items() if k != "x"})
        t["norm_in"] = _draw((d,), 0.1, 1.0, s("norm_in", l))
        t["norm_post"] = _draw((d,), 0.1, 1.0, s("norm_post", l))
        layers.append(t)
    g = torch.Generator(device="cpu")
    g.manual_seed(s("z"))
    return {"layers": layers, "w_in": _draw((d, patch_dim), 0.02, 0.0, s("w_in")),
            "norm_out": _draw((d,), 0.1, 1.0, s("norm_out")), "w_out": _draw((patch_dim, d), 0.02, 0.0, s("w_out")),
            "z": torch.randn(wl.img_tokens, patch_dim, generator=g, dtype=torch.float32)}


# the A3B gen tower's mixture-of-experts MLP: hidden 2048, 32 experts, top-8,
# expert width 768 ("SenseNova-U1" vLLM-Omni recipe, A3B variant)
MOE_HIDDEN, MOE_EXPERTS, MOE_TOP_K, MOE_INTER = 2048, 32, 8, 768
_MOE_TENSOR_INDEX = {"x": 80, "w_router": 81, "w_gate": 82, "w_up": 83, "w_down": 84}


def make_moe_inputs(tokens: int, hidden: int, inter: int, experts: int, seed_base: int) -> Dict[str, torch.Tensor]:
    """CPU bf16 tensors for one MoE MLP call: x [tokens, hidden] N(0, 1);
    w_router [E, hidden], w_gate, w_up [E, inter, hidden], w_down [E, hidden,
    inter], all N(0, 0.02) (the attention layer's weight recipe)."""
    s = lambda name: seed_base + _MOE_TENSOR_INDEX[name]
    return {"x": _draw((tokens, hidden), 1.0, 0.0, s("x")),
            "w_router": _draw((experts, hidden), 0.02, 0.0, s("w_router")),
            "w_gate": _draw((experts, inter, hidden), 0.02, 0.0, s("w_gate")),
            "w_up": _draw((experts, inter, hidden), 0.02, 0.0, s("w_up")),
            "w_down": _draw((experts, hidden, inter), 0.02, 0.0, s("w_down"))}


def draw_device(shape, std: float, mean: float, seed: int, device) -> torch.Tensor:
    """bf16 N(mean, std^2) drawn on the device from a seeded generator of that
    device (the large multi-layer benchmark stacks; the oracle never sees these)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    t = torch.randn(*shape, generator=g, dtype=torch.float32, device=device)
    if std != 1.0:
        t.mul_(std)
    if mean != 0.0:
        t.add_(mean)
    return t.to(torch.bfloat16)


def workload_inputs(index: int, with_dy: Optional[bool] = None, shard: int = 0) -> Dict[str, torch.Tensor]:
    return make_inputs(WORKLOADS[index], 1000 * index, with_dy, shard)


def tiny_workload(batch=2, img_tokens=5, prefix=3, lora_rank=2, lora_alpha=4.0, hidden=64,
                  n_q_heads=4, n_kv_heads=2, head_dim=16, train=True) -> Workload:
    """Small shapes for oracle checks (finite differences, brute force)."""
    dims = LayerDims(hidden=hidden, n_q_heads=n_q_heads, n_kv_heads=n_kv_heads, head_dim=head_dim)
    return Workload("tiny", batch, img_tokens, prefix, lora_rank, lora_alpha, train=train, dims=dims)

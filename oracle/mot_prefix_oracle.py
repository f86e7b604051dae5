"""Oracle for the prefix-tower attention layer that builds the prefix-KV cache
-- TEST INFRASTRUCTURE ONLY.

A plain, slow, fp64 CPU statement of one prefix-tower (understanding branch,
``*_mot`` modules) attention layer over the prompt tokens: it produces the
layer's output and the cache entry the gen tower's layer attends to. Like the
other oracles it is imported only by ``tests/`` and ``bench.py``'s CPU arm;
the library never imports it and shares no code with it.

What it is (sources, by page title and section):
  * "SenseNova-U1" (DiffSynth-Studio docs), architecture note: the prompt is
    encoded once by the understanding branch into ``past_key_values``; the
    image tokens of every denoise step attend to that cache.
  * "Setup notes" (LoRA trainer docs), "Why bf16 base on CPU + tower
    offload?": the prefix tower computes the static prefix-KV cache once, in
    bf16; the LoRA adapters sit on the gen tower only.
  * "SenseNova-U1" (vLLM-Omni recipe), Summary: a Qwen3-based LLM, whose
    self-attention over text is causal.

Readings where the pages are silent:
  P1 the prefix tower's attention layer has the gen tower's structure
     (q/k/v/o projections without bias, per-head QK-RMSNorm with its own
     gains, rotate-half RoPE; readings R2-R4 of the attention oracle) with
     the understanding weights and no adapters.
  P2 causal: prompt token i of branch b attends to tokens j <= i with
     j < len_b (len_b <= P, the rest of the P rows is padding).
  P3 positions 0 .. len_b - 1; the gen tower's image tokens continue at
     len_b (reading R3 of the attention oracle).
  P4 the cache entry of the layer for branch b is the normalised, rotated
     keys and the values of its len_b prompt tokens, stored in bf16 (rows
     at or beyond len_b are padding, never read).
"""
from __future__ import annotations

import math
from typing import Dict, Sequence

import numpy as np

from oracle.mot_attn_oracle import lora_linear, rms_norm_heads, rope_rotate, round_to_bf16


def causal_gqa_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, length: int):
    """Causal grouped-query attention over the first ``length`` tokens (P2).

    q [Hq, n, dh], k, v [Hkv, n, dh]. Query i (i < length) attends to keys
    j <= i; query rows at or beyond ``length`` attend to all ``length`` keys
    (their output is padding). Returns (o [Hq, n, dh], lse [Hq, n]).
    """
    hq, hkv, dh = q.shape[0], k.shape[0], q.shape[-1]
    n = q.shape[1]
    group = hq // hkv
    scale = 1.0 / math.sqrt(dh)
    i = np.arange(n)[:, None]
    j = np.arange(k.shape[1])[None, :]
    allowed = (j <= np.minimum(i, length - 1)) & (j < length)
    o = np.empty(q.shape, dtype=np.float64)
    lse = np.empty((hq, n), dtype=np.float64)
    for h in range(hq):
        s = (q[h] @ k[h // group].T) * scale
        s = np.where(allowed, s, -np.inf)
        m = s.max(axis=-1, keepdims=True)
        e = np.exp(s - m)
        den = e.sum(axis=-1, keepdims=True)
        o[h] = (e / den) @ v[h // group]
        lse[h] = (m + np.log(den))[:, 0]
    return o, lse


def prefix_forward(inp: Dict[str, np.ndarray], dims: Dict, lengths: Sequence[int]) -> Dict:
    """One prefix-tower attention layer over B branches of P prompt tokens.

    inp: x [B, P, d]; w_q, w_k, w_v, w_o; q_norm, k_norm (the understanding
    weights). Returns y [B, P, d] and the cache entry k_cache, v_cache
    [B, Hkv, P, dh] in fp64 (normalised + rotated keys, values), before the
    bf16 rounding of P4 (``cache_bf16`` applies it).
    """
    hq, hkv, dh = dims["n_q_heads"], dims["n_kv_heads"], dims["head_dim"]
    eps, theta = dims["rms_eps"], dims["rope_theta"]
    x = inp["x"]
    nb, n, _ = x.shape
    ys, ks, vs = [], [], []
    pos = np.arange(n)
    for b in range(nb):
        q = lora_linear(x[b], inp["w_q"], None, None, 0.0).reshape(n, hq, dh).transpose(1, 0, 2)
        k = lora_linear(x[b], inp["w_k"], None, None, 0.0).reshape(n, hkv, dh).transpose(1, 0, 2)
        v = lora_linear(x[b], inp["w_v"], None, None, 0.0).reshape(n, hkv, dh).transpose(1, 0, 2)
        q = rope_rotate(rms_norm_heads(q, inp["q_norm"], eps)[0], pos, theta)
        k = rope_rotate(rms_norm_heads(k, inp["k_norm"], eps)[0], pos, theta)
        o, _ = causal_gqa_attention(q, k, v, int(lengths[b]))
        ys.append(lora_linear(o.transpose(1, 0, 2).reshape(n, hq * dh), inp["w_o"], None, None, 0.0))
        ks.append(k)
        vs.append(v)
    return {"y": np.stack(ys), "k_cache": np.stack(ks), "v_cache": np.stack(vs)}


def cache_bf16(c: np.ndarray) -> np.ndarray:
    """The cache as stored (P4): one round to nearest bf16."""
    return round_to_bf16(c)

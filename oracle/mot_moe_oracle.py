"""Oracle for the A3B gen-tower mixture-of-experts MLP block -- TEST
INFRASTRUCTURE ONLY.

A plain, slow, fp64 CPU statement of the sparse MLP that replaces the dense
SwiGLU MLP in the A3B variant's generation tower. Imported only by
``tests/`` (and ``bench.py``'s CPU arm); the library never imports it and
shares no code with it.

What it is (sources, by page title and section):
  * "SenseNova-U1" (vLLM-Omni recipe), A3B (MoE) variant: a Qwen3-MoE
    backbone; the generation branch ``mlp_mot_gen`` routes over 32 experts,
    top-8, per-expert width ``moe_intermediate_size`` = 768.
  * the same page, measured kernel table: ``fused_moe_kernel`` (the top-8
    expert GEMMs on the 32-expert generation tower), MoE routing (top-k),
    ``act_and_mul`` (SwiGLU).
  * the same page, memory table: 7.25 B generation-path expert parameters
    for 32 experts per layer.

Readings where the pages are silent:
  E1 router: logits = x W_r^T (no bias), p = softmax over the E experts,
     the top_k experts by p (ties to the lower expert index), their weights
     p renormalised to sum to one (the Qwen3-MoE top-k convention).
  E2 every expert is the SwiGLU MLP of reading M1 without adapters:
     e(x) = (silu(x Wg_e^T) * (x Wu_e^T)) Wd_e^T.
  E3 y = sum over the rank k = 0 .. top_k - 1 of w_k e_{i_k}(x).
  E4 hidden width 2048: 7.25 B expert parameters = layers x 32 experts x
     3 x 768 x hidden fits 48 layers of hidden 2048 (the Qwen3-30B-A3B
     class); x is the already-normalised hidden state, y the block output
     (no residual).
"""
from __future__ import annotations

from typing import Dict

import numpy as np

from oracle.mot_mlp_oracle import mlp_forward


def route(x: np.ndarray, w_router: np.ndarray, top_k: int):
    """E1: returns (experts [T, top_k] int, weights [T, top_k], probs [T, E])."""
    logits = x @ w_router.T
    m = logits.max(axis=-1, keepdims=True)
    e = np.exp(logits - m)
    p = e / e.sum(axis=-1, keepdims=True)
    # stable sort on -p: equal probabilities keep the lower expert first
    order = np.argsort(-p, axis=-1, kind="stable")[:, :top_k]
    w = np.take_along_axis(p, order, axis=-1)
    return order, w / w.sum(axis=-1, keepdims=True), p


def expert_forward(x: np.ndarray, w: Dict[str, np.ndarray], e: int) -> np.ndarray:
    """E2 for expert e of the stacked weights w_gate, w_up [E, I, d], w_down [E, d, I]."""
    return mlp_forward(x, {"w_gate": w["w_gate"][e], "w_up": w["w_up"][e], "w_down": w["w_down"][e]}, 0.0)["y"]


def moe_forward(x: np.ndarray, w: Dict[str, np.ndarray], top_k: int) -> Dict[str, np.ndarray]:
    """The block for tokens x [T, d]: w_router [E, d], w_gate, w_up [E, I, d],
    w_down [E, d, I]. Returns y [T, d] and the routing (E1)."""
    experts, weights, probs = route(x, w["w_router"], top_k)
    y = np.zeros_like(x)
    for k in range(top_k):
        for e in np.unique(experts[:, k]):
            rows = np.nonzero(experts[:, k] == e)[0]
            y[rows] += weights[rows, k][:, None] * expert_forward(x[rows], w, int(e))
    return {"y": y, "experts": experts, "weights": weights, "probs": probs}

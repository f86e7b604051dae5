"""Oracle for the gen-tower SwiGLU MLP with LoRA -- TEST INFRASTRUCTURE ONLY.

A plain, slow, fp64 CPU statement of the MLP half of a generation-tower
decoder layer. Like the attention oracle it is imported only by ``tests/``
(and, once the MLP has kernels, by ``smoke()`` and ``bench.py``'s CPU arms);
the library never imports it and shares no code with it. Matrix products use
numpy's ``@`` as a library primitive.

What the block is (sources, by page title and section):
  * "SenseNova-U1" (DiffSynth-Studio docs), training section: the LoRA
    targets of the generation branch are the attention projections and
    ``mlp_mot_gen.gate_proj``, ``mlp_mot_gen.up_proj`` and
    ``mlp_mot_gen.down_proj`` (the ``_mot_gen`` suffix keeps the
    understanding branch's ``mlp.*`` untouched).
  * "SenseNova-U1" (vLLM-Omni recipe), measured kernel table: an
    ``act_and_mul`` (SwiGLU) element-wise kernel sits between the fused
    gate/up projection and ``down_proj``.

Readings where the pages are silent:
  M1 SwiGLU: h = silu(g) * u with silu(z) = z / (1 + exp(-z)); the gate is
     the activated half (the ``act_and_mul`` convention: first half through
     the activation, times the second half).
  M2 LoRA on each of gate, up and down as in the attention layer:
     y = x W^T + s (x A^T) B^T, s = lora_alpha / lora_rank, no dropout, no
     bias.
  M3 boundary: x is the already-normalised hidden state entering the MLP;
     y is the down_proj output (no residual add).
  M4 backward: base weights frozen; gradients of x and of every A, B.
  M5 sizes: the pages give no dense intermediate width; workloads use the
     dense 8B-class width 12288 (3 x hidden) as a stated choice.
"""
from __future__ import annotations

from typing import Dict

import numpy as np

from oracle.mot_attn_oracle import lora_linear

MLP_PROJ = ("gate", "up", "down")


def silu(z: np.ndarray) -> np.ndarray:
    """silu(z) = z * sigmoid(z) (M1), written with the sigmoid of |z| so that
    exp never overflows."""
    z = np.asarray(z, dtype=np.float64)
    e = np.exp(-np.abs(z))
    sig = np.where(z >= 0, 1.0 / (1.0 + e), e / (1.0 + e))
    return z * sig


def silu_grad(z: np.ndarray) -> np.ndarray:
    """d silu / dz = sigmoid(z) (1 + z (1 - sigmoid(z)))."""
    z = np.asarray(z, dtype=np.float64)
    e = np.exp(-np.abs(z))
    sig = np.where(z >= 0, 1.0 / (1.0 + e), e / (1.0 + e))
    return sig * (1.0 + z * (1.0 - sig))


def _lora(w: Dict[str, np.ndarray], name: str):
    a = w.get("a_" + name)
    b = w.get("b_" + name)
    if a is None or a.shape[0] == 0:
        return None, None
    return a, b


def mlp_forward(x: np.ndarray, w: Dict[str, np.ndarray], lora_scale: float) -> Dict[str, np.ndarray]:
    """Forward of the SwiGLU MLP with LoRA (M1-M3).

    x: [..., d]. w: w_gate, w_up [I, d], w_down [d, I]; optional a_gate,
    a_up [r, d], b_gate, b_up [I, r], a_down [r, I], b_down [d, r].
    Returns the pre-activations g, u, the product h = silu(g) * u and y.
    """
    s = lora_scale
    g = lora_linear(x, w["w_gate"], *_lora(w, "gate"), s)
    u = lora_linear(x, w["w_up"], *_lora(w, "up"), s)
    h = silu(g) * u
    y = lora_linear(h, w["w_down"], *_lora(w, "down"), s)
    return {"g": g, "u": u, "h": h, "y": y}


def mlp_backward(x: np.ndarray, w: Dict[str, np.ndarray], lora_scale: float,
                 dy: np.ndarray) -> Dict[str, np.ndarray]:
    """LoRA-training backward of the MLP (M4) for x, dy of shape [T, d].

    Returns dx [T, d] and dA_*, dB_* for gate, up and down (when LoRA is on).
    For a LoRA linear y = x W^T + s (x A^T) B^T with upstream dy:
      dx = dy W + s (dy B) A,   dA = s (dy B)^T x,   dB = s dy^T (x A^T).
    """
    s = lora_scale
    f = mlp_forward(x, w, s)
    grads: Dict[str, np.ndarray] = {}

    def back(name, inp, dout):
        a, b = _lora(w, name)
        din = dout @ w["w_" + name]
        if a is not None:
            g_in = dout @ b
            grads["dA_" + name] = s * (g_in.T @ inp)
            grads["dB_" + name] = s * (dout.T @ (inp @ a.T))
            din = din + s * (g_in @ a)
        return din

    dh = back("down", f["h"], dy)
    dg = dh * f["u"] * silu_grad(f["g"])
    du = dh * silu(f["g"])
    grads["dx"] = back("gate", x, dg) + back("up", x, du)
    return grads

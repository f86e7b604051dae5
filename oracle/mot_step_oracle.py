"""Oracle for one gen-tower flow-matching denoise step -- TEST INFRASTRUCTURE ONLY.

A plain, slow, fp64 CPU statement of one Euler step of the generation tower
over the image tokens of a CFG batch: patch embedding, the stack of decoder
layers (the attention half of oracle/mot_attn_oracle.py and the MLP half of
oracle/mot_mlp_oracle.py, each behind a pre-norm residual), the flow head,
the guidance combine and the Euler update. Imported only by ``tests/``; the
library never imports it and shares no code with it.

What the pages give (by page title and section):
  * "SenseNova-U1" (DiffSynth-Studio docs), inference parameters: 50 steps,
    cfg_scale 4.0 with a fixed unconditional branch, shift 3.0 ("affects the
    sigma computation"), 2048^2 images in 32-pixel patches, no VAE (pixel
    space).
  * "SenseNova-U1" (vLLM-Omni recipe), measured case: 50 Euler steps,
    cfg_norm none, timestep_shift 3.0, t_eps 0.02; image editing uses dual
    CFG with img_cfg_scale over three branches (cond, image-cond, uncond).
  * "Setup notes" (LoRA trainer docs), default training config: x0 loss, a
    timestep/noise embedder, an fm_head.

Readings where the pages give no formula:
  S1 decoder layer (the Qwen3 pre-norm layer): h <- h + Attn(RMSNorm(h) g_in),
     h <- h + MLP(RMSNorm(h) g_post); RMSNorm over the hidden width.
  S2 the image enters as 32-px patch tokens z [N, C] (C = 3 * 32 * 32);
     h0 = z W_in^T + e(sigma), e = sinusoidal embedding of 1000 sigma
     (cos then sin, frequencies 10000^(-k/(d/2))) for the pages'
     "timestep/noise embedder", whose form they do not give.
  S3 the flow head predicts x0 (the training config's x0 loss):
     x0 = (RMSNorm(h) g_out) W_out^T.
  S4 guidance on the head output, cfg_norm none: two branches (cond,
     uncond): x0 = x0_u + cfg (x0_c - x0_u); three (cond, image-cond,
     uncond): x0 = x0_u + img_cfg (x0_i - x0_u) + cfg (x0_c - x0_i); one
     branch: x0 = x0_c.
  S5 Euler on the straight flow z_s = (1 - s) x0 + s noise: velocity
     v = (z - x0) / max(sigma, t_eps), z <- z + (sigma_next - sigma) v
     (t_eps keeps the division away from sigma = 0).
  S6 shifted schedule: sigma_i = shift u_i / (1 + (shift - 1) u_i),
     u_i = 1 - i / steps, i = 0..steps.
  S7 bf16 exchange points: the tower is a bf16 model (bf16 weights, bf16
     GEMM operands), so every GEMM input that the step forms itself is one
     round-to-nearest-even bf16 value: the patch tokens entering the
     embedding, RMSNorm(h) g entering each attention and MLP half, and the
     normed state entering the head. The residual stream h and the Euler
     update stay in full precision (z there is the unrounded input).
"""
from __future__ import annotations

from typing import Dict, Sequence

import numpy as np

from oracle.mot_attn_oracle import layer_forward, round_to_bf16
from oracle.mot_mlp_oracle import mlp_forward


def rms_norm_rows(h: np.ndarray, gain: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis with a gain (S1)."""
    return h / np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + eps) * gain


def timestep_embedding(sigma: float, dim: int) -> np.ndarray:
    """e(sigma) of S2: [cos(1000 sigma f_k), sin(1000 sigma f_k)], k < dim/2."""
    k = np.arange(dim // 2, dtype=np.float64)
    ang = 1000.0 * sigma * 10000.0 ** (-k / (dim // 2))
    return np.concatenate([np.cos(ang), np.sin(ang)])


def sigma_schedule(steps: int, shift: float) -> np.ndarray:
    """sigma_0 = 1 > ... > sigma_steps = 0 (S6)."""
    u = 1.0 - np.arange(steps + 1, dtype=np.float64) / steps
    return shift * u / (1.0 + (shift - 1.0) * u)


def guidance(x0: np.ndarray, cfg: float, img_cfg: float) -> np.ndarray:
    """Combine the branches' head outputs x0 [B, ...] (S4)."""
    if x0.shape[0] == 1:
        return x0[0]
    if x0.shape[0] == 2:
        return x0[1] + cfg * (x0[0] - x0[1])
    return x0[2] + img_cfg * (x0[1] - x0[2]) + cfg * (x0[0] - x0[1])


def euler_update(z: np.ndarray, x0: np.ndarray, sigma: float, sigma_next: float, t_eps: float) -> np.ndarray:
    """One Euler step of S5."""
    v = (z - x0) / max(sigma, t_eps)
    return z + (sigma_next - sigma) * v


def denoise_step(z: np.ndarray, model: Dict, layers: Sequence[Dict], caches: Sequence[Dict],
                 prefix_len: Sequence[int], attn_dims: Dict, lora_scale: float, sigma: float,
                 sigma_next: float, cfg: float, img_cfg: float, t_eps: float, eps: float = 1e-6) -> Dict:
    """One denoise step for the B branches of one image.

    z [N, C]: the image's patch tokens at sigma. model: w_in [d, C], norm_out
    [d], w_out [C, d]. layers[l]: the attention weights (w_q .. w_o, q_norm,
    k_norm, optional a_*/b_*), the MLP weights (w_gate, w_up, w_down,
    optional a_gate .. b_down) and norm_in, norm_post [d]. caches[l]: k_cache,
    v_cache [B, Hkv, P, dh]. Returns z_next [N, C] and the per-branch x0.
    """
    nb = len(prefix_len)
    h0 = round_to_bf16(z) @ model["w_in"].T + timestep_embedding(sigma, model["w_in"].shape[0])  # S2, S7
    h = np.repeat(h0[None], nb, axis=0)
    for lw, cache in zip(layers, caches):
        attn_in = dict(lw)
        attn_in["x"] = round_to_bf16(rms_norm_rows(h, lw["norm_in"], eps))  # S1, S7
        attn_in["k_cache"], attn_in["v_cache"] = cache["k_cache"], cache["v_cache"]
        attn_in["prefix_len"] = np.asarray(prefix_len)
        h = h + layer_forward(attn_in, attn_dims, lora_scale)["y"]
        mw = {k[4:]: v for k, v in lw.items() if k.startswith("mlp_")}
        h = h + np.stack([mlp_forward(round_to_bf16(rms_norm_rows(h[b], lw["norm_post"], eps)), mw,
                                      lora_scale)["y"] for b in range(nb)])
    x0 = round_to_bf16(rms_norm_rows(h, model["norm_out"], eps)) @ model["w_out"].T  # S3, S7
    xg = guidance(x0, cfg, img_cfg)
    return {"z_next": euler_update(z, xg, sigma, sigma_next, t_eps), "x0": x0, "h": h}

"""Oracle for the gen-tower attention layer -- TEST INFRASTRUCTURE ONLY.

A plain, slow, fp64 CPU statement of what the layer computes. Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline and reference
arms) may import it; the library never does, and the library shares no code
with it. Matrix products use numpy's ``@`` as a library primitive; nothing is
blocked, fused or reordered beyond the definitions below.

What the layer is (sources, by page title and section):
  * "SenseNova-U1" (DiffSynth-Studio docs), architecture note: every decoder
    layer holds an understanding and a generation weight set; the prompt is
    encoded once by the understanding branch into ``past_key_values``, and at
    every denoise step the image tokens go through the generation branch and
    attend to that cache.
  * "Setup notes" (LoRA trainer docs), "Why bf16 base on CPU + tower offload?":
    prefix tower (``*_mot``) vs gen tower (``*_mot_gen``, LoRA-wrapped); a
    static prefix-KV cache computed once.
  * "SenseNova-U1" (DiffSynth-Studio docs), training section: LoRA targets
    ``q_proj_mot_gen, k_proj_mot_gen, v_proj_mot_gen, o_proj_mot_gen``.
  * "SenseNova-U1" (vLLM-Omni recipe), measured kernel table: attention runs in
    FlashAttention, q/k use a fused "RMSNorm + RoPE" kernel; the backbone is
    Qwen3-based (Summary).

Readings where the pages are silent (each stated where it is used):
  R1 LoRA: y = x W^T + s (x A^T) B^T with s = alpha / r, added before the
     q/k norm, no dropout, no bias anywhere.
  R2 QK-RMSNorm: per head over head_dim, gain after normalisation, frozen.
  R3 RoPE: rotate-half pairs (j, j + dh/2), inv_j = theta^(-2j/dh), angles in
     fp64; cached keys are already normalised and rotated; image token i of
     branch b sits at position prefix_len[b] + i.
  R4 GQA: query head h reads KV head floor(h / (Hq/Hkv)); scale 1/sqrt(dh);
     non-causal; cache rows at or beyond prefix_len[b] are excluded.
  R5 layer boundary: x is the already-normalised hidden state; y is the
     o_proj output (no residual).
  R6 backward: base weights, norm gains and the cache are frozen.
  R7 merge: W' = RNE_bf16(W + s B A) with one rounding.
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence

import numpy as np


# --------------------------------------------------------------------------
# rounding (used by the merge, R7)
# --------------------------------------------------------------------------
def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bfloat16, ties to even, in one step.

    bfloat16 keeps 8 significant bits. With x = m * 2^e (0.5 <= |m| < 1),
    the nearest value is rint(m * 2^8) * 2^(e - 8); ``np.rint`` rounds half to
    even. Normal range only (the weights involved are far from under/overflow).
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


# --------------------------------------------------------------------------
# building blocks
# --------------------------------------------------------------------------
def lora_linear(x: np.ndarray, w: np.ndarray, a: Optional[np.ndarray], b: Optional[np.ndarray],
                scale: float) -> np.ndarray:
    """y = x W^T + s (x A^T) B^T  (R1; LoRA naming lora_down = A [r, in], lora_up = B [out, r])."""
    y = x @ w.T
    if a is not None and a.shape[0] > 0:
        y = y + scale * ((x @ a.T) @ b.T)
    return y


def rms_norm_heads(x: np.ndarray, gain: np.ndarray, eps: float):
    """Per-head RMSNorm over the last axis (R2).

    Returns (y, xhat, rstd) with rstd = 1/sqrt(mean(x^2) + eps), xhat = x * rstd
    and y = xhat * gain.
    """
    rstd = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    xhat = x * rstd
    return xhat * gain, xhat, rstd


def rms_norm_heads_backward(dy: np.ndarray, xhat: np.ndarray, rstd: np.ndarray, gain: np.ndarray):
    """Gradient of rms_norm_heads w.r.t. x with the gain frozen (R6).

    With g = gain * dy: dx = rstd * (g - xhat * mean(g * xhat)).
    """
    g = dy * gain
    return rstd * (g - xhat * np.mean(g * xhat, axis=-1, keepdims=True))


def rope_angles(positions: np.ndarray, head_dim: int, theta: float) -> np.ndarray:
    """phi[p, j] = position_p * theta^(-2j/dh), j < dh/2, in fp64 (R3)."""
    j = np.arange(head_dim // 2, dtype=np.float64)
    inv = theta ** (-2.0 * j / head_dim)
    return np.asarray(positions, dtype=np.float64)[:, None] * inv[None, :]


def rope_rotate(x: np.ndarray, positions: np.ndarray, theta: float, inverse: bool = False) -> np.ndarray:
    """Rotate-half RoPE on the last axis of x [..., n, dh] at the n positions (R3).

    Pair (x_j, x_{j+dh/2}) -> (x_j cos phi - x_{j+dh/2} sin phi,
                               x_{j+dh/2} cos phi + x_j sin phi).
    ``inverse`` rotates by -phi (the transpose, used by the backward).
    """
    dh = x.shape[-1]
    half = dh // 2
    phi = rope_angles(positions, dh, theta)
    c, s = np.cos(phi), np.sin(phi)
    if inverse:
        s = -s
    lo, hi = x[..., :half], x[..., half:]
    return np.concatenate([lo * c - hi * s, hi * c + lo * s], axis=-1)


def gqa_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray):
    """Softmax attention, grouped-query, non-causal (R4).

    q [Hq, n, dh]; k, v [Hkv, L, dh]. Query head h reads KV head h // (Hq/Hkv).
    Returns (o [Hq, n, dh], probs [Hq, n, L], lse [Hq, n]) with
    lse = log sum_j exp(s_j) in natural log.
    """
    hq, hkv, dh = q.shape[0], k.shape[0], q.shape[-1]
    group = hq // hkv
    scale = 1.0 / math.sqrt(dh)
    o = np.empty(q.shape, dtype=np.float64)
    probs = np.empty((hq, q.shape[1], k.shape[1]), dtype=np.float64)
    lse = np.empty((hq, q.shape[1]), dtype=np.float64)
    for h in range(hq):
        g = h // group
        s = (q[h] @ k[g].T) * scale
        m = s.max(axis=-1, keepdims=True)
        e = np.exp(s - m)
        den = e.sum(axis=-1, keepdims=True)
        probs[h] = e / den
        lse[h] = (m + np.log(den))[:, 0]
        o[h] = probs[h] @ v[g]
    return o, probs, lse


def merge_attention_partials(partials: Sequence):
    """Combine partial attention results over disjoint key ranges.

    Each partial is (o_s, lse_s): softmax attention restricted to one key
    range (o_s [..., n, dh] normalised within the range, lse_s [..., n] its
    natural-log normaliser). Over the union of the ranges
        lse = log sum_s exp(lse_s),   o = sum_s exp(lse_s - lse) o_s,
    since exp(lse_s - lse) is the share of the total softmax mass that range s
    holds. This is the split-KV merge the flash-attention kernels of
    "SenseNova-U1" (vLLM-Omni recipe, measured kernel table) rest on.
    """
    lses = np.stack([np.asarray(l, dtype=np.float64) for _, l in partials])
    m = lses.max(axis=0)
    lse = m + np.log(np.sum(np.exp(lses - m), axis=0))
    o = sum(np.exp(l - lse)[..., None] * np.asarray(o_s, dtype=np.float64) for o_s, l in partials)
    return o, lse


def gqa_attention_split_kv(q: np.ndarray, k: np.ndarray, v: np.ndarray, bounds: Sequence[int]):
    """gqa_attention over the keys cut at ``bounds`` (0 < b_1 < ... < L,
    contiguous ranges [b_i, b_{i+1})), each range computed on its own and the
    partials merged by merge_attention_partials. Returns (o, lse)."""
    cuts = [0] + [int(b) for b in bounds] + [k.shape[1]]
    parts = []
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        o_s, _, lse_s = gqa_attention(q, k[:, lo:hi], v[:, lo:hi])
        parts.append((o_s, lse_s))
    return merge_attention_partials(parts)


def gqa_attention_backward(do: np.ndarray, q: np.ndarray, k: np.ndarray, v: np.ndarray,
                           o: np.ndarray, probs: np.ndarray):
    """Backward of gqa_attention; returns (dq, dk, dv) with dk, dv summed over
    the query heads of each group."""
    hq, hkv, dh = q.shape[0], k.shape[0], q.shape[-1]
    group = hq // hkv
    scale = 1.0 / math.sqrt(dh)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for h in range(hq):
        g = h // group
        p = probs[h]
        dp = do[h] @ v[g].T
        delta = np.sum(do[h] * o[h], axis=-1, keepdims=True)
        ds = p * (dp - delta)
        dq[h] = (ds @ k[g]) * scale
        dk[g] += (ds.T @ q[h]) * scale
        dv[g] += p.T @ do[h]
    return dq, dk, dv


def merge_lora(w: np.ndarray, a: np.ndarray, b: np.ndarray, scale: float) -> np.ndarray:
    """W' = RNE_bf16(W + s B A) (R7). "SenseNova-U1.5" (vLLM-Omni recipe),
    8-step distilled LoRA: the adapter is fused into the gen tower at load."""
    return round_to_bf16(w + scale * (b @ a))


# --------------------------------------------------------------------------
# the layer
# --------------------------------------------------------------------------
_PROJ = ("q", "k", "v", "o")


def _lora_parts(w: Dict[str, np.ndarray], name: str):
    a = w.get("a_" + name)
    b = w.get("b_" + name)
    return a, b


def _branch_forward(xb, w, kc_b, vc_b, plen, dims, scale, rows=None, positions=None):
    """One CFG branch. xb [N, d]; kc_b, vc_b [Hkv, P, dh]; plen = prefix_len[b].

    ``rows`` restricts the query rows (K/V still cover all N image tokens).
    ``positions`` overrides the image-token positions (default plen + i).
    """
    n = xb.shape[0]
    hq, hkv, dh = dims["n_q_heads"], dims["n_kv_heads"], dims["head_dim"]
    eps, theta = dims["rms_eps"], dims["rope_theta"]
    pos = plen + np.arange(n) if positions is None else np.asarray(positions)
    qrows = np.arange(n) if rows is None else np.asarray(rows)

    q_pre = lora_linear(xb[qrows], w["w_q"], *_lora_parts(w, "q"), scale)
    k_pre = lora_linear(xb, w["w_k"], *_lora_parts(w, "k"), scale)
    v_self = lora_linear(xb, w["w_v"], *_lora_parts(w, "v"), scale)

    q_pre = q_pre.reshape(len(qrows), hq, dh).transpose(1, 0, 2)
    k_pre = k_pre.reshape(n, hkv, dh).transpose(1, 0, 2)
    v_self = v_self.reshape(n, hkv, dh).transpose(1, 0, 2)

    q_n, q_hat, q_rstd = rms_norm_heads(q_pre, w["q_norm"], eps)
    k_n, k_hat, k_rstd = rms_norm_heads(k_pre, w["k_norm"], eps)
    q_rot = rope_rotate(q_n, pos[qrows], theta)
    k_rot = rope_rotate(k_n, pos, theta)

    k_all = np.concatenate([kc_b[:, :plen], k_rot], axis=1)
    v_all = np.concatenate([vc_b[:, :plen], v_self], axis=1)
    o, probs, lse = gqa_attention(q_rot, k_all, v_all)
    attn = o.transpose(1, 0, 2).reshape(len(qrows), hq * dh)
    y = lora_linear(attn, w["w_o"], *_lora_parts(w, "o"), scale)
    return dict(y=y, attn=attn, o=o, probs=probs, lse=lse, q_rot=q_rot, k_all=k_all,
                v_all=v_all, q_hat=q_hat, q_rstd=q_rstd, k_hat=k_hat, k_rstd=k_rstd, pos=pos,
                q_pre=q_pre, k_pre=k_pre, v_self=v_self)


def layer_forward(inp: Dict[str, np.ndarray], dims: Dict, lora_scale: float,
                  query_rows: Optional[Sequence[np.ndarray]] = None,
                  positions: Optional[Sequence[np.ndarray]] = None,
                  keep: bool = False) -> Dict:
    """Forward of the gen-tower attention layer for all CFG branches.

    inp: x [B, N, d]; w_* ; q_norm, k_norm [dh]; optional a_*, b_*;
         k_cache, v_cache [B, Hkv, P, dh]; prefix_len [B].
    Returns {"y": [B, N|rows, d]} (plus per-branch intermediates if keep).
    """
    x = inp["x"]
    out_y, branches = [], []
    for b in range(x.shape[0]):
        rows = None if query_rows is None else query_rows[b]
        pos = None if positions is None else positions[b]
        r = _branch_forward(x[b], inp, inp["k_cache"][b], inp["v_cache"][b],
                            int(inp["prefix_len"][b]), dims, lora_scale, rows, pos)
        out_y.append(r["y"])
        if keep:
            branches.append(r)
    res = {"y": np.stack(out_y) if query_rows is None else out_y}
    if keep:
        res["branches"] = branches
    return res


def layer_backward(inp: Dict[str, np.ndarray], dims: Dict, lora_scale: float, dy: np.ndarray) -> Dict:
    """LoRA-training backward through the layer (R6).

    Returns dx [B, N, d] and, for each of q, k, v, o, dA [r, in] and dB [out, r],
    summed over the CFG branches. No gradient flows into the cache, the base
    weights or the norm gains.
    """
    hq, hkv, dh = dims["n_q_heads"], dims["n_kv_heads"], dims["head_dim"]
    s = lora_scale
    x = inp["x"]
    nb, n, _ = x.shape
    has_lora = inp.get("a_q") is not None and inp["a_q"].shape[0] > 0
    grads = {}
    if has_lora:
        for name in _PROJ:
            grads["dA_" + name] = np.zeros_like(inp["a_" + name])
            grads["dB_" + name] = np.zeros_like(inp["b_" + name])
    dx = np.zeros_like(x)
    for b in range(nb):
        plen = int(inp["prefix_len"][b])
        f = _branch_forward(x[b], inp, inp["k_cache"][b], inp["v_cache"][b], plen, dims, s)
        # output projection: y = attn W_o^T + s (attn A_o^T) B_o^T
        dyb = dy[b]
        dattn = dyb @ inp["w_o"]
        if has_lora:
            g_o = dyb @ inp["b_o"]
            grads["dB_o"] += s * (dyb.T @ (f["attn"] @ inp["a_o"].T))
            grads["dA_o"] += s * (g_o.T @ f["attn"])
            dattn = dattn + s * (g_o @ inp["a_o"])
        do = dattn.reshape(n, hq, dh).transpose(1, 0, 2)
        dq_rot, dk_all, dv_all = gqa_attention_backward(do, f["q_rot"], f["k_all"], f["v_all"],
                                                        f["o"], f["probs"])
        dk_rot = dk_all[:, plen:]
        dv_self = dv_all[:, plen:]
        dq_n = rope_rotate(dq_rot, f["pos"], dims["rope_theta"], inverse=True)
        dk_n = rope_rotate(dk_rot, f["pos"], dims["rope_theta"], inverse=True)
        dq_pre = rms_norm_heads_backward(dq_n, f["q_hat"], f["q_rstd"], inp["q_norm"])
        dk_pre = rms_norm_heads_backward(dk_n, f["k_hat"], f["k_rstd"], inp["k_norm"])
        douts = {
            "q": dq_pre.transpose(1, 0, 2).reshape(n, hq * dh),
            "k": dk_pre.transpose(1, 0, 2).reshape(n, hkv * dh),
            "v": dv_self.transpose(1, 0, 2).reshape(n, hkv * dh),
        }
        for name, dout in douts.items():
            dx[b] += dout @ inp["w_" + name]
            if has_lora:
                a, bb = inp["a_" + name], inp["b_" + name]
                g_in = dout @ bb
                grads["dB_" + name] += s * (dout.T @ (x[b] @ a.T))
                grads["dA_" + name] += s * (g_in.T @ x[b])
                dx[b] += s * (g_in @ a)
    grads["dx"] = dx
    return grads


def dims_of(wl) -> Dict:
    """Plain dict of layer dims from a synth.LayerDims-like object."""
    d = wl.dims if hasattr(wl, "dims") else wl
    return dict(hidden=d.hidden, n_q_heads=d.n_q_heads, n_kv_heads=d.n_kv_heads,
                head_dim=d.head_dim, rms_eps=d.rms_eps, rope_theta=d.rope_theta)


def to_f64(tensors: Dict) -> Dict[str, np.ndarray]:
    """bf16/int torch tensors -> fp64 / int numpy arrays (exact)."""
    out = {}
    for k, t in tensors.items():
        if hasattr(t, "detach"):
            t = t.detach().cpu()
            out[k] = t.numpy() if not t.is_floating_point() else t.double().numpy()
        else:
            out[k] = np.asarray(t)
    return out

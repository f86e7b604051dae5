"""Pins for the prefix-tower oracle (oracle/mot_prefix_oracle.py), tied to
torch library routines (causal scaled_dot_product_attention, rms_norm,
complex rotation) and to properties of a causal encoder.

A plausible slip (mask off by one or missing, positions not starting at 0,
the key length ignored, the norm gain on the wrong tensor, a transposed
projection) fails at least one test here.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import mot_prefix_oracle as PO
from oracle import mot_attn_oracle as O
from mot_flow_matching_b200 import synth


def _inputs(seed, B=2, P=11, hidden=64, hq=4, hkv=2, dh=16):
    wl = synth.tiny_workload(batch=B, img_tokens=P, prefix=0, lora_rank=0, hidden=hidden, n_q_heads=hq,
                             n_kv_heads=hkv, head_dim=dh)
    t = synth.make_inputs(wl, seed, with_dy=False)
    return wl, O.to_f64({k: v for k, v in t.items() if k in ("x", "w_q", "w_k", "w_v", "w_o", "q_norm", "k_norm")})


def _torch_layer(t, dims, length):
    """The same layer from torch library routines, one branch at a time,
    over the first `length` tokens."""
    hq, hkv, dh = dims["n_q_heads"], dims["n_kv_heads"], dims["head_dim"]
    out = []
    for b in range(t["x"].shape[0]):
        x = torch.from_numpy(t["x"][b, :length])
        n = x.shape[0]

        def proj(w, h):
            return F.linear(x, torch.from_numpy(t[w])).view(n, h, dh).transpose(0, 1)

        def rope(z):
            pos = torch.arange(n, dtype=torch.float64)
            inv = dims["rope_theta"] ** (-2.0 * torch.arange(dh // 2, dtype=torch.float64) / dh)
            c = torch.polar(torch.ones(n, dh // 2, dtype=torch.float64), pos[:, None] * inv[None, :])
            zc = torch.complex(z[..., :dh // 2], z[..., dh // 2:]) * c
            return torch.cat([zc.real, zc.imag], dim=-1)

        q = rope(F.rms_norm(proj("w_q", hq), (dh,), torch.from_numpy(t["q_norm"]), eps=dims["rms_eps"]))
        k = rope(F.rms_norm(proj("w_k", hkv), (dh,), torch.from_numpy(t["k_norm"]), eps=dims["rms_eps"]))
        v = proj("w_v", hkv)
        o = F.scaled_dot_product_attention(q[None], k[None], v[None], is_causal=True, enable_gqa=True)[0]
        y = F.linear(o.transpose(0, 1).reshape(n, hq * dh), torch.from_numpy(t["w_o"]))
        out.append((y.numpy(), k.numpy(), v.numpy()))
    return out


def test_causal_attention_matches_sdpa():
    g = np.random.default_rng(1)
    q, k, v = g.standard_normal((4, 13, 8)), g.standard_normal((2, 13, 8)), g.standard_normal((2, 13, 8))
    o, lse = PO.causal_gqa_attention(q, k, v, 13)
    ref = F.scaled_dot_product_attention(torch.from_numpy(q)[None], torch.from_numpy(k)[None],
                                         torch.from_numpy(v)[None], is_causal=True, enable_gqa=True)[0]
    np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)
    # first query sees only the first key: its output is that key's value
    np.testing.assert_allclose(o[:, 0], np.repeat(v[:, 0], 2, axis=0), rtol=0, atol=1e-14)


@pytest.mark.parametrize("length", [1, 6, 11])
def test_layer_matches_torch_composition(length):
    wl, t = _inputs(7)
    dims = O.dims_of(wl)
    res = PO.prefix_forward(t, dims, [length, length])
    for b, (y, k, v) in enumerate(_torch_layer(t, dims, length)):
        np.testing.assert_allclose(res["y"][b, :length], y, rtol=0, atol=1e-11)
        np.testing.assert_allclose(res["k_cache"][b][:, :length], k, rtol=0, atol=1e-12)
        np.testing.assert_allclose(res["v_cache"][b][:, :length], v, rtol=0, atol=1e-12)


def test_prefix_property_and_padding():
    # a causal encoder: the first k rows do not depend on tokens after them,
    # and rows past a branch's length never reach rows before it
    wl, t = _inputs(8, P=11)
    dims = O.dims_of(wl)
    full = PO.prefix_forward(t, dims, [11, 11])
    part = PO.prefix_forward({**t, "x": t["x"][:, :5]}, dims, [5, 5])
    np.testing.assert_allclose(part["y"], full["y"][:, :5], rtol=0, atol=1e-12)
    np.testing.assert_allclose(part["k_cache"], full["k_cache"][:, :, :5], rtol=0, atol=1e-12)
    t2 = {**t, "x": t["x"].copy()}
    t2["x"][1, 7:] = 1e3  # padding rows of branch 1
    pad = PO.prefix_forward(t2, dims, [11, 7])
    ref = PO.prefix_forward(t, dims, [11, 7])
    np.testing.assert_allclose(pad["y"][1, :7], ref["y"][1, :7], rtol=0, atol=1e-12)
    np.testing.assert_allclose(pad["k_cache"][1][:, :7], ref["k_cache"][1][:, :7], rtol=0, atol=1e-12)


def test_cache_feeds_the_gen_layer_like_a_joint_sequence():
    # the gen layer's attention over [prefix cache ; self] equals causal-free
    # attention of the image tokens over the prompt keys computed here plus
    # their own keys: the positions of the cache are 0..len-1 and the image
    # tokens continue at len (P3 / R3)
    wl, t = _inputs(9, P=6)
    dims = O.dims_of(wl)
    res = PO.prefix_forward(t, dims, [6, 4])
    kc = PO.cache_bf16(res["k_cache"])
    # rows at or beyond len are padding: the gen layer ignores them
    gen = synth.tiny_workload(batch=2, img_tokens=5, prefix=6, lora_rank=0)
    tg = O.to_f64(synth.make_inputs(gen, 31, with_dy=False))
    tg["k_cache"], tg["v_cache"] = kc, PO.cache_bf16(res["v_cache"])
    tg["prefix_len"] = np.array([6, 4])
    out = O.layer_forward(tg, O.dims_of(gen), 0.0, keep=True)
    for b, pl in enumerate((6, 4)):
        br = out["branches"][b]
        np.testing.assert_array_equal(br["k_all"][:, :pl], kc[b][:, :pl])
        np.testing.assert_allclose(br["pos"], pl + np.arange(5))
    assert np.array_equal(PO.cache_bf16(np.array([1.0 + 2 ** -8, -3.0])), np.array([1.0, -3.0]))

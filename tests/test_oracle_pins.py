"""Pins for the oracle: each check ties it to something other than itself --
library routines (torch rms_norm, scaled_dot_product_attention, autograd,
complex exponentials, scipy logsumexp), closed forms, invariants of the method
and central finite differences on tiny shapes.

A plausible slip in the oracle (dropped LoRA term, wrong RoPE sign or pairing,
wrong GQA group mapping, transposed operand, missing 1/sqrt(dh), wrong norm
axis) fails at least one test here.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F
from scipy.special import logsumexp

from oracle import mot_attn_oracle as O
from mot_flow_matching_b200 import synth

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def rng(seed=0):
    return np.random.default_rng(seed)


# ------------------------------------------------------------------ rounding
def test_round_to_bf16_matches_torch_on_fp32_values():
    x = rng(1).standard_normal(20000).astype(np.float32) * np.float32(3.0)
    ref = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    assert np.array_equal(O.round_to_bf16(x.astype(np.float64)), ref)


def test_round_to_bf16_ties_and_single_rounding():
    one = 1.0
    # spacing of bf16 at 1 is 2^-7; halfway points go to the even mantissa
    assert O.round_to_bf16(np.array([one + 2**-8]))[0] == 1.0
    assert O.round_to_bf16(np.array([one + 3 * 2**-8]))[0] == one + 2**-6
    # just above a tie must round up (a detour through fp32 would lose 2^-40)
    assert O.round_to_bf16(np.array([one + 2**-8 + 2**-40]))[0] == one + 2**-7
    assert O.round_to_bf16(np.array([-(one + 2**-8 + 2**-40)]))[0] == -(one + 2**-7)


# ------------------------------------------------------------------ RMSNorm
def test_rmsnorm_matches_torch_rms_norm():
    x = rng(2).standard_normal((3, 7, 16))
    g = 1 + 0.1 * rng(3).standard_normal(16)
    y, _, _ = O.rms_norm_heads(x, g, 1e-6)
    ref = F.rms_norm(torch.from_numpy(x), (16,), torch.from_numpy(g), eps=1e-6).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_rmsnorm_constant_vector_closed_form():
    # x = c * ones -> rms |c| -> output sign(c) * gain (eps = 0)
    for c in (0.25, 3.0, -7.5):
        y, xhat, rstd = O.rms_norm_heads(np.full((1, 8), c), np.full(8, 2.0), 0.0)
        np.testing.assert_allclose(y, np.sign(c) * 2.0, rtol=1e-14)
        np.testing.assert_allclose(rstd, 1 / abs(c), rtol=1e-14)


def test_rmsnorm_unit_gain_rms_and_scale_invariance():
    x = rng(4).standard_normal((5, 128))
    y, _, _ = O.rms_norm_heads(x, np.ones(128), 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-13)
    y2, _, _ = O.rms_norm_heads(37.0 * x, np.ones(128), 0.0)
    np.testing.assert_allclose(y2, y, rtol=1e-12)
    # with eps > 0 a zero head maps to zero
    z, _, _ = O.rms_norm_heads(np.zeros((1, 128)), np.ones(128), 1e-6)
    assert np.all(z == 0)


def test_rmsnorm_backward_finite_difference():
    r = rng(5)
    x = r.standard_normal((4, 16))
    g = 1 + 0.1 * r.standard_normal(16)
    dy = r.standard_normal((4, 16))
    _, xhat, rstd = O.rms_norm_heads(x, g, 1e-6)
    dx = O.rms_norm_heads_backward(dy, xhat, rstd, g)
    h = 1e-6
    fd = np.zeros_like(x)
    for i in range(x.shape[0]):
        for j in range(x.shape[1]):
            xp, xm = x.copy(), x.copy()
            xp[i, j] += h
            xm[i, j] -= h
            fd[i, j] = np.sum(dy * (O.rms_norm_heads(xp, g, 1e-6)[0] - O.rms_norm_heads(xm, g, 1e-6)[0])) / (2 * h)
    np.testing.assert_allclose(dx, fd, rtol=1e-6, atol=1e-8)


# ------------------------------------------------------------------ RoPE
def test_rope_matches_complex_rotation():
    dh, theta = 128, 1e6
    x = rng(6).standard_normal((3, 11, dh))
    pos = np.array([0, 1, 2, 5, 63, 64, 400, 401, 4095, 4495, 8591])
    y = O.rope_rotate(x, pos, theta)
    z = x[..., : dh // 2] + 1j * x[..., dh // 2:]
    freq = 1.0 / theta ** (np.arange(0, dh, 2) / dh)
    zr = z * np.exp(1j * pos[:, None] * freq[None, :])
    np.testing.assert_allclose(y, np.concatenate([zr.real, zr.imag], -1), rtol=1e-12, atol=1e-12)


def test_rope_angle_closed_forms():
    phi = O.rope_angles(np.array([1.0, 1000.0]), 128, 1e6)
    assert phi[0, 0] == 1.0                       # j = 0: inverse frequency 1
    np.testing.assert_allclose(phi[0, 32], 1e-3, rtol=1e-14)  # theta^(-1/2)
    np.testing.assert_allclose(phi[1, 32], 1.0, rtol=1e-14)


def test_rope_identity_norm_relative_and_inverse():
    dh, theta = 128, 1e6
    r = rng(7)
    q = r.standard_normal((1, 1, dh))
    k = r.standard_normal((1, 1, dh))
    np.testing.assert_array_equal(O.rope_rotate(q, np.array([0]), theta), q)
    qr = O.rope_rotate(q, np.array([777]), theta)
    np.testing.assert_allclose(np.linalg.norm(qr), np.linalg.norm(q), rtol=1e-13)
    for m, n in ((9, 4), (4500, 17), (3, 3000)):
        lhs = np.sum(O.rope_rotate(q, np.array([m]), theta) * O.rope_rotate(k, np.array([n]), theta))
        rhs = np.sum(O.rope_rotate(q, np.array([m - n]), theta) * k)
        np.testing.assert_allclose(lhs, rhs, rtol=1e-9, atol=1e-9)
    back = O.rope_rotate(qr, np.array([777]), theta, inverse=True)
    np.testing.assert_allclose(back, q, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ attention
def _sdpa_ref(q, k, v):
    qt, kt, vt = (torch.from_numpy(t)[None] for t in (q, k, v))
    return F.scaled_dot_product_attention(qt, kt, vt, enable_gqa=True)[0].numpy()


def test_gqa_attention_matches_torch_sdpa():
    r = rng(8)
    q = r.standard_normal((8, 9, 16))
    k = r.standard_normal((2, 13, 16))
    v = r.standard_normal((2, 13, 16))
    o, probs, lse = O.gqa_attention(q, k, v)
    np.testing.assert_allclose(o, _sdpa_ref(q, k, v), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(probs.sum(-1), 1.0, rtol=1e-14)
    # lse against scipy on the explicitly expanded heads (group = 4, contiguous)
    s = np.einsum("hnd,hld->hnl", q, np.repeat(k, 4, axis=0)) / 4.0
    np.testing.assert_allclose(lse, logsumexp(s, axis=-1), rtol=1e-13)


def test_attention_zero_query_is_mean_of_values():
    r = rng(9)
    v = r.standard_normal((2, 29, 16))
    o, _, _ = O.gqa_attention(np.zeros((4, 3, 16)), r.standard_normal((2, 29, 16)), v)
    for h in range(4):
        np.testing.assert_allclose(o[h], np.broadcast_to(v[h // 2].mean(0), (3, 16)), rtol=1e-13)


def test_attention_single_key_returns_value():
    r = rng(10)
    v = r.standard_normal((1, 1, 16))
    o, _, _ = O.gqa_attention(r.standard_normal((2, 5, 16)), r.standard_normal((1, 1, 16)), v)
    np.testing.assert_allclose(o, np.broadcast_to(v[0, 0], o.shape), rtol=1e-14)


def test_attention_backward_finite_difference():
    r = rng(11)
    q = r.standard_normal((4, 3, 8))
    k = r.standard_normal((2, 5, 8))
    v = r.standard_normal((2, 5, 8))
    do = r.standard_normal((4, 3, 8))
    o, probs, _ = O.gqa_attention(q, k, v)
    dq, dk, dv = O.gqa_attention_backward(do, q, k, v, o, probs)
    h = 1e-6

    def loss(qq, kk, vv):
        return np.sum(do * O.gqa_attention(qq, kk, vv)[0])

    for arr, grad, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        fd = np.zeros_like(arr)
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            args_p = [q.copy(), k.copy(), v.copy()]
            args_m = [q.copy(), k.copy(), v.copy()]
            args_p[which][idx] += h
            args_m[which][idx] -= h
            fd[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        np.testing.assert_allclose(grad, fd, rtol=1e-6, atol=1e-8)


# ------------------------------------------------------------------ LoRA / merge
def test_lora_zero_up_equals_base_and_merge_identity():
    r = rng(12)
    x = r.standard_normal((6, 32))
    w = r.standard_normal((24, 32))
    a = r.standard_normal((4, 32))
    b = r.standard_normal((24, 4))
    base = O.lora_linear(x, w, None, None, 2.0)
    np.testing.assert_array_equal(O.lora_linear(x, w, a, np.zeros_like(b), 2.0), base)
    np.testing.assert_allclose(O.lora_linear(x, w, a, b, 0.5), x @ (w + 0.5 * b @ a).T, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(O.lora_linear(x, w, a, b, 0.5), base + 0.5 * (x @ (b @ a).T), rtol=1e-12, atol=1e-12)


def test_merge_rounds_once():
    r = rng(13)
    w = O.round_to_bf16(0.02 * r.standard_normal((16, 32)))
    a = O.round_to_bf16(r.standard_normal((4, 32)) / 16)
    b = O.round_to_bf16(0.01 * r.standard_normal((16, 4)))
    m = O.merge_lora(w, a, b, 1.0)
    exact = w + b @ a
    # nearest bf16: error at most half the bf16 spacing 2^(e-8) of exact's binade
    _, e = np.frexp(exact)
    assert np.all(np.abs(m - exact) <= np.ldexp(1.0, e - 9))
    np.testing.assert_array_equal(O.round_to_bf16(m), m)
    # and it is the bf16 neighbour that torch picks for fp32-exact sums
    np.testing.assert_array_equal(
        torch.from_numpy(exact.astype(np.float32)).to(torch.bfloat16).double().numpy()[np.abs(exact.astype(np.float32) - exact) == 0],
        m[np.abs(exact.astype(np.float32) - exact) == 0])


# ------------------------------------------------------------------ whole layer
def _tiny(seed=0, **kw):
    wl = synth.tiny_workload(**kw)
    t = synth.make_inputs(wl, 500 + seed, with_dy=True)
    return wl, t, O.to_f64(t), O.dims_of(wl)


def _torch_layer(t64, dims, scale):
    """The layer composed from torch library routines (fp64), autograd-capable."""
    hq, hkv, dh = dims["n_q_heads"], dims["n_kv_heads"], dims["head_dim"]
    T = {k: torch.from_numpy(np.asarray(v)) for k, v in t64.items()}
    for k in T:
        if k.startswith(("a_", "b_")) or k == "x":
            T[k].requires_grad_(True)
    x = T["x"]
    ys = []
    for b in range(x.shape[0]):
        plen = int(T["prefix_len"][b])
        n = x.shape[1]

        def lin(inp, name):
            out = F.linear(inp, T["w_" + name])
            if "a_" + name in T:
                out = out + scale * F.linear(F.linear(inp, T["a_" + name]), T["b_" + name])
            return out

        def rot(t, pos):  # complex-multiplication RoPE
            z = torch.complex(t[..., : dh // 2], t[..., dh // 2:])
            freq = 1.0 / dims["rope_theta"] ** (torch.arange(0, dh, 2, dtype=torch.float64) / dh)
            zr = z * torch.polar(torch.ones_like(freq)[None], pos[:, None] * freq[None])
            return torch.cat([zr.real, zr.imag], -1)

        pos = plen + torch.arange(n, dtype=torch.float64)
        q = lin(x[b], "q").view(n, hq, dh).transpose(0, 1)
        k = lin(x[b], "k").view(n, hkv, dh).transpose(0, 1)
        v = lin(x[b], "v").view(n, hkv, dh).transpose(0, 1)
        q = rot(F.rms_norm(q, (dh,), T["q_norm"], eps=dims["rms_eps"]), pos)
        k = rot(F.rms_norm(k, (dh,), T["k_norm"], eps=dims["rms_eps"]), pos)
        kk = torch.cat([T["k_cache"][b][:, :plen], k], 1)
        vv = torch.cat([T["v_cache"][b][:, :plen], v], 1)
        o = F.scaled_dot_product_attention(q[None], kk[None], vv[None], enable_gqa=True)[0]
        ys.append(lin(o.transpose(0, 1).reshape(n, hq * dh), "o"))
    return torch.stack(ys), T


@pytest.mark.parametrize("seed,kw", [(0, {}), (1, dict(n_q_heads=4, n_kv_heads=4)),
                                     (2, dict(n_q_heads=6, n_kv_heads=2, batch=3, prefix=4))])
def test_layer_forward_matches_torch_library_composition(seed, kw):
    wl, _, t64, dims = _tiny(seed, **kw)
    s = wl.lora_alpha / wl.lora_rank
    y = O.layer_forward(t64, dims, s)["y"]
    ref, _ = _torch_layer(t64, dims, s)
    np.testing.assert_allclose(y, ref.detach().numpy(), rtol=1e-11, atol=1e-12)


def test_layer_backward_matches_torch_autograd():
    wl, _, t64, dims = _tiny(3, n_q_heads=4, n_kv_heads=2)
    s = wl.lora_alpha / wl.lora_rank
    g = O.layer_backward(t64, dims, s, t64["dy"])
    ref, T = _torch_layer(t64, dims, s)
    (ref * torch.from_numpy(t64["dy"])).sum().backward()
    np.testing.assert_allclose(g["dx"], T["x"].grad.numpy(), rtol=1e-9, atol=1e-11)
    for name in ("q", "k", "v", "o"):
        np.testing.assert_allclose(g["dA_" + name], T["a_" + name].grad.numpy(), rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(g["dB_" + name], T["b_" + name].grad.numpy(), rtol=1e-9, atol=1e-11)


def test_layer_backward_central_differences():
    # d = 64, Hq = 4, Hkv = 2, dh = 16, N = 5, P = 3, r = 2, two branches
    wl, _, t64, dims = _tiny(4)
    s = wl.lora_alpha / wl.lora_rank
    g = O.layer_backward(t64, dims, s, t64["dy"])
    r = rng(14)

    def loss(inp):
        return float(np.sum(t64["dy"] * O.layer_forward(inp, dims, s)["y"]))

    h = 1e-5
    for name, gname in (("x", "dx"), ("a_q", "dA_q"), ("a_k", "dA_k"), ("a_v", "dA_v"), ("a_o", "dA_o"),
                        ("b_q", "dB_q"), ("b_k", "dB_k"), ("b_v", "dB_v"), ("b_o", "dB_o")):
        for _ in range(3):
            direction = r.standard_normal(t64[name].shape)
            p, m = dict(t64), dict(t64)
            p[name] = t64[name] + h * direction
            m[name] = t64[name] - h * direction
            fd = (loss(p) - loss(m)) / (2 * h)
            an = float(np.sum(g[gname] * direction))
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_layer_zero_lora_up_equals_rank0():
    wl, _, t64, dims = _tiny(5)
    t0 = {k: v for k, v in t64.items() if not k.startswith(("a_", "b_"))}
    tz = dict(t64)
    for name in ("q", "k", "v", "o"):
        tz["b_" + name] = np.zeros_like(t64["b_" + name])
    np.testing.assert_array_equal(O.layer_forward(tz, dims, 2.0)["y"], O.layer_forward(t0, dims, 2.0)["y"])


def test_layer_zero_query_weights_give_mean_of_values():
    # W_q = 0 and no q adapter -> q_pre = 0 -> RMSNorm(0) = 0 -> uniform attention
    wl, _, t64, dims = _tiny(6, lora_rank=0)
    t64["w_q"] = np.zeros_like(t64["w_q"])
    res = O.layer_forward(t64, dims, 1.0, keep=True)
    for b, br in enumerate(res["branches"]):
        for h in range(dims["n_q_heads"]):
            g = h // (dims["n_q_heads"] // dims["n_kv_heads"])
            np.testing.assert_allclose(br["o"][h], np.broadcast_to(br["v_all"][g].mean(0), br["o"][h].shape),
                                       rtol=1e-12, atol=1e-14)


def test_layer_ignores_cache_rows_beyond_prefix_len():
    wl, _, t64, dims = _tiny(7, prefix=6)
    t64["prefix_len"] = np.array([4, 6])
    y = O.layer_forward(t64, dims, 2.0)["y"]
    t2 = dict(t64)
    t2["k_cache"] = t64["k_cache"].copy()
    t2["v_cache"] = t64["v_cache"].copy()
    t2["k_cache"][0, :, 4:] = 1e3
    t2["v_cache"][0, :, 4:] = -1e3
    np.testing.assert_array_equal(O.layer_forward(t2, dims, 2.0)["y"], y)


def test_layer_token_permutation_with_positions():
    wl, _, t64, dims = _tiny(8)
    perm = np.array([3, 0, 4, 2, 1])
    pos = [3 + np.arange(5), 3 + np.arange(5)]
    y = O.layer_forward(t64, dims, 2.0, positions=pos)["y"]
    tp = dict(t64)
    tp["x"] = t64["x"][:, perm]
    yp = O.layer_forward(tp, dims, 2.0, positions=[p[perm] for p in pos])["y"]
    np.testing.assert_allclose(yp, y[:, perm], rtol=1e-12, atol=1e-13)


def test_layer_query_row_subset_matches_full():
    wl, _, t64, dims = _tiny(9)
    full = O.layer_forward(t64, dims, 2.0)["y"]
    rows = [np.array([4, 1]), np.array([0])]
    sub = O.layer_forward(t64, dims, 2.0, query_rows=rows)["y"]
    for b in range(2):
        np.testing.assert_allclose(sub[b], full[b][rows[b]], rtol=1e-13, atol=1e-14)


def test_merged_forward_close_to_unmerged():
    wl, _, t64, dims = _tiny(10)
    s = wl.lora_alpha / wl.lora_rank
    y = O.layer_forward(t64, dims, s)["y"]
    tm = {k: v for k, v in t64.items() if not k.startswith(("a_", "b_"))}
    for name in ("q", "k", "v", "o"):
        tm["w_" + name] = O.merge_lora(t64["w_" + name], t64["a_" + name], t64["b_" + name], s)
    ym = O.layer_forward(tm, dims, s)["y"]
    rms = np.sqrt(np.mean(y * y))
    assert np.max(np.abs(ym - y)) < 2e-2 * rms

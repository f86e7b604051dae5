"""Pins for the denoise-step oracle (oracle/mot_step_oracle.py): library
routines (torch rms_norm), closed forms of the schedule, the embedding and
the guidance, exactness of the Euler step on a straight flow, and invariants
of the composed step (residual identity, equal branches).

A plausible slip (guidance branches swapped, the velocity sign or its
divisor wrong, the shift formula inverted, a residual dropped, the norm on
the wrong axis) fails at least one test here.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from mot_flow_matching_b200 import synth
from oracle import mot_attn_oracle as O
from oracle import mot_step_oracle as SO


def test_rms_norm_rows_matches_torch():
    g = np.random.default_rng(1)
    h, gain = g.standard_normal((3, 5, 32)), 1 + 0.1 * g.standard_normal(32)
    ref = F.rms_norm(torch.from_numpy(h), (32,), torch.from_numpy(gain), eps=1e-6).numpy()
    np.testing.assert_allclose(SO.rms_norm_rows(h, gain, 1e-6), ref, rtol=1e-12, atol=1e-12)


def test_timestep_embedding_closed_form():
    e0 = SO.timestep_embedding(0.0, 8)
    np.testing.assert_array_equal(e0, [1, 1, 1, 1, 0, 0, 0, 0])
    e = SO.timestep_embedding(0.25, 8)
    # k = 0: frequency 1, angle 250; k = 2: frequency 10000^-0.5
    np.testing.assert_allclose([e[0], e[4]], [np.cos(250.0), np.sin(250.0)], rtol=1e-13)
    np.testing.assert_allclose([e[2], e[6]], [np.cos(2.5), np.sin(2.5)], rtol=1e-12)


def test_sigma_schedule():
    s = SO.sigma_schedule(4, 3.0)
    assert s[0] == 1.0 and s[-1] == 0.0 and np.all(np.diff(s) < 0)
    assert s[2] == pytest.approx(0.75)  # u = 1/2: 3 * 0.5 / (1 + 2 * 0.5)
    np.testing.assert_allclose(SO.sigma_schedule(5, 1.0), np.linspace(1, 0, 6), rtol=0, atol=1e-15)
    # a larger shift keeps sigma higher (more steps at high noise)
    assert np.all(SO.sigma_schedule(8, 3.0)[1:-1] > SO.sigma_schedule(8, 1.0)[1:-1])


def test_guidance_closed_forms():
    g = np.random.default_rng(2)
    c, i, u = (g.standard_normal(6) for _ in range(3))
    np.testing.assert_allclose(SO.guidance(np.stack([c, u]), 1.0, 1.0), c, rtol=0, atol=1e-15)
    np.testing.assert_allclose(SO.guidance(np.stack([c, u]), 0.0, 1.0), u, rtol=0, atol=1e-15)
    np.testing.assert_allclose(SO.guidance(np.stack([c, u]), 4.0, 1.0), u + 4 * (c - u), rtol=1e-14)
    np.testing.assert_allclose(SO.guidance(np.stack([c, i, u]), 1.0, 1.0), c, rtol=0, atol=1e-14)
    np.testing.assert_allclose(SO.guidance(np.stack([c, i, u]), 0.0, 1.0), i, rtol=0, atol=1e-14)
    np.testing.assert_allclose(SO.guidance(np.stack([c, i, u]), 0.0, 0.0), u, rtol=0, atol=1e-14)
    np.testing.assert_array_equal(SO.guidance(c[None], 4.0, 2.0), c)


def test_euler_is_exact_on_a_straight_flow():
    # z at sigma on the straight path from x0 to noise; with the exact x0 the
    # step lands on the same path at sigma_next
    g = np.random.default_rng(3)
    x0, noise = g.standard_normal(10), g.standard_normal(10)
    for s, s2 in ((1.0, 0.8), (0.5, 0.2), (0.1, 0.0)):
        z = (1 - s) * x0 + s * noise
        np.testing.assert_allclose(SO.euler_update(z, x0, s, s2, 0.02), (1 - s2) * x0 + s2 * noise, rtol=0,
                                   atol=1e-14)


def _tiny_model(seed, layers=2, B=2, N=5, P=3, C=12, I=48, rank=2):
    wl = synth.tiny_workload(batch=B, img_tokens=N, prefix=P, lora_rank=rank)
    d = wl.dims.hidden
    g = np.random.default_rng(seed)
    lw, caches = [], []
    for l in range(layers):
        t = O.to_f64(synth.make_inputs(wl, seed + 10 * l, with_dy=False))
        m = O.to_f64(synth.make_mlp_inputs(N, d, I, rank, seed + 10 * l + 5))
        w = {k: v for k, v in t.items() if k.startswith(("w_", "a_", "b_", "q_norm", "k_norm"))}
        w.update({"mlp_" + k: v for k, v in m.items() if k.startswith(("w_", "a_", "b_"))})
        w["norm_in"] = 1 + 0.1 * g.standard_normal(d)
        w["norm_post"] = 1 + 0.1 * g.standard_normal(d)
        lw.append(w)
        caches.append({"k_cache": t["k_cache"], "v_cache": t["v_cache"]})
    model = {"w_in": 0.05 * g.standard_normal((d, C)), "norm_out": 1 + 0.1 * g.standard_normal(d),
             "w_out": 0.05 * g.standard_normal((C, d))}
    return wl, model, lw, caches, g.standard_normal((N, C))


def test_step_residual_identity():
    # zero output projections and no adapters: every layer adds zero, so the
    # head sees h0 and the step is the closed-form composition
    wl, model, lw, caches, z = _tiny_model(4, rank=0)
    for w in lw:
        w["w_o"] = np.zeros_like(w["w_o"])
        w["mlp_w_down"] = np.zeros_like(w["mlp_w_down"])
    res = SO.denoise_step(z, model, lw, caches, [3, 2], O.dims_of(wl), 0.0, 0.6, 0.4, 4.0, 1.0, 0.02)
    h0 = O.round_to_bf16(z) @ model["w_in"].T + SO.timestep_embedding(0.6, wl.dims.hidden)
    x0 = O.round_to_bf16(SO.rms_norm_rows(h0, model["norm_out"], 1e-6)) @ model["w_out"].T
    np.testing.assert_allclose(res["h"][0], h0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(res["z_next"], z + (0.4 - 0.6) * (z - x0) / 0.6, rtol=0, atol=1e-12)


def test_step_equal_branches_make_guidance_vanish():
    # both branches see the same cache: their x0 agree, so any cfg gives the
    # single-branch step
    wl, model, lw, caches, z = _tiny_model(5, rank=2)
    for c in caches:
        c["k_cache"][1] = c["k_cache"][0]
        c["v_cache"][1] = c["v_cache"][0]
    a = SO.denoise_step(z, model, lw, caches, [3, 3], O.dims_of(wl), 1.0, 0.9, 0.7, 4.0, 1.0, 0.02)
    one = [{"k_cache": c["k_cache"][:1], "v_cache": c["v_cache"][:1]} for c in caches]
    b = SO.denoise_step(z, model, lw, one, [3], O.dims_of(wl), 1.0, 0.9, 0.7, 4.0, 1.0, 0.02)
    np.testing.assert_allclose(a["x0"][0], a["x0"][1], rtol=0, atol=1e-12)
    np.testing.assert_allclose(a["z_next"], b["z_next"], rtol=0, atol=1e-11)


def test_step_norm_gains_feed_their_own_half():
    # a zero post-attention gain zeroes the MLP's input, and the MLP maps 0 to
    # 0 (no bias): the step equals the one without the MLP's output weights
    wl, model, lw, caches, z = _tiny_model(6, rank=2)
    zero_post = [dict(w, norm_post=np.zeros_like(w["norm_post"])) for w in lw]
    no_mlp = [dict(w, mlp_w_down=np.zeros_like(w["mlp_w_down"]), mlp_b_down=np.zeros_like(w["mlp_b_down"]))
              for w in lw]
    args = ([3, 1], O.dims_of(wl), 1.0, 0.5, 0.3, 2.0, 1.0, 0.02)
    a = SO.denoise_step(z, model, zero_post, caches, *args)
    b = SO.denoise_step(z, model, no_mlp, caches, *args)
    np.testing.assert_allclose(a["h"], b["h"], rtol=0, atol=1e-12)
    full = SO.denoise_step(z, model, lw, caches, *args)
    assert not np.allclose(full["h"], a["h"])


def test_step_gemm_inputs_are_bf16_and_euler_uses_the_exact_z(monkeypatch):
    # S7: every input the step hands to a layer is a bf16 value (within half a
    # bf16 ulp of the unrounded norm), while the Euler update keeps the exact
    # z: moving z inside its bf16 rounding cell leaves x0 unchanged and moves
    # z_next by (z - z') sigma_next / sigma
    seen = []
    real_attn, real_mlp = SO.layer_forward, SO.mlp_forward

    def attn_spy(inp, dims, s):
        seen.append(inp["x"])
        return real_attn(inp, dims, s)

    def mlp_spy(x, w, s):
        seen.append(x)
        return real_mlp(x, w, s)

    monkeypatch.setattr(SO, "layer_forward", attn_spy)
    monkeypatch.setattr(SO, "mlp_forward", mlp_spy)
    wl, model, lw, caches, z = _tiny_model(7, rank=2)
    args = ([3, 2], O.dims_of(wl), 1.0, 0.8, 0.6, 4.0, 1.0, 0.02)
    a = SO.denoise_step(z, model, lw, caches, *args)
    assert len(seen) == len(lw) * (1 + len(args[0]))  # one attention call, one MLP call per branch
    for x in seen:
        assert np.array_equal(O.round_to_bf16(x), x)
    assert all(np.any(x != 0) for x in seen)
    z2 = O.round_to_bf16(z)
    assert not np.array_equal(z2, z)
    b = SO.denoise_step(z2, model, lw, caches, *args)
    np.testing.assert_array_equal(a["x0"], b["x0"])
    np.testing.assert_allclose(a["z_next"] - b["z_next"], (z - z2) * 0.6 / 0.8, rtol=0, atol=1e-14)

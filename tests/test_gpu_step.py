"""One gen-tower denoise step (mot_step_forward: patch embedding, pre-norm
decoder layers of the attention and MLP kernels, x0 head, guidance, Euler
update) against its fp64 oracle (oracle/mot_step_oracle.py).

With sigma = 0.5 and sigma_next = 0 the Euler update returns the guided x0
itself (z + (0 - 0.5)(z - x0)/0.5 = x0). Guidance is linear in the branches'
head outputs, x0_g = sum_b c_b x0_b with (cfg, 1 - cfg) for two branches and
(cfg, img_cfg - cfg, 1 - img_cfg) for three, so guidance weights that pick
one branch (cfg 1 or 0, img_cfg 1 or 0) return that branch's x0, and each
branch is held to the layers' parity bar on its own. The pages' guidance
(cfg 4, img_cfg 1.5) is then checked as that linear combination of the GPU's
own branch outputs (f32 arithmetic), and against the oracle within the bound
the same combination puts on the branch errors. A generic sigma pair checks
the update.

Bar: each branch's x0 comes out of 2 L sublayers (attention and MLP per
layer) whose errors, each within the layer bar, add into the residual
stream independently, so the step's bar is the layer bar times sqrt(2 L)."""
import numpy as np
import pytest
import torch

from mot_flow_matching_b200 import synth
from mot_flow_matching_b200.layer import MotAttnLayer
from mot_flow_matching_b200.mlp import MotMlp
from mot_flow_matching_b200.step import MotStep
from oracle import mot_attn_oracle as O
from oracle import mot_step_oracle as SO
from tests.gpu_helpers import MAX_TOL, MEAN_TOL, assert_parity, ensure_built

pytestmark = pytest.mark.gpu

ATTN_KEYS = ("w_q", "w_k", "w_v", "w_o", "q_norm", "k_norm", "a_q", "a_k", "a_v", "a_o", "b_q", "b_k", "b_v", "b_o")
MLP_KEYS = ("w_gate", "w_up", "w_down", "a_gate", "a_up", "a_down", "b_gate", "b_up", "b_down")


def _build(inp, wl, inter):
    ensure_built()
    d = wl.dims
    attn, mlps, keep = [], [], []
    for t in inp["layers"]:
        td = {k: v.cuda() for k, v in t.items() if k != "prefix_len"}
        keep.append(td)
        attn.append(MotAttnLayer({k: td[k] for k in ATTN_KEYS if k in td}, lora_rank=wl.lora_rank,
                                 lora_alpha=wl.lora_alpha, max_batch=wl.batch, max_img_tokens=wl.img_tokens,
                                 max_prefix=wl.prefix, hidden=d.hidden, n_q_heads=d.n_q_heads,
                                 n_kv_heads=d.n_kv_heads))
        mlps.append(MotMlp({k: td["mlp_" + k] for k in MLP_KEYS if "mlp_" + k in td}, lora_rank=wl.lora_rank,
                           lora_alpha=wl.lora_alpha, max_tokens=wl.batch * wl.img_tokens, hidden=d.hidden,
                           intermediate=inter))
    w_in, norm_out, w_out = (inp[k].cuda() for k in ("w_in", "norm_out", "w_out"))
    step = MotStep(attn, mlps, [td["norm_in"] for td in keep], [td["norm_post"] for td in keep], w_in, norm_out,
                   w_out)
    return step, keep, (w_in, norm_out, w_out)


def _oracle(inp, wl, plen, sigma, sigma_next, cfg, img_cfg):
    layers, caches = [], []
    for t in inp["layers"]:
        t64 = O.to_f64({k: v for k, v in t.items() if k != "prefix_len"})
        layers.append({k: v for k, v in t64.items() if k not in ("x", "k_cache", "v_cache")})
        caches.append({"k_cache": t64["k_cache"], "v_cache": t64["v_cache"]})
    model = {k: inp[k].double().numpy() for k in ("w_in", "norm_out", "w_out")}
    s = wl.lora_alpha / wl.lora_rank if wl.lora_rank else 0.0
    return SO.denoise_step(inp["z"].double().numpy(), model, layers, caches, plen, O.dims_of(wl), s, sigma,
                           sigma_next, cfg, img_cfg, 0.02)


def _run(step, keep, inp, wl, plen, sigma, sigma_next, cfg, img_cfg):
    z = inp["z"].cuda()
    zn = torch.empty_like(z)
    zb = torch.empty(z.shape, dtype=torch.bfloat16, device="cuda")
    step.forward(z, [td["k_cache"] for td in keep], [td["v_cache"] for td in keep], plen, sigma, sigma_next,
                 cfg, img_cfg, 0.02, z_next=zn, z_next_bf16=zb)
    torch.cuda.synchronize()
    for a in step.attn_layers:
        assert a.device_status() == 0
    for m in step.mlps:
        assert m.device_status() == 0
    assert torch.equal(zn.to(torch.bfloat16).view(torch.int16), zb.view(torch.int16))
    return zn.double().cpu().numpy()


SMALL = synth.LayerDims(hidden=512, n_q_heads=4, n_kv_heads=2)


def _branch_coeffs(B, cfg, img_cfg):
    """x0_g = sum_b c_b x0_b: the guidance of the pages as branch weights."""
    if B == 1:
        return [1.0]
    if B == 2:
        return [cfg, 1.0 - cfg]
    return [cfg, img_cfg - cfg, 1.0 - img_cfg]


def _picks(B):
    """(cfg, img_cfg) that return branch b alone, for each b."""
    return {1: [(1.0, 1.0)], 2: [(1.0, 1.0), (0.0, 1.0)], 3: [(1.0, 1.0), (0.0, 1.0), (0.0, 0.0)]}[B]


def _bar(n_layers):
    f = float(np.sqrt(2 * n_layers))
    return dict(max_tol=MAX_TOL * f, mean_tol=MEAN_TOL * f)


def _check_branches_and_guidance(step, keep, inp, wl, plen, cfg, img_cfg, what):
    B = wl.batch
    bar = _bar(len(inp["layers"]))
    ref = _oracle(inp, wl, plen, 0.5, 0.0, cfg, img_cfg)
    branch = []
    for b, (c, ic) in enumerate(_picks(B)):
        assert _branch_coeffs(B, c, ic) == [1.0 if i == b else 0.0 for i in range(B)]
        got = _run(step, keep, inp, wl, plen, 0.5, 0.0, c, ic)
        assert_parity(got, ref["x0"][b], f"{what}: x0 of branch {b}", **bar)
        branch.append(got)
    got = _run(step, keep, inp, wl, plen, 0.5, 0.0, cfg, img_cfg)
    co = _branch_coeffs(B, cfg, img_cfg)
    lin = sum(c * x for c, x in zip(co, branch))
    # the combine and the Euler update (which passes z - x0 through f32) in
    # f32: a few roundings of each term, z included
    az = np.abs(inp["z"].double().numpy())
    scale = sum(abs(c) * (np.abs(x) + az) for c, x in zip(co, branch)) + np.abs(lin) + az
    assert np.all(np.abs(got - lin) <= 8 * 2.0 ** -24 * scale + 1e-30), what
    exp = SO.guidance(ref["x0"], cfg, img_cfg)
    np.testing.assert_allclose(ref["z_next"], exp, rtol=0, atol=1e-12)
    err = sum(abs(c) * np.abs(x - r) for c, x, r in zip(co, branch, ref["x0"]))
    assert np.all(np.abs(got - exp) <= err * (1 + 1e-6) + 8 * 2.0 ** -24 * scale), what


@pytest.mark.parametrize("B,N,P,plen,n_layers,rank,cfg,img_cfg", [
    (2, 200, 37, [37, 20], 2, 16, 4.0, 1.0),
    (3, 129, 64, [64, 64, 0], 2, 8, 4.0, 1.5),
    (1, 77, 5, [5], 1, 0, 4.0, 1.0),
])
def test_step_small_dims_x0(cuda_ready, B, N, P, plen, n_layers, rank, cfg, img_cfg):
    wl = synth.Workload("step", B, N, P, rank, float(rank), dims=SMALL)
    inp = synth.make_step_inputs(n_layers, wl, 384, 256, 7100 + N)
    for t in inp["layers"]:
        t["prefix_len"] = torch.tensor(plen, dtype=torch.int32)
    step, keep, _ = _build(inp, wl, 384)
    _check_branches_and_guidance(step, keep, inp, wl, plen, cfg, img_cfg, "guided x0")
    step.close()


@pytest.mark.parametrize("which", ["schedule_step", "below_t_eps"])
def test_step_euler_update(cuda_ready, which):
    wl = synth.Workload("step", 2, 160, 48, 16, 16.0, dims=SMALL)
    inp = synth.make_step_inputs(2, wl, 384, 256, 7300)
    step, keep, _ = _build(inp, wl, 384)
    sig = SO.sigma_schedule(8, 3.0)
    # a step of the shifted schedule, or the last one from sigma = 0.01 below
    # t_eps = 0.02, where the velocity divides by t_eps instead of sigma
    s0, s1 = (float(sig[3]), float(sig[4])) if which == "schedule_step" else (0.01, 0.0)
    # cfg 1: the update applied to the conditional branch's x0 (the guidance
    # combine has its own test)
    got = _run(step, keep, inp, wl, [48, 48], s0, s1, 1.0, 1.0)
    ref = _oracle(inp, wl, [48, 48], s0, s1, 1.0, 1.0)
    z = inp["z"].double().numpy()
    # the update part of the step, z_next - z = (s1 - s0) (z - x0) / max(s0, t_eps)
    assert_parity(got - z, ref["z_next"] - z, "z_next - z", **_bar(2))
    step.close()


def test_step_full_dims_two_layers(cuda_ready):
    # the layer dims of the 2048^2 workloads (hidden 4096, 32/8 heads,
    # intermediate 12288, 3072 pixel values per patch), two layers, a
    # 512^2 image (256 tokens) with CFG over 64 cached keys
    wl = synth.Workload("step", 2, 256, 64, 16, 16.0)
    inp = synth.make_step_inputs(2, wl, synth.MLP_INTER, 3072, 7400)
    step, keep, _ = _build(inp, wl, synth.MLP_INTER)
    _check_branches_and_guidance(step, keep, inp, wl, [64, 64], 4.0, 1.0, "guided x0 (full dims)")
    step.close()

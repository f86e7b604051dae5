"""One gen-tower denoise step (mot_step_forward: patch embedding, pre-norm
decoder layers of the attention and MLP kernels, x0 head, guidance, Euler
update) against its fp64 oracle (oracle/mot_step_oracle.py).

With sigma = 0.5 and sigma_next = 0 the Euler update returns the guided x0
itself (z + (0 - 0.5)(z - x0)/0.5 = x0), so the step's output is compared
with the oracle's guided head output directly; a generic sigma pair checks
the update. Parity bar on the f32 result as for the layers."""
import numpy as np
import pytest
import torch

from mot_flow_matching_b200 import synth
from mot_flow_matching_b200.layer import MotAttnLayer
from mot_flow_matching_b200.mlp import MotMlp
from mot_flow_matching_b200.step import MotStep
from oracle import mot_attn_oracle as O
from oracle import mot_step_oracle as SO
from tests.gpu_helpers import assert_parity, ensure_built

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


@pytest.mark.parametrize("B,N,P,plen,n_layers,rank,cfg,img_cfg", [
    (2, 200, 37, [37, 20], 2, 16, 4.0, 1.0),
    (3, 129, 64, [64, 64, 0], 2, 8, 4.0, 1.5),
    (1, 77, 5, [5], 1, 0, 1.0, 1.0),
])
def test_step_small_dims_x0(cuda_ready, B, N, P, plen, n_layers, rank, cfg, img_cfg):
    wl = synth.Workload("step", B, N, P, rank, float(rank), dims=SMALL)
    inp = synth.make_step_inputs(n_layers, wl, 384, 256, 7100 + N)
    for t in inp["layers"]:
        t["prefix_len"] = torch.tensor(plen, dtype=torch.int32)
    step, keep, _ = _build(inp, wl, 384)
    got = _run(step, keep, inp, wl, plen, 0.5, 0.0, cfg, img_cfg)
    ref = _oracle(inp, wl, plen, 0.5, 0.0, cfg, img_cfg)
    # sigma 0.5 -> 0: the step returns the guided x0
    assert_parity(got, SO.guidance(ref["x0"], cfg, img_cfg), "guided x0")
    np.testing.assert_allclose(ref["z_next"], SO.guidance(ref["x0"], cfg, img_cfg), rtol=0, atol=1e-12)
    step.close()


def test_step_euler_update(cuda_ready):
    wl = synth.Workload("step", 2, 160, 48, 16, 16.0, dims=SMALL)
    inp = synth.make_step_inputs(2, wl, 384, 256, 7300)
    step, keep, _ = _build(inp, wl, 384)
    sig = SO.sigma_schedule(8, 3.0)
    s0, s1 = float(sig[3]), float(sig[4])
    got = _run(step, keep, inp, wl, [48, 48], s0, s1, 4.0, 1.0)
    ref = _oracle(inp, wl, [48, 48], s0, s1, 4.0, 1.0)
    z = inp["z"].double().numpy()
    # the update part of the step, z_next - z = (s1 - s0) (z - x0) / s0
    assert_parity(got - z, ref["z_next"] - z, "z_next - z")
    step.close()


def test_step_full_dims_two_layers(cuda_ready):
    # the layer dims of the 2048^2 workloads (hidden 4096, 32/8 heads,
    # intermediate 12288, 3072 pixel values per patch), two layers, a
    # 512^2 image (256 tokens) with CFG over 64 cached keys
    wl = synth.Workload("step", 2, 256, 64, 16, 16.0)
    inp = synth.make_step_inputs(2, wl, synth.MLP_INTER, 3072, 7400)
    step, keep, _ = _build(inp, wl, synth.MLP_INTER)
    got = _run(step, keep, inp, wl, [64, 64], 0.5, 0.0, 4.0, 1.0)
    ref = _oracle(inp, wl, [64, 64], 0.5, 0.0, 4.0, 1.0)
    assert_parity(got, SO.guidance(ref["x0"], 4.0, 1.0), "guided x0 (full dims)")
    step.close()

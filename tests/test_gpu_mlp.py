"""Parity of the gen-tower SwiGLU MLP (through the C ABI, include/mot_mlp.h)
against its fp64 oracle on seeded synth inputs: full forward outputs at the
512^2, 1024^2 and 2048^2 CFG token counts, the saved g, u, h, small-dim
ragged shapes, the LoRA-training backward (dx, dA, dB) in full at the 2048^2
training size and on small dims, and the invariants (lora_up = 0 equals the
rank-0 path bit for bit, bf16 = RNE(f32), determinism, accumulate, f16
overflow reported)."""
import numpy as np
import pytest
import torch

from mot_flow_matching_b200 import synth
from mot_flow_matching_b200.mlp import MotMlp
from oracle import mot_mlp_oracle as MO
from tests.gpu_helpers import assert_parity, bf16_is_rne_of_f32, ensure_built

pytestmark = pytest.mark.gpu

NAMES = ("gate", "up", "down")


def _dev(t):
    return {k: v.cuda() for k, v in t.items()}


def _f64(t):
    return {k: v.double().numpy() for k, v in t.items()}


def _make(t, rank, alpha, tokens, hidden, inter, backward=False):
    ensure_built()
    td = _dev(t)
    w = {k: td[k] for k in td if k.startswith(("w_", "a_", "b_"))}
    return td, MotMlp(w, lora_rank=rank if "a_gate" in td else 0, lora_alpha=alpha, max_tokens=tokens,
                      enable_backward=backward, hidden=hidden, intermediate=inter)


def _forward(mlp, td, saved=None):
    x = td["x"]
    y = torch.empty_like(x)
    y32 = torch.empty(x.shape, dtype=torch.float32, device=x.device)
    mlp.forward(x, y=y, y_f32=y32, saved=saved)
    torch.cuda.synchronize()
    return y, y32, mlp.device_status()


@pytest.mark.parametrize("index", [0, 1, 2])
def test_mlp_forward_full(cuda_ready, index):
    wl = synth.MLP_WORKLOADS[index]
    t = synth.mlp_workload_inputs(index)
    td, mlp = _make(t, wl.lora_rank, wl.lora_alpha, wl.tokens, wl.hidden, wl.inter, backward=index == 0)
    saved = mlp.new_saved(wl.tokens) if index == 0 else None
    y, y32, status = _forward(mlp, td, saved)
    assert status == 0
    s = wl.lora_alpha / wl.lora_rank
    ref = MO.mlp_forward(t["x"].double().numpy(), _f64(t), s)
    assert_parity(y32.double().cpu().numpy(), ref["y"], "y f32")
    assert bf16_is_rne_of_f32(y, y32)
    if saved is not None:
        # saved activations: u_gu, then h, g, u (f16 [T, I] each)
        T, I, RP = wl.tokens, wl.inter, 64
        off = ((T * 2 * RP * 2 + 1023) // 1024) * 1024
        nb = T * I * 2
        stride = ((nb + 1023) // 1024) * 1024
        for k, name in enumerate(("h", "g", "u")):
            got = saved[off + k * stride: off + k * stride + nb].view(torch.float16).view(T, I).double().cpu().numpy()
            assert_parity(got, ref[name], name)
    assert mlp.last_launch_count() == 5  # prep, LoRA down gu, gate/up, LoRA down d, down
    mlp.close()


SMALL = dict(hidden=512, inter=384)


@pytest.mark.parametrize("tokens,rank", [(1, 0), (77, 8), (300, 16), (129, 64), (200, 128)])
def test_mlp_forward_small_dims_ragged(cuda_ready, tokens, rank):
    t = synth.make_mlp_inputs(tokens, SMALL["hidden"], SMALL["inter"], rank, 7000 + tokens)
    td, mlp = _make(t, rank, float(2 * rank), tokens, SMALL["hidden"], SMALL["inter"])
    y, y32, status = _forward(mlp, td)
    assert status == 0
    ref = MO.mlp_forward(t["x"].double().numpy(), _f64(t), 2.0 if rank else 0.0)
    assert_parity(y32.double().cpu().numpy(), ref["y"], "y f32")
    assert bf16_is_rne_of_f32(y, y32)
    mlp.close()


def test_mlp_zero_lora_up_is_bitwise_rank0(cuda_ready):
    wl = synth.MLP_WORKLOADS[0]
    t = synth.mlp_workload_inputs(0)
    for n in NAMES:
        t["b_" + n] = torch.zeros_like(t["b_" + n])
    td, mlp = _make(t, wl.lora_rank, wl.lora_alpha, wl.tokens, wl.hidden, wl.inter)
    y_lora = _forward(mlp, td)[1].clone()
    t0 = {k: v for k, v in t.items() if not k.startswith(("a_", "b_"))}
    td0, mlp0 = _make(t0, 0, 0.0, wl.tokens, wl.hidden, wl.inter)
    y_base = _forward(mlp0, td0)[1]
    assert torch.equal(y_lora.view(torch.int32), y_base.view(torch.int32))
    mlp.close()
    mlp0.close()


def _backward(mlp, td, tokens, rank, accumulate=False, d_a=None, d_b=None):
    saved = mlp.new_saved(tokens)
    x = td["x"]
    mlp.forward(x, saved=saved)
    if rank and d_a is None:
        d_a = [torch.zeros(td["a_" + n].shape, device="cuda") for n in NAMES]
        d_b = [torch.zeros(td["b_" + n].shape, device="cuda") for n in NAMES]
    dx = torch.empty_like(x)
    dx32 = torch.empty(x.shape, dtype=torch.float32, device="cuda")
    mlp.backward(td["dy"], x, saved, dx=dx, dx_f32=dx32, d_a=d_a, d_b=d_b, accumulate=accumulate)
    torch.cuda.synchronize()
    return dx, dx32, d_a, d_b, mlp.device_status()


def _check_grads(t, s, dx, dx32, d_a, d_b, rank):
    ref = MO.mlp_backward(t["x"].double().numpy(), _f64(t), s, t["dy"].double().numpy())
    assert_parity(dx32.double().cpu().numpy(), ref["dx"], "dx f32")
    assert bf16_is_rne_of_f32(dx, dx32)
    if rank:
        for j, n in enumerate(NAMES):
            assert_parity(d_a[j].double().cpu().numpy(), ref["dA_" + n], "dA_" + n)
            assert_parity(d_b[j].double().cpu().numpy(), ref["dB_" + n], "dB_" + n)
    return ref


def test_mlp_backward_train_2048sq_full(cuda_ready):
    wl = synth.MLP_WORKLOADS[4]
    t = synth.mlp_workload_inputs(4)
    td, mlp = _make(t, wl.lora_rank, wl.lora_alpha, wl.tokens, wl.hidden, wl.inter, backward=True)
    dx, dx32, d_a, d_b, status = _backward(mlp, td, wl.tokens, wl.lora_rank)
    assert status == 0
    _check_grads(t, wl.lora_alpha / wl.lora_rank, dx, dx32, d_a, d_b, wl.lora_rank)
    # deterministic, and accumulate adds into what is there
    dx2, dx32_2, d_a2, d_b2, status = _backward(mlp, td, wl.tokens, wl.lora_rank)
    assert status == 0
    assert torch.equal(dx32.view(torch.int32), dx32_2.view(torch.int32))
    for j in range(3):
        assert torch.equal(d_a[j].view(torch.int32), d_a2[j].view(torch.int32))
        assert torch.equal(d_b[j].view(torch.int32), d_b2[j].view(torch.int32))
    acc_a = [a.clone() for a in d_a]
    acc_b = [b.clone() for b in d_b]
    _backward(mlp, td, wl.tokens, wl.lora_rank, accumulate=True, d_a=acc_a, d_b=acc_b)
    for j in range(3):
        torch.testing.assert_close(acc_a[j], 2 * d_a[j], rtol=1e-5, atol=1e-6)
        torch.testing.assert_close(acc_b[j], 2 * d_b[j], rtol=1e-5, atol=1e-6)
    mlp.close()


@pytest.mark.parametrize("tokens,rank", [(77, 8), (300, 16), (129, 0), (200, 128)])
def test_mlp_backward_small_dims(cuda_ready, tokens, rank):
    t = synth.make_mlp_inputs(tokens, SMALL["hidden"], SMALL["inter"], rank, 8000 + tokens, with_dy=True)
    td, mlp = _make(t, rank, float(rank), tokens, SMALL["hidden"], SMALL["inter"], backward=True)
    dx, dx32, d_a, d_b, status = _backward(mlp, td, tokens, rank)
    assert status == 0
    _check_grads(t, 1.0 if rank else 0.0, dx, dx32, d_a, d_b, rank)
    mlp.close()


def test_mlp_f16_overflow_is_reported(cuda_ready):
    t = synth.make_mlp_inputs(64, SMALL["hidden"], SMALL["inter"], 0, 99)
    t["x"][3] = 3e4  # g, u far beyond the f16 range for this token
    td, mlp = _make(t, 0, 0.0, 64, SMALL["hidden"], SMALL["inter"])
    assert _forward(mlp, td)[2] == 7  # MOT_ERR_NUMERIC
    t2 = synth.make_mlp_inputs(64, SMALL["hidden"], SMALL["inter"], 0, 98)
    td2 = {"x": t2["x"].cuda()}
    y = torch.empty_like(td2["x"])
    mlp.forward(td2["x"], y=y)
    torch.cuda.synchronize()
    assert mlp.device_status() == 0
    mlp.close()

"""LoRA-training backward of the CUDA layer (through the C ABI) against the
oracle's analytic backward on the same seeded inputs: dx, dA and dB of the
q/k/v/o adapters, each within max |err| <= 1e-2 RMS(ref) and mean |err| <=
2e-3 RMS(ref) on the f32 outputs."""
import numpy as np
import pytest
import torch

from mot_flow_matching_b200 import synth
from oracle import mot_attn_oracle as O
from tests.gpu_helpers import assert_parity, bf16_is_rne_of_f32, make_layer, run_forward, to_dev

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "o")


def run_backward(wl, t, accumulate=False, init=None, layer=None):
    td = to_dev(t)
    if layer is None:
        layer = make_layer(wl, td, backward=True)
    _, _, sv, status = run_forward(layer, td, saved=True)
    assert status == 0
    x = td["x"]
    dx = torch.full_like(x, float("nan"))
    dx32 = torch.full(x.shape, float("nan"), dtype=torch.float32, device="cuda")
    d_a = d_b = None
    if wl.lora_rank:
        d_a = [(init["dA_" + n].clone() if init else torch.zeros(td["a_" + n].shape, device="cuda")) for n in NAMES]
        d_b = [(init["dB_" + n].clone() if init else torch.zeros(td["b_" + n].shape, device="cuda")) for n in NAMES]
    layer.backward(td["dy"], x, td["k_cache"], td["v_cache"], [int(v) for v in t["prefix_len"]], sv, dx=dx,
                   dx_f32=dx32, d_a=d_a, d_b=d_b, accumulate=accumulate)
    torch.cuda.synchronize()
    status = layer.device_status()
    return dx, dx32, d_a, d_b, status, layer


def oracle_backward(wl, t):
    t64 = O.to_f64(t)
    s = wl.lora_alpha / wl.lora_rank if wl.lora_rank else 0.0
    return O.layer_backward(t64, O.dims_of(wl), s, t64["dy"])


def check_all(wl, t, dx, dx32, d_a, d_b, ref):
    assert_parity(dx32.double().cpu().numpy(), ref["dx"], "dx f32")
    assert bf16_is_rne_of_f32(dx, dx32)
    if wl.lora_rank:
        for i, n in enumerate(NAMES):
            assert_parity(d_a[i].double().cpu().numpy(), ref["dA_" + n], "dA_" + n)
            assert_parity(d_b[i].double().cpu().numpy(), ref["dB_" + n], "dB_" + n)


SMALL = dict(hidden=512, n_q_heads=4, n_kv_heads=2)


@pytest.mark.parametrize("batch,n,p,plen,rank", [
    (1, 128, 64, [64], 16),
    (2, 200, 37, [37, 20], 16),   # ragged query and key tiles, prefix shorter than P_max
    (3, 129, 128, [0, 128, 5], 8),
    (1, 77, 5, [5], 128),
    (2, 256, 0, [0, 0], 0),       # no cache, no adapters
])
def test_backward_small_dims(cuda_ready, batch, n, p, plen, rank):
    dims = synth.LayerDims(**SMALL)
    wl = synth.Workload("small", batch, n, p, rank, float(2 * rank), train=True, dims=dims)
    t = synth.make_inputs(wl, 7000 + n + rank, with_dy=True)
    t["prefix_len"] = torch.tensor(plen, dtype=torch.int32)
    dx, dx32, d_a, d_b, status, _ = run_backward(wl, t)
    assert status == 0
    check_all(wl, t, dx, dx32, d_a, d_b, oracle_backward(wl, t))


def test_backward_1024sq_full_dims(cuda_ready):
    # the training layer at 1024^2: one branch, 1024 image tokens, 400 cached keys, LoRA r32
    wl = synth.Workload("train_1024sq_b1", 1, 1024, 400, 32, 32.0, train=True)
    t = synth.make_inputs(wl, 4000, with_dy=True)
    dx, dx32, d_a, d_b, status, _ = run_backward(wl, t)
    assert status == 0
    check_all(wl, t, dx, dx32, d_a, d_b, oracle_backward(wl, t))


def test_backward_accumulate_and_determinism(cuda_ready):
    dims = synth.LayerDims(**SMALL)
    wl = synth.Workload("small", 2, 160, 40, 16, 16.0, train=True, dims=dims)
    t = synth.make_inputs(wl, 8080, with_dy=True)
    dx1, dx32a, da1, db1, st1, layer = run_backward(wl, t)
    dx2, dx32b, da2, db2, st2, _ = run_backward(wl, t, layer=layer)
    assert st1 == 0 and st2 == 0
    assert torch.equal(dx32a.view(torch.int32), dx32b.view(torch.int32))
    for a, b in zip(da1 + db1, da2 + db2):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    init = {"dA_" + n: torch.full_like(da1[i], 0.25) for i, n in enumerate(NAMES)}
    init.update({"dB_" + n: torch.full_like(db1[i], -0.5) for i, n in enumerate(NAMES)})
    _, _, da3, db3, st3, _ = run_backward(wl, t, accumulate=True, init=init, layer=layer)
    assert st3 == 0
    for i, n in enumerate(NAMES):
        torch.testing.assert_close(da3[i], da1[i] + 0.25, rtol=0, atol=1e-6 * (1 + da1[i].abs().max().item()))
        torch.testing.assert_close(db3[i], db1[i] - 0.5, rtol=0, atol=1e-6 * (1 + db1[i].abs().max().item()))


def test_backward_rejects_missing_saved_state(cuda_ready):
    from mot_flow_matching_b200._abi import MOT_ERR_NO_SAVED_STATE, MotError
    dims = synth.LayerDims(**SMALL)
    wl = synth.Workload("small", 1, 64, 8, 0, 0.0, train=True, dims=dims)
    t = synth.make_inputs(wl, 5, with_dy=True)
    td = to_dev(t)
    layer = make_layer(wl, td, backward=True)
    with pytest.raises(MotError) as e:
        layer.backward(td["dy"], td["x"], td["k_cache"], td["v_cache"], [8], None)
    assert e.value.status == MOT_ERR_NO_SAVED_STATE


def test_backward_2048sq_train_full(cuda_ready):
    # the training workload at full size: 2048^2 (4096 image tokens), 400 cached
    # keys, LoRA r32 on q/k/v/o; every output element compared
    wl = synth.WORKLOADS[4]
    t = synth.workload_inputs(4)
    dx, dx32, d_a, d_b, status, _ = run_backward(wl, t)
    assert status == 0
    check_all(wl, t, dx, dx32, d_a, d_b, oracle_backward(wl, t))


def test_backward_on_caller_stream(cuda_ready):
    # forward and backward issued on a caller-created stream: the layer's side
    # stream work (LoRA gradients) must be joined back into that stream, so
    # synchronising the caller's stream alone (not the device) is enough to
    # read every output, and the results equal a default-stream run bit for bit
    wl = synth.Workload("train_1024sq_b1", 1, 1024, 400, 32, 32.0, train=True)
    t = synth.make_inputs(wl, 4100, with_dy=True)
    dx_ref, dx32_ref, da_ref, db_ref, st, layer = run_backward(wl, t)
    assert st == 0
    td = to_dev(t)
    pl = [int(v) for v in t["prefix_len"]]
    x = td["x"]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        sv = layer.new_saved(*x.shape[:2], td["k_cache"].shape[2])
        layer.forward(x, td["k_cache"], td["v_cache"], pl, y=torch.empty_like(x), saved=sv, stream=s)
        dx = torch.empty_like(x)
        dx32 = torch.empty(x.shape, dtype=torch.float32, device="cuda")
        d_a = [torch.zeros(td["a_" + n].shape, device="cuda") for n in NAMES]
        d_b = [torch.zeros(td["b_" + n].shape, device="cuda") for n in NAMES]
        layer.backward(td["dy"], x, td["k_cache"], td["v_cache"], pl, sv, dx=dx, dx_f32=dx32, d_a=d_a,
                       d_b=d_b, stream=s)
        host = [v.cpu() for v in [dx32] + d_a + d_b]  # copies ordered on s only
    s.synchronize()
    assert layer.device_status(stream=s) == 0
    for got, ref in zip(host, [dx32_ref] + da_ref + db_ref):
        assert torch.equal(got.view(torch.int32), ref.cpu().view(torch.int32))


@pytest.mark.parametrize("hidden,hq,hkv", [(512, 4, 4), (1024, 8, 2)])
def test_backward_other_head_groupings(cuda_ready, hidden, hq, hkv):
    # the dk/dv CTAs sum over the query heads of their KV head's group: group
    # sizes 1 and 4 besides the small dims' 2
    dims = synth.LayerDims(hidden=hidden, n_q_heads=hq, n_kv_heads=hkv)
    wl = synth.Workload("groups", 2, 160, 48, 16, 32.0, train=True, dims=dims)
    t = synth.make_inputs(wl, 9600 + hq * 10 + hkv, with_dy=True)
    t["prefix_len"] = torch.tensor([48, 17], dtype=torch.int32)
    dx, dx32, d_a, d_b, status, _ = run_backward(wl, t)
    assert status == 0
    check_all(wl, t, dx, dx32, d_a, d_b, oracle_backward(wl, t))

"""Host-buffer forward (mot_attn_forward_host): several calls whose inputs
and outputs live in host memory, pipelined over two device staging slots on
the handle's copy streams. Every call's output must equal, bit for bit, a
device-buffer forward of the same inputs; pinned and pageable host memory
and calls without a prefix cache are covered."""
import pytest
import torch

from mot_flow_matching_b200 import synth
from tests.gpu_helpers import make_layer, to_dev

pytestmark = pytest.mark.gpu


def _inputs(wl, seeds):
    return [synth.make_inputs(wl, s) for s in seeds]


def _device_outputs(layer, ts):
    ys = []
    for t in ts:
        td = to_dev(t)
        P = td["k_cache"].shape[2]
        y = layer.forward(td["x"], td["k_cache"] if P else None, td["v_cache"] if P else None,
                          [int(v) for v in t["prefix_len"]])
        torch.cuda.synchronize()
        ys.append(y.cpu())
    return ys


def _host_run(layer, ts, pinned):
    def host(a):
        a = a.contiguous().clone()
        return a.pin_memory() if pinned else a
    xs = [host(t["x"]) for t in ts]
    P = ts[0]["k_cache"].shape[2]
    kcs = [host(t["k_cache"]) for t in ts] if P else None
    vcs = [host(t["v_cache"]) for t in ts] if P else None
    ys = [torch.full_like(x, float("nan")) for x in xs]
    if pinned:
        ys = [y.pin_memory() for y in ys]
    layer.forward_host(xs, kcs, vcs, [int(v) for v in ts[0]["prefix_len"]], ys)
    torch.cuda.current_stream().synchronize()  # the caller's stream alone covers every copy-out
    assert layer.device_status() == 0
    return ys


@pytest.mark.parametrize("pinned", [True, False])
def test_forward_host_matches_device_forward(cuda_ready, pinned):
    wl = synth.WORKLOADS[1]  # 1024^2 CFG: B=2, N=1024, P=400, r=32
    ts = _inputs(wl, [11, 12, 13, 14, 15])
    for t in ts[1:]:
        t["prefix_len"] = ts[0]["prefix_len"]  # one prefix_len array for all calls
    layer = make_layer(wl, to_dev(ts[0]))
    ref = _device_outputs(layer, ts)
    got = _host_run(layer, ts, pinned)
    for i, (a, b) in enumerate(zip(got, ref)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), f"call {i}"


def test_forward_host_without_cache_and_single_call(cuda_ready):
    dims = synth.LayerDims(hidden=512, n_q_heads=4, n_kv_heads=2)
    wl = synth.Workload("small", 2, 200, 0, 16, 16.0, dims=dims)
    ts = _inputs(wl, [21, 22, 23])
    layer = make_layer(wl, to_dev(ts[0]))
    ref = _device_outputs(layer, ts)
    got = _host_run(layer, ts, pinned=True)
    for a, b in zip(got, ref):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    one = _host_run(layer, ts[2:], pinned=True)
    assert torch.equal(one[0].view(torch.int16), ref[2].view(torch.int16))


def test_forward_host_rejects_small_staging(cuda_ready):
    from mot_flow_matching_b200._abi import MOT_ERR_WORKSPACE_TOO_SMALL, MotError
    dims = synth.LayerDims(hidden=512, n_q_heads=4, n_kv_heads=2)
    wl = synth.Workload("small", 1, 64, 8, 0, 0.0, dims=dims)
    t = synth.make_inputs(wl, 5)
    layer = make_layer(wl, to_dev(t))
    staging = layer.host_staging(1, 64, 8)
    with pytest.raises(MotError) as e:
        layer.forward_host([t["x"]], [t["k_cache"]], [t["v_cache"]], [8], [torch.empty_like(t["x"])],
                           staging=staging[:-256])
    assert e.value.status == MOT_ERR_WORKSPACE_TOO_SMALL

"""Ordering of the library's kernels when calls follow one another on one
stream with no host synchronisation. Consecutive kernels are launched so that
the next one's prologue overlaps the previous one's tail; every kernel waits
for the previous grid before its first global access. A chain whose input is
the previous call's output (two stacked layers, then a backward through the
second) must therefore give bit for bit what the same calls give with the
host synchronising after each one."""
import pytest
import torch

from mot_flow_matching_b200 import synth
from mot_flow_matching_b200.layer import mot_dev_profile, mot_dev_stage_timeline, mot_dev_stage_times
from tests.gpu_helpers import make_layer, to_dev

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "o")


def _chain(layer, td, pl, sync):
    x = td["x"]
    y1 = torch.empty_like(x)
    y2 = torch.empty_like(x)
    B, N, _ = x.shape
    P = td["k_cache"].shape[2]
    sv = layer.new_saved(B, N, P)
    d_a = [torch.zeros(td["a_" + n].shape, device="cuda") for n in NAMES]
    d_b = [torch.zeros(td["b_" + n].shape, device="cuda") for n in NAMES]
    dx = torch.empty_like(x)
    dx32 = torch.empty(x.shape, dtype=torch.float32, device="cuda")

    def barrier():
        if sync:
            torch.cuda.synchronize()

    layer.forward(x, td["k_cache"], td["v_cache"], pl, y=y1)
    barrier()
    # the second layer call reads the first one's output as its input
    layer.forward(y1, td["k_cache"], td["v_cache"], pl, y=y2, saved=sv)
    barrier()
    # gradient of the second call, with its own output standing in for dy
    layer.backward(y2, y1, td["k_cache"], td["v_cache"], pl, sv, dx=dx, dx_f32=dx32, d_a=d_a, d_b=d_b)
    barrier()
    # and the first call again, overwriting y1 right after the backward read it
    layer.forward(x, td["k_cache"], td["v_cache"], pl, y=y1)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    return [t.clone() for t in [y1, y2, dx, dx32] + d_a + d_b]


def test_chained_calls_without_host_sync_match_synchronised(cuda_ready):
    wl = synth.Workload("train_1024sq_b1", 1, 1024, 400, 32, 32.0, train=True)
    t = synth.make_inputs(wl, 4200, with_dy=True)
    td = to_dev(t)
    layer = make_layer(wl, td, backward=True)
    pl = [int(v) for v in t["prefix_len"]]
    ref = _chain(layer, td, pl, sync=True)
    for _ in range(3):
        got = _chain(layer, td, pl, sync=False)
        for a, b in zip(got, ref):
            assert torch.equal(a.view(torch.int16) if a.element_size() == 2 else a.view(torch.int32),
                               b.view(torch.int16) if b.element_size() == 2 else b.view(torch.int32))


def test_stage_timeline_is_consistent_with_stage_times(cuda_ready):
    wl = synth.Workload("train_1024sq_b1", 1, 1024, 400, 32, 32.0, train=True)
    t = synth.make_inputs(wl, 4300, with_dy=True)
    td = to_dev(t)
    layer = make_layer(wl, td, backward=True)
    pl = [int(v) for v in t["prefix_len"]]
    x = td["x"]
    sv = layer.new_saved(1, wl.img_tokens, wl.prefix)
    d_a = [torch.zeros(td["a_" + n].shape, device="cuda") for n in NAMES]
    d_b = [torch.zeros(td["b_" + n].shape, device="cuda") for n in NAMES]
    layer.forward(x, td["k_cache"], td["v_cache"], pl, saved=sv)
    mot_dev_profile(layer.handle, True)
    layer.backward(td["dy"], x, td["k_cache"], td["v_cache"], pl, sv, d_a=d_a, d_b=d_b)
    times = mot_dev_stage_times(layer.handle)
    line = mot_dev_stage_timeline(layer.handle)
    mot_dev_profile(layer.handle, False)
    torch.cuda.synchronize()
    assert [n for n, _ in times] == [n for n, _, _ in line]
    assert "attn_bwd" in [n for n, _ in times]
    assert line[0][1] == 0.0
    for (n, ms), (_, t0, t1) in zip(times, line):
        assert t0 >= 0.0 and t1 >= t0
        assert t1 - t0 == pytest.approx(ms, abs=2e-3)
    # main-stream launches follow one another: each starts where the previous main launch ended
    main = [(t0, t1) for n, t0, t1 in line if n in ("bwd_cvt_lora", "bwd_g_o", "bwd_do_gemm", "attn_bwd")]
    for (a0, a1), (b0, b1) in zip(main, main[1:]):
        assert b0 == pytest.approx(a1, abs=1e-3)

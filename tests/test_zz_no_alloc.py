"""The forward that allocates nothing (mot_attn_forward_noalloc) against the
ordinary forward with a caller workspace.

It serves callers that cannot allocate device memory per call (plug-ins in
hosts that own all device memory, latency-critical loops where cudaMalloc's
implicit synchronisation is not acceptable). Its scratch is one fixed device
array inside the library, shared by every call; this file is collected last
so that a failure here stops a -x run only after every other test has run.
"""
import pytest
import torch

from mot_flow_matching_b200 import synth
from mot_flow_matching_b200._abi import MOT_ERR_WORKSPACE_TOO_SMALL, MotError
from mot_flow_matching_b200.layer import mot_attn_forward_noalloc
from tests.gpu_helpers import bf16_is_rne_of_f32, make_layer, to_dev

pytestmark = pytest.mark.gpu


def test_noalloc_forward_matches_workspace_forward_twice(cuda_ready):
    wl = synth.WORKLOADS[0]  # 512^2, one branch, 256 image tokens, 64 cached keys, LoRA r16
    td = to_dev(synth.workload_inputs(0))
    layer = make_layer(wl, td)
    B, N, P = wl.batch, wl.img_tokens, wl.prefix
    pl = [int(v) for v in td["prefix_len"]]
    ref32 = torch.empty(B, N, wl.dims.hidden, dtype=torch.float32, device="cuda")
    ref = layer.forward(td["x"], td["k_cache"], td["v_cache"], pl, y_f32=ref32)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    for _ in range(2):  # the second call runs on the scratch the first one left behind
        y = torch.full_like(td["x"], float("nan"))
        y32 = torch.full((B, N, wl.dims.hidden), float("nan"), dtype=torch.float32, device="cuda")
        mot_attn_forward_noalloc(layer.handle, td["x"], B, N, td["k_cache"], td["v_cache"], pl, P, y, y32)
        torch.cuda.synchronize()
        assert layer.device_status() == 0
        # the same kernels on the same inputs, only at another scratch
        # address: the results must agree bit for bit (a stale read of the
        # shared array or a race in it would show here)
        assert torch.equal(y32.view(torch.int32), ref32.view(torch.int32))
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
        assert bf16_is_rne_of_f32(y, y32)


def test_noalloc_forward_rejects_shapes_beyond_its_scratch(cuda_ready):
    wl = synth.WORKLOADS[1]  # 1024^2 CFG: two branches of 1024 tokens need ~46 MiB of scratch
    t = synth.workload_inputs(1)
    td = to_dev(t)
    layer = make_layer(wl, td)
    y = torch.empty_like(td["x"])
    with pytest.raises(MotError) as e:
        mot_attn_forward_noalloc(layer.handle, td["x"], wl.batch, wl.img_tokens, td["k_cache"], td["v_cache"],
                                 [int(v) for v in t["prefix_len"]], wl.prefix, y)
    assert e.value.status == MOT_ERR_WORKSPACE_TOO_SMALL

"""Failure detection without a GPU fault: a kernel whose one wait is on a
barrier nothing completes gives up after the bounded-wait limit, the timeout
is reported by the next status query (and cleared by it), and the handle and
the context stay usable -- the next forward reproduces the earlier output bit
for bit."""
import pytest
import torch

from mot_flow_matching_b200 import synth
from mot_flow_matching_b200._abi import MOT_ERR_TIMEOUT, MOT_OK
from mot_flow_matching_b200.layer import mot_dev_wait_probe
from tests.gpu_helpers import make_layer, run_forward, to_dev

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_the_context_stays_usable(cuda_ready):
    dims = synth.LayerDims(hidden=512, n_q_heads=4, n_kv_heads=2)
    wl = synth.Workload("small", 2, 160, 40, 16, 16.0, dims=dims)
    td = to_dev(synth.make_inputs(wl, 9100))
    layer = make_layer(wl, td)
    y0, y0_32, _, status = run_forward(layer, td)
    assert status == MOT_OK
    mot_dev_wait_probe(layer.handle)
    assert layer.device_status() == MOT_ERR_TIMEOUT
    assert layer.device_status() == MOT_OK  # the query cleared it
    y1, y1_32, _, status = run_forward(layer, td)
    assert status == MOT_OK
    assert torch.equal(y1.view(torch.int16), y0.view(torch.int16))
    assert torch.equal(y1_32.view(torch.int32), y0_32.view(torch.int32))

"""Split-KV attention forward on the GPU: the key range of every (branch,
head, query pair) cut into S contiguous ranges, one CTA each, merged through
distributed shared memory. For S in {1, 2, 3, 7} (forced through
mot_dev_set_attn_splits) the layer output, the attention output and the LSE
are compared with the single pass (S = 1, f32 summation-order error) and the
layer output with the oracle (the parity bar). The oracle's own merge rule is
pinned in test_oracle_split_kv_pins.py."""
import numpy as np
import pytest
import torch

from mot_flow_matching_b200 import synth
from mot_flow_matching_b200._abi import MOT_ERR_UNSUPPORTED_SHAPE, MotError
from mot_flow_matching_b200.layer import (mot_dev_last_attn_full_units, mot_dev_last_attn_splits,
                                          mot_dev_saved_layout, mot_dev_set_attn_splits)
from oracle import mot_attn_oracle as O
from tests.gpu_helpers import assert_parity, bf16_is_rne_of_f32, make_layer, oracle_forward, run_forward, to_dev

pytestmark = pytest.mark.gpu

SMALL = dict(hidden=512, n_q_heads=4, n_kv_heads=2)


def _attn_and_lse(layer, sv, B, N, P, Hq):
    offs, _ = mot_dev_saved_layout(layer.cfg, B, N, P)
    n = B * N * Hq * 128
    attn = sv[offs[3]:offs[3] + 2 * n].view(torch.float16).view(B, N, Hq * 128).double().cpu().numpy()
    m = B * Hq * N
    lse = sv[offs[4]:offs[4] + 4 * m].view(torch.float32).view(B, Hq, N).double().cpu().numpy()
    return attn, lse


def _run_splits(wl, t, splits_list):
    td = to_dev(t)
    layer = make_layer(wl, td, backward=True)
    out = {}
    for S in splits_list:
        mot_dev_set_attn_splits(layer.handle, S)
        y, y32, sv, status = run_forward(layer, td, saved=True)
        assert status == 0
        assert mot_dev_last_attn_splits(layer.handle) == S
        attn, lse = _attn_and_lse(layer, sv, wl.batch, wl.img_tokens, wl.prefix, wl.dims.n_q_heads)
        out[S] = (y.clone(), y32.clone(), attn, lse)
    return layer, out


def _check_against_single_pass(out, splits_list):
    y1, y32_1, attn1, lse1 = out[1]
    amax = np.abs(attn1).max()
    for S in splits_list:
        y, y32, attn, lse = out[S]
        # f16 attention output: the split changes only the f32 summation order
        # (and the running max each range's f16 probabilities are taken
        # against), so it stays within a couple of f16 roundings
        np.testing.assert_allclose(attn, attn1, rtol=0, atol=4e-3 * amax, err_msg=f"S={S} attention output")
        assert np.mean(np.abs(attn - attn1)) <= 2e-4 * amax, S
        np.testing.assert_allclose(lse, lse1, rtol=0, atol=2e-4, err_msg=f"S={S} lse")
        assert_parity(y32.double().cpu().numpy(), y32_1.double().cpu().numpy(), f"S={S} y vs single pass",
                      max_tol=3e-3, mean_tol=3e-4)
        assert bf16_is_rne_of_f32(y, y32)


def test_split_kv_512sq(cuda_ready):
    # 512^2 workload: 64 cached + 256 image keys = 3 key tiles
    wl = synth.WORKLOADS[0]
    t = synth.workload_inputs(0)
    splits = [1, 2, 3]
    layer, out = _run_splits(wl, t, splits)
    _check_against_single_pass(out, splits)
    ref = oracle_forward(wl, t, keep=True)
    br = ref["branches"][0]
    for S in splits:
        assert_parity(out[S][1].double().cpu().numpy(), ref["y"], f"S={S} y f32 vs oracle")
        assert_parity(out[S][2][0], br["attn"], f"S={S} attention output vs oracle")
        np.testing.assert_allclose(out[S][3][0], br["lse"], rtol=0, atol=2e-3 * np.abs(br["lse"]).max())
    # more splits than the shortest branch has key tiles: refused before any launch
    mot_dev_set_attn_splits(layer.handle, 4)
    with pytest.raises(MotError) as e:
        run_forward(layer, to_dev(t))
    assert e.value.status == MOT_ERR_UNSUPPORTED_SHAPE
    layer.close()


def test_split_kv_ragged_small_dims(cuda_ready):
    # two branches of different key counts (1200 and 900 keys: 10 and 8 key
    # tiles, the last ones ragged), poisoned cache rows past prefix_len
    dims = synth.LayerDims(**SMALL)
    wl = synth.Workload("small", 2, 900, 300, 16, 32.0, dims=dims)
    t = synth.make_inputs(wl, 5151, with_dy=False)
    t["prefix_len"] = torch.tensor([300, 0], dtype=torch.int32)
    t["k_cache"][1] = 3e4
    t["v_cache"][1] = -3e4
    splits = [1, 2, 3, 7]
    layer, out = _run_splits(wl, t, splits)
    _check_against_single_pass(out, splits)
    ref = oracle_forward(wl, t, keep=True)
    for S in splits:
        assert_parity(out[S][1].double().cpu().numpy(), ref["y"], f"S={S} y f32 vs oracle")
        for b in range(2):
            br = ref["branches"][b]
            np.testing.assert_allclose(out[S][3][b], br["lse"], rtol=0, atol=2e-3 * np.abs(br["lse"]).max())
    # the oracle's own split merge at the kernel's cut points (whole 128-key
    # tiles, ranges split*T/S) equals its single pass on this data
    br = ref["branches"][0]
    T = (300 + 900 + 127) // 128
    bounds = [(s * T // 7) * 128 for s in range(1, 7)]
    o_split, lse_split = O.gqa_attention_split_kv(br["q_rot"], br["k_all"], br["v_all"], bounds)
    np.testing.assert_allclose(o_split, br["o"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse_split, br["lse"], rtol=0, atol=1e-12)
    layer.close()


def test_split_kv_deterministic_and_planned(cuda_ready):
    wl = synth.WORKLOADS[0]
    td = to_dev(synth.workload_inputs(0))
    layer = make_layer(wl, td)
    mot_dev_set_attn_splits(layer.handle, 3)
    a = run_forward(layer, td)[1].clone()
    b = run_forward(layer, td)[1]
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    # back to the planner: it picks a split count the shape allows
    mot_dev_set_attn_splits(layer.handle, 0)
    c = run_forward(layer, td)[1]
    assert 1 <= mot_dev_last_attn_splits(layer.handle) <= 3
    assert torch.isfinite(c).all()
    layer.close()


def test_planned_tail_split(cuda_ready):
    # 2 branches x 4 heads x 20 query pairs = 160 units: one full wave of 148
    # CTAs and a tail of 12 units, which the planner runs split (a second
    # launch of clusters); the result must match the unsplit forward and the
    # oracle
    dims = synth.LayerDims(**SMALL)
    wl = synth.Workload("small", 2, 5120, 200, 16, 16.0, dims=dims)
    t = synth.make_inputs(wl, 6262, with_dy=False)
    t["prefix_len"] = torch.tensor([200, 150], dtype=torch.int32)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    units = 2 * 4 * 20
    td = to_dev(t)
    layer = make_layer(wl, td, backward=True)
    y, y32, sv, status = run_forward(layer, td, saved=True)
    assert status == 0
    full, S = mot_dev_last_attn_full_units(layer.handle), mot_dev_last_attn_splits(layer.handle)
    if units % sms:
        assert full == (units // sms) * sms and S > 1, (full, S)
    attn, lse = _attn_and_lse(layer, sv, 2, 5120, 200, 4)
    mot_dev_set_attn_splits(layer.handle, 1)
    y1, y32_1, sv1, status = run_forward(layer, td, saved=True)
    assert status == 0 and mot_dev_last_attn_full_units(layer.handle) == 0
    attn1, lse1 = _attn_and_lse(layer, sv1, 2, 5120, 200, 4)
    np.testing.assert_allclose(attn, attn1, rtol=0, atol=4e-3 * np.abs(attn1).max())
    np.testing.assert_allclose(lse, lse1, rtol=0, atol=2e-4)
    # the units of the full waves ran unsplit in both calls: bit for bit the
    # same (units are ordered branch, head, query pair)
    for u in range(full):
        b, h, qp = u // 80, (u // 20) % 4, u % 20
        blk = (b, slice(qp * 256, qp * 256 + 256), slice(h * 128, h * 128 + 128))
        assert np.array_equal(attn[blk], attn1[blk]), u
    rows = [np.concatenate([np.arange(0, 256), np.arange(5120 - 300, 5120)]) for _ in range(2)]
    ref = oracle_forward(wl, t, rows=rows)
    got = np.concatenate([y32[b].double().cpu().numpy()[rows[b]] for b in range(2)])
    assert_parity(got, np.concatenate(ref["y"]), "y f32 (tail split) vs oracle")
    assert bf16_is_rne_of_f32(y, y32)
    layer.close()

"""Forward parity of the CUDA layer (through the C ABI) against the oracle,
on seeded synth inputs: full outputs for the 512^2, 1024^2 and 2048^2 CFG
workloads and small-dim ragged cases, sampled query rows (>= 256 per branch)
for the 2048^2 edit workload, per-stage checks of the saved activations, and
the method's invariants on the GPU."""
import numpy as np
import pytest
import torch

from mot_flow_matching_b200 import synth
from mot_flow_matching_b200.layer import mot_dev_saved_layout
from oracle import mot_attn_oracle as O
from tests.gpu_helpers import (assert_parity, bf16_is_rne_of_f32, make_layer, oracle_forward, parity_stats,
                               run_forward, sample_rows, to_dev)

pytestmark = pytest.mark.gpu


def _f16(buf, off, shape):
    n = int(np.prod(shape))
    return buf[off:off + 2 * n].view(torch.float16).view(*shape).double().cpu().numpy()


def _f32(buf, off, shape):
    n = int(np.prod(shape))
    return buf[off:off + 4 * n].view(torch.float32).view(*shape).double().cpu().numpy()


def test_fwd_512sq_full_and_stages(cuda_ready):
    wl = synth.WORKLOADS[0]
    t = synth.workload_inputs(0)
    td = to_dev(t)
    layer = make_layer(wl, td, backward=True)
    y, y32, sv, status = run_forward(layer, td, saved=True)
    assert status == 0
    ref = oracle_forward(wl, t, keep=True)
    br = ref["branches"][0]
    offs, lcap = mot_dev_saved_layout(layer.cfg, 1, wl.img_tokens, wl.prefix)
    N, P, Hq, Hkv = wl.img_tokens, wl.prefix, 32, 8
    q_hat = _f16(sv, offs[0], (1, Hq, N, 128))[0]
    assert_parity(q_hat, br["q_rot"], "q^")
    k_all = _f16(sv, offs[1], (1, Hkv, lcap, 128))[0]
    v_all = _f16(sv, offs[2], (1, Hkv, lcap, 128))[0]
    # prefix rows are the cache rounded to f16 (exact except f16 subnormals);
    # self rows are the projection
    np.testing.assert_array_equal(k_all[:, :P], t["k_cache"][0].to(torch.float16).double().numpy())
    np.testing.assert_array_equal(v_all[:, :P], t["v_cache"][0].to(torch.float16).double().numpy())
    assert_parity(k_all[:, P:P + N], br["k_all"][:, P:], "k^ self")
    assert_parity(v_all[:, P:P + N], br["v_all"][:, P:], "v self")
    assert np.all(k_all[:, P + N:] == 0) and np.all(v_all[:, P + N:] == 0)
    attn = _f16(sv, offs[3], (N, Hq * 128))
    assert_parity(attn, br["attn"], "attention output")
    lse = _f32(sv, offs[4], (1, Hq, N))[0]
    np.testing.assert_allclose(lse, br["lse"], rtol=0, atol=2e-3 * np.abs(br["lse"]).max())
    assert_parity(y32.double().cpu().numpy(), ref["y"], "y f32")
    assert bf16_is_rne_of_f32(y, y32)
    # build_kv (+ LoRA f16 copies), LoRA-down qkv, QKV GEMM, attention, LoRA-down o, O GEMM
    assert layer.last_launch_count() == 6


def test_fwd_1024sq_cfg_full(cuda_ready):
    wl = synth.WORKLOADS[1]
    t = synth.workload_inputs(1)
    td = to_dev(t)
    layer = make_layer(wl, td)
    y, y32, _, status = run_forward(layer, td)
    assert status == 0
    ref = oracle_forward(wl, t)
    assert_parity(y32.double().cpu().numpy(), ref["y"], "y f32")
    assert bf16_is_rne_of_f32(y, y32)
    # bf16 output vs oracle: reported bound (bf16 rounding alone ~ 1.6e-2 RMS max)
    mx, mean = parity_stats(y.double().cpu().numpy(), ref["y"])
    assert mean < 3e-3 and mx < 3e-2


def test_fwd_2048sq_cfg_full(cuda_ready):
    # every element of the 2 x 4096 x 4096 output against the oracle
    wl = synth.WORKLOADS[2]
    t = synth.workload_inputs(2)
    td = to_dev(t)
    layer = make_layer(wl, td)
    y, y32, _, status = run_forward(layer, td)
    assert status == 0
    ref = oracle_forward(wl, t)
    assert_parity(y32.double().cpu().numpy(), ref["y"], "y f32")
    assert bf16_is_rne_of_f32(y, y32)


def test_fwd_2048sq_edit_merged_sampled_rows(cuda_ready):
    wl = synth.WORKLOADS[3]
    t = synth.workload_inputs(3)
    td = to_dev(t)
    layer = make_layer(wl, td)
    s = wl.lora_alpha / wl.lora_rank
    merged = {n: torch.empty_like(td["w_" + n]) for n in ("q", "k", "v", "o")}
    layer.merge_lora(merged["q"], merged["k"], merged["v"], merged["o"])
    torch.cuda.synchronize()
    # merged weights: nearest bf16 of W + s B A (f32 on the GPU, f64 in the oracle)
    t64 = O.to_f64(t)
    oracle_merged = {}
    for n in ("q", "k", "v", "o"):
        om = O.merge_lora(t64["w_" + n], t64["a_" + n], t64["b_" + n], s)
        oracle_merged[n] = om
        gm = merged[n].double().cpu().numpy()
        diff = gm != om
        _, e = np.frexp(om)
        ulp = np.ldexp(1.0, e - 8)
        # one bf16 ulp, plus the f32 error of the rank-32 sum where W + s B A
        # cancels to nearly zero (there a bf16 ulp is smaller than that error)
        f32_err = 2.0**-22 * (np.abs(t64["b_" + n]) @ np.abs(t64["a_" + n]) * s + np.abs(t64["w_" + n]))
        bad = np.abs(gm - om) > ulp + f32_err
        assert not bad.any(), (n, int(bad.sum()), gm[bad][:4], om[bad][:4])
        assert diff.mean() < 1e-3, (n, diff.mean())
    y, y32, _, status = run_forward(layer, td)
    assert status == 0
    tm = {k: v for k, v in t.items() if not k.startswith(("a_", "b_"))}
    # 384 random query rows per branch plus the first and last (all keys and
    # values of every branch projected in full)
    rows = [sample_rows(wl.img_tokens, 384, 30 + b) for b in range(wl.batch)]
    assert all(len(r) >= 256 for r in rows)
    tm64 = O.to_f64(tm)
    for n in ("q", "k", "v", "o"):
        tm64["w_" + n] = oracle_merged[n]
    ref = O.layer_forward(tm64, O.dims_of(wl), 0.0, query_rows=rows)
    got = np.concatenate([y32[b].double().cpu().numpy()[rows[b]] for b in range(wl.batch)])
    assert_parity(got, np.concatenate(ref["y"]), "y f32 sampled (merged)")


SMALL = dict(hidden=512, n_q_heads=4, n_kv_heads=2)


@pytest.mark.parametrize("batch,n,p,plen,rank", [
    (1, 1, 0, [0], 0),            # one token, no cache
    (2, 200, 37, [37, 20], 16),   # ragged tiles, prefix shorter than P_max
    (3, 129, 128, [0, 128, 5], 8),
    (2, 384, 300, [300, 1], 64),
    (1, 77, 5, [5], 128),
])
def test_fwd_small_dims_ragged(cuda_ready, batch, n, p, plen, rank):
    dims = synth.LayerDims(**SMALL)
    wl = synth.Workload("small", batch, n, p, rank, float(2 * rank), dims=dims)
    t = synth.make_inputs(wl, 9000 + n, with_dy=False)
    t["prefix_len"] = torch.tensor(plen, dtype=torch.int32)
    # rows beyond prefix_len hold values the layer must ignore
    for b, pl in enumerate(plen):
        t["k_cache"][b, :, pl:] = 3e4
        t["v_cache"][b, :, pl:] = -3e4
    td = to_dev(t)
    layer = make_layer(wl, td)
    y, y32, _, status = run_forward(layer, td)
    assert status == 0
    ref = oracle_forward(wl, t)
    assert_parity(y32.double().cpu().numpy(), ref["y"], "y f32")
    assert bf16_is_rne_of_f32(y, y32)


def test_zero_lora_up_is_bitwise_rank0(cuda_ready):
    wl = synth.WORKLOADS[0]
    t = synth.workload_inputs(0)
    td = to_dev(t)
    for n in ("q", "k", "v", "o"):
        td["b_" + n] = torch.zeros_like(td["b_" + n])
    y_lora = run_forward(make_layer(wl, td), td)[1]
    td0 = {k: v for k, v in td.items() if not k.startswith(("a_", "b_"))}
    y_base = run_forward(make_layer(wl, td0), td0)[1]
    assert torch.equal(y_lora.view(torch.int32), y_base.view(torch.int32))


def test_zero_query_gives_mean_of_values(cuda_ready):
    dims = synth.LayerDims(**SMALL)
    wl = synth.Workload("small", 2, 300, 100, 0, 0.0, dims=dims)
    t = synth.make_inputs(wl, 4242, with_dy=False)
    t["w_q"] = torch.zeros_like(t["w_q"])
    td = to_dev(t)
    layer = make_layer(wl, td, backward=True)
    _, _, sv, status = run_forward(layer, td, saved=True)
    assert status == 0
    offs, lcap = mot_dev_saved_layout(layer.cfg, 2, 300, 100)
    attn = _f16(sv, offs[3], (2, 300, 4, 128))
    ref = oracle_forward(wl, t, keep=True)
    for b in range(2):
        v_all = ref["branches"][b]["v_all"]
        for h in range(4):
            mean_v = v_all[h // 2].mean(0)
            np.testing.assert_allclose(attn[b, :, h], np.broadcast_to(mean_v, (300, 128)), rtol=0,
                                       atol=2e-3 * np.abs(mean_v).max() + 1e-3)


def test_deterministic(cuda_ready):
    wl = synth.WORKLOADS[0]
    td = to_dev(synth.workload_inputs(0))
    layer = make_layer(wl, td)
    a = run_forward(layer, td)[1].clone()
    b = run_forward(layer, td)[1]
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))


def test_f16_overflow_is_reported(cuda_ready):
    dims = synth.LayerDims(**SMALL)
    wl = synth.Workload("small", 1, 64, 16, 0, 0.0, dims=dims)
    t = synth.make_inputs(wl, 77, with_dy=False)
    t["v_cache"][0, 0, 3, 5] = 1e6   # beyond the f16 range
    td = to_dev(t)
    layer = make_layer(wl, td)
    _, _, _, status = run_forward(layer, td)
    assert status == 7  # MOT_ERR_NUMERIC
    _, _, _, status = run_forward(layer, to_dev(synth.make_inputs(wl, 78, with_dy=False)))
    assert status == 0


@pytest.mark.parametrize("hidden,hq,hkv", [
    (512, 4, 4),     # no grouping: plain multi-head attention
    (1024, 8, 2),    # a group of 4 query heads per KV head, as the full layer
])
def test_fwd_other_head_groupings(cuda_ready, hidden, hq, hkv):
    # the KV head of query head h is h / (Hq / Hkv): other group sizes than
    # the small dims' 2 and the full layer's 4-of-32
    dims = synth.LayerDims(hidden=hidden, n_q_heads=hq, n_kv_heads=hkv)
    wl = synth.Workload("groups", 2, 160, 48, 16, 32.0, dims=dims)
    t = synth.make_inputs(wl, 9500 + hq * 10 + hkv, with_dy=False)
    t["prefix_len"] = torch.tensor([48, 17], dtype=torch.int32)
    td = to_dev(t)
    layer = make_layer(wl, td)
    y, y32, _, status = run_forward(layer, td)
    assert status == 0
    ref = oracle_forward(wl, t)
    assert_parity(y32.double().cpu().numpy(), ref["y"], f"y f32 (Hq {hq}, Hkv {hkv})")
    assert bf16_is_rne_of_f32(y, y32)


def test_fwd_1536x2720_cfg_full(cuda_ready):
    # the pages' measured end-to-end image size, 1536 x 2720: 48 x 85 patch
    # tokens = 4080 per branch, not a multiple of the 256-query unit or the
    # 128-key tile, at the full layer dims with CFG over 400 cached keys
    # (branch 1 with a 231-token prompt); every output element compared
    wl = synth.Workload("fwd_1536x2720_cfg2", 2, 4080, 400, 32, 32.0)
    t = synth.make_inputs(wl, 6100, with_dy=False)
    t["prefix_len"] = torch.tensor([400, 231], dtype=torch.int32)
    td = to_dev(t)
    layer = make_layer(wl, td)
    y, y32, _, status = run_forward(layer, td)
    assert status == 0
    ref = oracle_forward(wl, t)
    assert_parity(y32.double().cpu().numpy(), ref["y"], "y f32")
    assert bf16_is_rne_of_f32(y, y32)

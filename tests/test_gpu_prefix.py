"""The prefix-tower layer that builds the prefix-KV cache
(mot_attn_prefix_forward) against its fp64 oracle (oracle/mot_prefix_oracle.py):
causal attention over the prompt, the layer output and the bf16 cache entry,
on the full layer dims and on small ragged shapes; then the cache it builds
fed to the gen-tower forward, end to end, against the oracle's pipeline."""
import numpy as np
import pytest
import torch

from mot_flow_matching_b200 import synth
from oracle import mot_attn_oracle as O
from oracle import mot_prefix_oracle as PO
from tests.gpu_helpers import assert_parity, bf16_is_rne_of_f32, make_layer, oracle_forward, run_forward, to_dev

pytestmark = pytest.mark.gpu


def _prefix_inputs(B, P, seed, dims=None):
    wl = synth.Workload("prefix", B, P, 0, 0, 0.0, dims=dims or synth.LayerDims())
    t = synth.make_inputs(wl, seed, with_dy=False)
    return wl, {k: t[k] for k in ("x", "w_q", "w_k", "w_v", "w_o", "q_norm", "k_norm")}


def _run(wl, t, lengths):
    td = to_dev(t)
    layer = make_layer(wl, td)
    B, N = wl.batch, wl.img_tokens
    y32 = torch.empty(B, N, wl.dims.hidden, dtype=torch.float32, device="cuda")
    y, kc, vc = layer.prefix_forward(td["x"], lengths, y_f32=y32)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    return layer, td, y, y32, kc, vc


def _check_cache(got_bf16, ref64, lengths, what):
    # one rounding to bf16 of an f32 value that is within f32 error of the
    # fp64 one: at most one bf16 ulp from the oracle's rounded value plus that
    # f32 error, and equal to it almost everywhere. The f32 error is absolute
    # (a K = 4096 dot product accumulates about sqrt(K) 2^-24 sum|x w|, some
    # 1e-4 of the RMS), so near-zero entries, whose ulp is tiny, get the floor
    # tau = 2^-10 RMS. (A max bar relative to the RMS does not fit a bf16
    # result: half an ulp of an element at 4x the RMS is already 1.6e-2 of the
    # RMS.) The mean bar still applies.
    for b, n in enumerate(lengths):
        g = got_bf16[b][:, :n].double().cpu().numpy()
        r = ref64[b][:, :n]
        assert_parity(g, r, f"{what} branch {b}", max_tol=np.inf, mean_tol=2e-3)
        rb = PO.cache_bf16(r)
        _, e = np.frexp(r)
        ulp = np.ldexp(1.0, e - 8)
        tau = 2.0 ** -10 * np.sqrt(np.mean(r * r))
        bad = np.abs(g - rb) > ulp * 1.0001 + tau
        if bad.any():
            i = np.unravel_index(np.argmax(np.abs(g - rb) - ulp), g.shape)
            raise AssertionError(f"{what} branch {b}: {int(bad.sum())} entries off by more than one ulp + tau; "
                                 f"worst at {i}: got {g[i]!r} oracle {r[i]!r} rounded {rb[i]!r} tau {tau:.3e}")
        assert np.mean(g != rb) < 0.01, (what, np.mean(g != rb))


def test_prefix_forward_full_dims(cuda_ready):
    wl, t = _prefix_inputs(2, 400, 5000)
    lengths = [400, 237]
    layer, td, y, y32, kc, vc = _run(wl, t, lengths)
    ref = PO.prefix_forward(O.to_f64(t), O.dims_of(wl), lengths)
    for b, n in enumerate(lengths):
        assert_parity(y32[b, :n].double().cpu().numpy(), ref["y"][b, :n], f"y f32 branch {b}")
    assert bf16_is_rne_of_f32(y, y32)
    _check_cache(kc, ref["k_cache"], lengths, "k cache")
    _check_cache(vc, ref["v_cache"], lengths, "v cache")
    layer.close()


SMALL = dict(hidden=512, n_q_heads=4, n_kv_heads=2)


@pytest.mark.parametrize("B,N,lengths", [(1, 1, [1]), (2, 77, [77, 1]), (3, 300, [300, 129, 256]), (1, 513, [500])])
def test_prefix_forward_small_dims(cuda_ready, B, N, lengths):
    wl, t = _prefix_inputs(B, N, 5100 + N, synth.LayerDims(**SMALL))
    layer, td, y, y32, kc, vc = _run(wl, t, lengths)
    ref = PO.prefix_forward(O.to_f64(t), O.dims_of(wl), lengths)
    for b, n in enumerate(lengths):
        assert_parity(y32[b, :n].double().cpu().numpy(), ref["y"][b, :n], f"y f32 branch {b}")
    _check_cache(kc, ref["k_cache"], lengths, "k cache")
    _check_cache(vc, ref["v_cache"], lengths, "v cache")
    layer.close()


def test_prefix_forward_is_causal_bitwise(cuda_ready):
    # later tokens never reach earlier rows: changing the tokens from 300 on
    # leaves rows [0, 300) and their cache rows unchanged bit for bit
    wl, t = _prefix_inputs(1, 400, 5200, synth.LayerDims(**SMALL))
    layer, td, y, y32, kc, vc = _run(wl, t, [400])
    t2 = dict(t)
    t2["x"] = t["x"].clone()
    t2["x"][:, 300:] = synth.make_inputs(wl, 5201, with_dy=False)["x"][:, 300:]
    y32b = torch.empty_like(y32)
    _, kcb, vcb = layer.prefix_forward(t2["x"].cuda(), [400], y_f32=y32b)
    torch.cuda.synchronize()
    assert torch.equal(y32[:, :300].view(torch.int32), y32b[:, :300].view(torch.int32))
    assert torch.equal(kc[:, :, :300].view(torch.int16), kcb[:, :, :300].view(torch.int16))
    assert not torch.equal(y32[:, 300:], y32b[:, 300:])
    layer.close()


def test_prefix_cache_feeds_gen_forward_end_to_end(cuda_ready):
    # prompt of 400 tokens (branch 1: 237 real) through the prefix layer, then
    # 1024 image tokens per branch through the gen layer over that cache
    wlp, tp = _prefix_inputs(2, 400, 5300)
    lengths = [400, 237]
    player, _, _, _, kc, vc = _run(wlp, tp, lengths)
    wl = synth.Workload("gen", 2, 1024, 400, 32, 32.0)
    t = synth.make_inputs(wl, 5400, with_dy=False)
    t["prefix_len"] = torch.tensor(lengths, dtype=torch.int32)
    t["k_cache"], t["v_cache"] = kc.cpu(), vc.cpu()
    td = to_dev(t)
    glayer = make_layer(wl, td)
    y, y32, _, status = run_forward(glayer, td)
    assert status == 0
    # the oracle's pipeline: its own prefix cache, rounded to bf16, then its gen layer
    ref_p = PO.prefix_forward(O.to_f64(tp), O.dims_of(wlp), lengths)
    t64 = O.to_f64(t)
    t64["k_cache"] = PO.cache_bf16(ref_p["k_cache"])
    t64["v_cache"] = PO.cache_bf16(ref_p["v_cache"])
    ref = O.layer_forward(t64, O.dims_of(wl), wl.lora_alpha / wl.lora_rank)
    assert_parity(y32.double().cpu().numpy(), ref["y"], "gen y f32 over the GPU-built cache")
    player.close()
    glayer.close()


def test_prefix_forward_refuses_empty_and_overlong_prompts(cuda_ready):
    # a branch with no prompt token (or more than N) has no causal key range:
    # refused on the host before anything is launched; the handle stays usable
    from mot_flow_matching_b200._abi import MOT_ERR_ALIGNMENT, MOT_ERR_INVALID_ARGUMENT, MotError
    from mot_flow_matching_b200.layer import mot_attn_prefix_forward
    wl, t = _prefix_inputs(2, 64, 5500, synth.LayerDims(**SMALL))
    td = to_dev(t)
    layer = make_layer(wl, td)
    for lengths in ([0, 64], [64, 65], [64, -1]):
        with pytest.raises(MotError) as e:
            layer.prefix_forward(td["x"], lengths)
        assert e.value.status == MOT_ERR_INVALID_ARGUMENT, lengths
    y = torch.empty_like(td["x"])
    kc = torch.empty(2 * 2 * 64 * 128 + 8, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(MotError) as e:  # cache output 2 bytes off the 16-byte alignment
        mot_attn_prefix_forward(layer.handle, td["x"], 2, 64, [64, 64], y, kc[1:], kc[1:],
                                workspace=layer.workspace(2, 64, 0))
    assert e.value.status == MOT_ERR_ALIGNMENT
    # still usable
    y, kc2, vc2 = layer.prefix_forward(td["x"], [64, 10])
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    layer.close()

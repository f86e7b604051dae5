"""The A3B gen-tower mixture-of-experts MLP (mot_moe_forward: router GEMM,
top-k routing, dispatch, grouped expert GEMMs on CTA pairs, combine) against
its fp64 oracle (oracle/mot_moe_oracle.py).

Routing is an integer decision taken on f32 logits on the GPU: where the
oracle's k-th and (k+1)-th probabilities are further apart than the f32
error, the GPU's chosen experts must be the oracle's; elsewhere (near ties)
any valid top-k set is correct, so the GPU's set is checked for validity and
the output is compared with the oracle's block evaluated on that set."""
import numpy as np
import pytest
import torch

from mot_flow_matching_b200 import synth
from mot_flow_matching_b200._abi import MOT_ERR_UNSUPPORTED_SHAPE, MotError
from mot_flow_matching_b200.moe import MotMoe
from oracle import mot_moe_oracle as EO
from tests.gpu_helpers import assert_parity, bf16_is_rne_of_f32, ensure_built

pytestmark = pytest.mark.gpu

TIE_TOL = 1e-5  # probability gap below which a top-k choice is a tie at f32


def _run(t, top_k):
    ensure_built()
    td = {k: v.cuda() for k, v in t.items()}
    T = t["x"].shape[0]
    moe = MotMoe({k: td[k] for k in ("w_router", "w_gate", "w_up", "w_down")}, top_k=top_k, max_tokens=T)
    y32 = torch.empty(td["x"].shape, dtype=torch.float32, device="cuda")
    ex = torch.empty(T, top_k, dtype=torch.int32, device="cuda")
    y = moe.forward(td["x"], y_f32=y32, experts_out=ex)
    torch.cuda.synchronize()
    assert moe.device_status() == 0
    return moe, td, y, y32, ex


def _check(t, top_k, y, y32, ex):
    w = {k: v.double().numpy() for k, v in t.items()}
    x = w["x"]
    ref = EO.moe_forward(x, w, top_k)
    p = ref["probs"]
    got_ex = ex.cpu().numpy().astype(np.int64)
    srt = -np.sort(-p, axis=1)
    kth = srt[:, top_k - 1]
    nxt = srt[:, top_k] if top_k < p.shape[1] else np.full(p.shape[0], -1.0)
    clear = (kth - nxt) > TIE_TOL
    # a valid top-k set everywhere; the oracle's set where the choice is clear
    chosen_p = np.take_along_axis(p, got_ex, axis=1)
    assert np.all(chosen_p >= kth[:, None] - TIE_TOL)
    assert np.all(np.sort(got_ex[clear], axis=1) == np.sort(ref["experts"][clear], axis=1))
    # expected output on the GPU's (valid) set: the oracle's block on those experts
    wk = chosen_p / chosen_p.sum(axis=1, keepdims=True)
    exp = np.zeros_like(x)
    for k in range(top_k):
        for e in np.unique(got_ex[:, k]):
            rows = np.nonzero(got_ex[:, k] == e)[0]
            exp[rows] += wk[rows, k][:, None] * EO.expert_forward(x[rows], w, int(e))
    np.testing.assert_allclose(exp[clear], ref["y"][clear], rtol=0, atol=1e-12)
    assert_parity(y32.double().cpu().numpy(), exp, "y f32")
    assert bf16_is_rne_of_f32(y, y32)
    return clear.mean()


@pytest.mark.parametrize("T,E,K", [(1, 8, 2), (77, 8, 8), (300, 16, 4), (513, 32, 8),
                                   (64, 4, 1),     # top-1, exactly one routing block of tokens
                                   (130, 1, 1)])   # one expert: the dense SwiGLU MLP
def test_moe_small_dims(cuda_ready, T, E, K):
    t = synth.make_moe_inputs(T, 256, 128, E, 8100 + T)
    t["w_router"] = (t["w_router"].float() * 8).to(torch.bfloat16)  # a spread of router probabilities
    moe, td, y, y32, ex = _run(t, K)
    _check(t, K, y, y32, ex)
    moe.close()


def test_moe_a3b_dims_1024sq_cfg_tokens(cuda_ready):
    # hidden 2048, 32 experts, top 8, width 768; the 2 x 1024 image tokens of
    # a 1024^2 CFG call
    t = synth.make_moe_inputs(2048, synth.MOE_HIDDEN, synth.MOE_INTER, synth.MOE_EXPERTS, 8200)
    moe, td, y, y32, ex = _run(t, synth.MOE_TOP_K)
    frac_clear = _check(t, synth.MOE_TOP_K, y, y32, ex)
    assert frac_clear > 0.99
    # deterministic: the slots of an expert are in token order, every row of
    # an expert's GEMM is computed on its own and the combine sums in rank
    # order
    y32b = torch.empty_like(y32)
    moe.forward(td["x"], y_f32=y32b)
    torch.cuda.synchronize()
    assert torch.equal(y32.view(torch.int32), y32b.view(torch.int32))
    with pytest.raises(MotError) as e:
        moe.forward(torch.empty(4096, synth.MOE_HIDDEN, dtype=torch.bfloat16, device="cuda"))
    assert e.value.status == MOT_ERR_UNSUPPORTED_SHAPE
    moe.close()

"""Pins for the MoE oracle (oracle/mot_moe_oracle.py): routing against
torch softmax + topk, closed forms at top_k = 1 and top_k = E (the dense
mixture), the block composed from torch library routines, and invariance
under relabelling the experts.

A plausible slip (no renormalisation of the top-k weights, softmax over the
wrong axis, top-k by logits of the wrong sign, gate and up swapped, an
expert's output added with another's weight) fails at least one test here.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from mot_flow_matching_b200 import synth
from oracle import mot_moe_oracle as EO


def _inputs(seed, T=37, d=64, I=48, E=8):
    t = synth.make_moe_inputs(T, d, I, E, seed)
    w = {k: v.double().numpy() for k, v in t.items()}
    w["w_router"] = w["w_router"] * 20  # spread the router's probabilities
    return w


def _torch_block(w, top_k):
    x = torch.from_numpy(w["x"])
    p = torch.softmax(F.linear(x, torch.from_numpy(w["w_router"])), dim=-1)
    val, idx = torch.topk(p, top_k, dim=-1)
    val = val / val.sum(-1, keepdim=True)
    y = torch.zeros_like(x)
    for t in range(x.shape[0]):
        for k in range(top_k):
            e = int(idx[t, k])
            h = F.silu(F.linear(x[t], torch.from_numpy(w["w_gate"][e]))) * F.linear(x[t], torch.from_numpy(w["w_up"][e]))
            y[t] += val[t, k] * F.linear(h, torch.from_numpy(w["w_down"][e]))
    return y.numpy(), idx.numpy(), val.numpy()


@pytest.mark.parametrize("top_k", [1, 3, 8])
def test_block_matches_torch_composition(top_k):
    w = _inputs(1)
    res = EO.moe_forward(w["x"], w, top_k)
    y, idx, val = _torch_block(w, top_k)
    np.testing.assert_allclose(res["y"], y, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(np.sort(res["experts"], axis=1), np.sort(idx, axis=1))
    np.testing.assert_allclose(np.sort(res["weights"], axis=1), np.sort(val, axis=1), rtol=0, atol=1e-14)


def test_routing_weights_and_ties():
    w = _inputs(2)
    ex, wt, p = EO.route(w["x"], w["w_router"], 4)
    np.testing.assert_allclose(wt.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    assert np.all(np.diff(np.take_along_axis(p, ex, axis=1), axis=1) <= 0)  # descending probability
    # equal logits: the lower expert index wins
    ex2, wt2, _ = EO.route(np.zeros((2, 4)), np.zeros((6, 4)), 3)
    np.testing.assert_array_equal(ex2, [[0, 1, 2], [0, 1, 2]])
    np.testing.assert_allclose(wt2, 1 / 3, rtol=0, atol=1e-15)


def test_all_experts_is_the_dense_mixture():
    w = _inputs(3, E=6)
    res = EO.moe_forward(w["x"], w, 6)
    p = res["probs"]
    dense = sum(p[:, e:e + 1] * EO.expert_forward(w["x"], w, e) for e in range(6))
    np.testing.assert_allclose(res["y"], dense, rtol=0, atol=1e-12)


def test_top1_is_the_argmax_expert():
    w = _inputs(4)
    res = EO.moe_forward(w["x"], w, 1)
    best = np.argmax(w["x"] @ w["w_router"].T, axis=1)
    for t in range(w["x"].shape[0]):
        np.testing.assert_allclose(res["y"][t], EO.expert_forward(w["x"][t:t + 1], w, int(best[t]))[0], rtol=0,
                                   atol=1e-13)


def test_relabelling_experts_changes_nothing():
    w = _inputs(5)
    perm = np.random.default_rng(0).permutation(8)
    w2 = dict(w)
    for k in ("w_router", "w_gate", "w_up", "w_down"):
        w2[k] = w[k][perm]
    np.testing.assert_allclose(EO.moe_forward(w["x"], w, 3)["y"], EO.moe_forward(w["x"], w2, 3)["y"], rtol=0,
                               atol=1e-12)


@pytest.mark.parametrize("E,top_k", [(5, 2), (6, 3), (7, 1)])
def test_routing_is_the_heaviest_subset_by_brute_force(E, top_k):
    # over every k-subset of the experts: the routed set is the one with the
    # largest total probability (probabilities drawn distinct, so it is
    # unique), and the weights are that subset's probabilities over their sum
    import itertools
    g = np.random.default_rng(10 + E)
    x, wr = g.standard_normal((9, 4)), 2 * g.standard_normal((E, 4))
    ex, wt, p = EO.route(x, wr, top_k)
    for t in range(x.shape[0]):
        best = max(itertools.combinations(range(E), top_k), key=lambda s: sum(p[t, list(s)]))
        assert set(ex[t]) == set(best)
        for k, e in enumerate(ex[t]):
            assert wt[t, k] == pytest.approx(p[t, e] / sum(p[t, list(best)]), rel=1e-13)
    # the probabilities themselves: softmax written out for one token
    z = x[0] @ wr.T
    np.testing.assert_allclose(p[0], np.exp(z) / np.exp(z).sum(), rtol=1e-13)

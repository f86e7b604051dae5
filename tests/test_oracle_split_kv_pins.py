"""Pins for the oracle's split-KV merge (merge_attention_partials,
gqa_attention_split_kv): the merge of k partials over disjoint key ranges
must give the single-pass attention, checked against torch's
scaled_dot_product_attention and scipy's logsumexp, plus closed forms.

A plausible slip in the merge (averaging the partial outputs, weighting by
exp(lse_s) without the normaliser, taking the max instead of the
log-sum-exp, mixing up which partial a weight belongs to) fails here.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F
from scipy.special import logsumexp

from oracle import mot_attn_oracle as O


def _qkv(seed, hq=4, hkv=2, n=9, length=37, dh=16, scale=1.0):
    g = np.random.default_rng(seed)
    q = g.standard_normal((hq, n, dh)) * scale
    k = g.standard_normal((hkv, length, dh))
    v = g.standard_normal((hkv, length, dh))
    return q, k, v


def _sdpa(q, k, v):
    out = F.scaled_dot_product_attention(torch.from_numpy(q)[None], torch.from_numpy(k)[None],
                                         torch.from_numpy(v)[None], enable_gqa=True)
    return out[0].numpy()


@pytest.mark.parametrize("splits", [1, 2, 3, 7])
def test_split_merge_equals_single_pass(splits):
    q, k, v = _qkv(10 + splits, scale=2.0)
    length = k.shape[1]
    # uneven contiguous ranges (the last one short, like a ragged key tile)
    bounds = sorted(np.random.default_rng(splits).choice(np.arange(1, length), splits - 1, replace=False))
    o, lse = O.gqa_attention_split_kv(q, k, v, bounds)
    np.testing.assert_allclose(o, _sdpa(q, k, v), rtol=0, atol=1e-12)
    s = np.einsum("hnd,hld->hnl", q, np.repeat(k, 2, axis=0)) / np.sqrt(q.shape[-1])
    np.testing.assert_allclose(lse, logsumexp(s, axis=-1), rtol=0, atol=1e-12)


def test_one_partial_is_identity():
    g = np.random.default_rng(3)
    o_s, l_s = g.standard_normal((2, 5, 8)), g.standard_normal((2, 5))
    o, lse = O.merge_attention_partials([(o_s, l_s)])
    np.testing.assert_array_equal(o, o_s)
    np.testing.assert_allclose(lse, l_s, rtol=0, atol=1e-15)


def test_merge_closed_form_two_partials():
    # two partials with normalisers e^a and e^b: weights e^a/(e^a+e^b), e^b/(e^a+e^b)
    a, b = 0.3, -1.7
    o1, o2 = np.array([[[1.0, 2.0]]]), np.array([[[-4.0, 0.5]]])
    o, lse = O.merge_attention_partials([(o1, np.array([[a]])), (o2, np.array([[b]]))])
    wa = np.exp(a) / (np.exp(a) + np.exp(b))
    np.testing.assert_allclose(o, wa * o1 + (1 - wa) * o2, rtol=1e-14)
    np.testing.assert_allclose(lse, np.log(np.exp(a) + np.exp(b)), rtol=1e-14)


def test_merge_is_order_free_and_handles_far_apart_normalisers():
    g = np.random.default_rng(5)
    parts = [(g.standard_normal((1, 4, 3)), g.standard_normal((1, 4)) * 300.0) for _ in range(5)]
    o1, l1 = O.merge_attention_partials(parts)
    o2, l2 = O.merge_attention_partials(parts[::-1])
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=1e-14)
    # normalisers hundreds apart: no overflow, the largest partial dominates
    assert np.all(np.isfinite(o1)) and np.all(np.isfinite(l1))
    top = np.argmax(np.stack([l for _, l in parts]), axis=0)
    lse_max = np.max(np.stack([l for _, l in parts]), axis=0)
    assert np.all(l1 >= lse_max - 1e-12)


def test_split_of_identical_ranges_gives_the_range_result():
    # both halves hold the same keys and values: each partial equals the
    # single pass over one half, and lse grows by exactly log 2
    q, k, v = _qkv(21, length=12)
    k2, v2 = np.concatenate([k, k], axis=1), np.concatenate([v, v], axis=1)
    o_half, _, lse_half = O.gqa_attention(q, k, v)
    o, lse = O.gqa_attention_split_kv(q, k2, v2, [12])
    np.testing.assert_allclose(o, o_half, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, lse_half + np.log(2.0), rtol=0, atol=1e-13)

"""Pins for the oracle's routing and its float32 exp (CPU only).

moe_exp is pinned against float64 ``math.exp`` (error bound in float32 ulps);
top-k ids by brute force over all experts; weights by their closed forms
(renormalised weights sum to 1, ratios equal exp(l_i - l_j) or
sigmoid(l_i)/sigmoid(l_j)).
"""
import itertools
import math

import numpy as np
import pytest

from oracle import moe_oracle as O


def _ulp32(x):
    x = abs(float(np.float32(x)))
    if x == 0:
        return float(np.float32(1.4e-45))
    return float(np.spacing(np.float32(x)))


def test_moe_exp_accuracy_dense_grid():
    xs = np.linspace(-87.0, 88.5, 400001).astype(np.float32)
    got = O.moe_exp(xs).astype(np.float64)
    ref = np.exp(xs.astype(np.float64))
    ulps = np.abs(got - ref) / np.spacing(ref.astype(np.float32)).astype(np.float64)
    assert ulps.max() <= 2.0, ulps.max()


def test_moe_exp_small_arguments_and_specials():
    xs = np.concatenate([np.linspace(-1, 1, 100001), [0.0, -0.0, 1e-8, -1e-8]]).astype(np.float32)
    got = O.moe_exp(xs).astype(np.float64)
    ref = np.exp(xs.astype(np.float64))
    ulps = np.abs(got - ref) / np.spacing(ref.astype(np.float32)).astype(np.float64)
    assert ulps.max() <= 2.0
    assert O.moe_exp(np.float32(0.0)) == np.float32(1.0)
    assert O.moe_exp(np.float32(-np.inf)) < np.float32(1e-44)
    assert np.isinf(O.moe_exp(np.float32(100.0)))
    # subnormal results: within 1 subnormal step of the true value
    xs = np.linspace(-103.0, -88.0, 1001).astype(np.float32)
    got = O.moe_exp(xs).astype(np.float64)
    ref = np.exp(xs.astype(np.float64))
    assert np.all(np.abs(got - ref) <= np.maximum(2.0 * np.spacing(ref.astype(np.float32)), 1.5e-45))


def _brute_topk(row, k):
    E = len(row)
    order = sorted(range(E), key=lambda e: (-float(row[e]), e))
    return order[:k]


@pytest.mark.parametrize("T,E,k", [(6, 5, 2), (4, 8, 8), (5, 7, 3)])
def test_topk_ids_brute_force(T, E, k):
    rng = np.random.default_rng(T + E + k)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    logits[0, :] = 0.5                      # all tied: lowest indices win
    logits[1, 1] = logits[1, 3] = 9.0       # a tie at the top
    logits[2, :2] = -np.inf
    ids = O.topk_ids(logits, k)
    for t in range(T):
        assert ids[t].tolist() == _brute_topk(logits[t], k)
        # exhaustive check that no other k-subset has a larger minimum-by-order
        best = max(itertools.combinations(range(E), k),
                   key=lambda c: sorted([float(logits[t, e]) for e in c], reverse=True))
        assert sorted(float(logits[t, e]) for e in ids[t]) == sorted(float(logits[t, e]) for e in best)
    assert ids[0].tolist() == list(range(k))


def test_softmax_renormalised_weights_closed_form():
    rng = np.random.default_rng(7)
    logits = rng.standard_normal((200, 64)).astype(np.float32) * 3
    ids, w = O.route_topk(logits, 8, O.SOFTMAX, True)
    assert w.dtype == np.float32
    assert np.all(np.abs(w.astype(np.float64).sum(1) - 1.0) <= 8 * 2 ** -24 * 2)
    sel = np.take_along_axis(logits, ids, 1).astype(np.float64)
    ratio = w[:, 1:].astype(np.float64) / w[:, :1].astype(np.float64)
    # float32 rounding of l_j - l_top1, two exp ulps and two division roundings
    assert np.allclose(ratio, np.exp(sel[:, 1:] - sel[:, :1]), rtol=2e-6, atol=0)
    # equals the full softmax restricted to the top-k and renormalised
    full = np.exp(logits.astype(np.float64) - logits.max(1, keepdims=True))
    full /= full.sum(1, keepdims=True)
    ref = np.take_along_axis(full, ids, 1)
    ref /= ref.sum(1, keepdims=True)
    assert np.allclose(w, ref, rtol=1e-6, atol=0)


def test_softmax_not_renormalised_is_full_softmax():
    rng = np.random.default_rng(8)
    logits = rng.standard_normal((50, 16)).astype(np.float32)
    ids, w = O.route_topk(logits, 4, O.SOFTMAX, False)
    full = np.exp(logits.astype(np.float64) - logits.max(1, keepdims=True))
    full /= full.sum(1, keepdims=True)
    assert np.allclose(w, np.take_along_axis(full, ids, 1), rtol=2e-6, atol=0)


def test_sigmoid_weights_closed_form():
    rng = np.random.default_rng(9)
    logits = rng.standard_normal((200, 256)).astype(np.float32)
    ids, w = O.route_topk(logits, 8, O.SIGMOID, True)
    sel = np.take_along_axis(logits, ids, 1).astype(np.float64)
    sig = 1.0 / (1.0 + np.exp(-sel))
    ref = sig / sig.sum(1, keepdims=True)
    assert np.allclose(w, ref, rtol=1e-6, atol=0)
    ids2, w2 = O.route_topk(logits, 8, O.SIGMOID, False)
    assert np.array_equal(ids, ids2)
    assert np.allclose(w2, sig, rtol=1e-6, atol=0)


def test_exp_is_float32_deterministic_steps():
    # a hand-worked instance of the documented steps for x = 1:
    # n = rint(1.4426950) = 1, r = 1 - 0.693359375 - ln2_lo, p(r) * 2**1
    x = np.float32(1.0)
    n = 1
    r = np.float32(np.float32(x - np.float32(n * 0.693359375)) - np.float32(n * np.float32(float.fromhex("-0x1.bd0106p-13"))))
    p = np.float32(1.0 / math.factorial(7))
    for i in range(6, -1, -1):
        p = np.float32(np.float32(p * r) + np.float32(1.0 / math.factorial(i)))
    assert O.moe_exp(x) == np.float32(p * np.float32(2.0))
    assert abs(float(O.moe_exp(x)) - math.e) <= _ulp32(math.e)

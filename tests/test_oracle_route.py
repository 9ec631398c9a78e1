"""Pins of the oracle's router (top-k of the logits, softmax of the chosen k).

The pages describe no router; the reading (the k largest logits, lower expert
index first among equal values, weights = the softmax of the chosen logits,
i.e. the full softmax restricted to them and renormalised) is stated in the
oracle's C source. These tests pin it to library routines and closed forms:
numpy's stable argsort for the selection and its order, scipy's softmax for the
weights, and exact values where the arithmetic fixes them.
"""
import numpy as np
import pytest
from scipy.special import softmax

import oracle
import workloads


def ulp32(x):
    x = np.abs(np.asarray(x, dtype=np.float32))
    return np.spacing(x).astype(np.float64)


def stable_topk(z, k):
    return np.argsort(-z, axis=1, kind="stable")[:, :k].astype(np.int32)


@pytest.mark.parametrize("T,E,k", [(64, 256, 8), (33, 16, 4), (7, 1024, 32), (5, 8, 8), (3, 1, 1)])
def test_ids_match_stable_argsort_random(T, E, k):
    z = np.random.default_rng(T * E + k).standard_normal((T, E)).astype(np.float32)
    ids, _ = oracle.route_topk(z, k)
    assert np.array_equal(ids, stable_topk(z, k))


def test_ids_ties_lower_index_first():
    # integer-valued logits: many equal values, so the order among ties decides the result
    rng = np.random.default_rng(3)
    z = rng.integers(-2, 3, size=(200, 64)).astype(np.float32)
    ids, _ = oracle.route_topk(z, 8)
    assert np.array_equal(ids, stable_topk(z, 8))


def test_signed_zeros_are_equal():
    z = np.zeros((1, 6), dtype=np.float32)
    z[0, [0, 2, 4]] = -0.0
    ids, w = oracle.route_topk(z, 4)
    assert ids.tolist() == [[0, 1, 2, 3]]
    assert np.all(w == np.float32(0.25))


def test_weights_match_scipy_softmax_of_chosen():
    z = np.random.default_rng(11).standard_normal((300, 256)).astype(np.float32)
    ids, w = oracle.route_topk(z, 8)
    chosen = np.take_along_axis(z, ids, axis=1).astype(np.float64)
    ref = softmax(chosen, axis=1)
    assert np.all(np.abs(w.astype(np.float64) - ref) <= ulp32(ref))
    # the same as the full softmax over all E restricted to the chosen k and renormalised
    full = softmax(z.astype(np.float64), axis=1)
    sub = np.take_along_axis(full, ids, axis=1)
    sub /= sub.sum(axis=1, keepdims=True)
    assert np.all(np.abs(w.astype(np.float64) - sub) <= 2 * ulp32(sub))


def test_weight_invariants():
    z = (3.0 * np.random.default_rng(5).standard_normal((100, 64))).astype(np.float32)
    ids, w = oracle.route_topk(z, 6)
    w64 = w.astype(np.float64)
    assert np.all(np.abs(w64.sum(axis=1) - 1.0) <= 6 * 2.0 ** -24)
    # ordered like the logits, and ratios follow the logit differences
    assert np.all(np.diff(w64, axis=1) <= 0)
    chosen = np.take_along_axis(z, ids, axis=1).astype(np.float64)
    ratio = w64[:, 1:] / w64[:, :1]
    assert np.allclose(ratio, np.exp(chosen[:, 1:] - chosen[:, :1]), rtol=4 * 2.0 ** -24 * 4, atol=0)


def test_closed_forms():
    # equal logits: the first k experts, each 1/k exactly (exp(0) = 1, the sum is k)
    z = np.full((2, 10), 1.5, dtype=np.float32)
    ids, w = oracle.route_topk(z, 5)
    assert ids.tolist() == [[0, 1, 2, 3, 4]] * 2
    assert np.all(w == np.float32(1.0 / 5.0))
    # k = 1: the argmax with weight exactly 1
    z = np.random.default_rng(2).standard_normal((50, 32)).astype(np.float32)
    ids, w = oracle.route_topk(z, 1)
    assert np.array_equal(ids[:, 0], np.argmax(z, axis=1))
    assert np.all(w == 1.0)


def test_negative_infinity_logits():
    z = np.random.default_rng(8).standard_normal((20, 12)).astype(np.float32)
    z[:, [1, 5, 6]] = -np.inf
    ids, w = oracle.route_topk(z, 8)
    # 9 finite experts per row: none of the -inf ones is chosen
    assert not np.isin(ids, [1, 5, 6]).any()
    assert np.array_equal(ids, stable_topk(z, 8))
    # fewer finite experts than k: the -inf ones follow by index with weight 0
    ids, w = oracle.route_topk(z[:, :8], 8)
    assert ids.tolist()[0][-3:] == [1, 5, 6]
    assert np.all(w[:, -3:] == 0.0)
    # a row of -inf only: the first k experts, 1/k each
    ids, w = oracle.route_topk(np.full((1, 9), -np.inf, dtype=np.float32), 3)
    assert ids.tolist() == [[0, 1, 2]]
    assert np.all(w == np.float32(1.0 / 3.0))


def test_reproduces_workload_routing():
    # the harness's routing (numpy, FP64 logits) picks the same experts as the router on those logits
    # rounded to FP32 wherever that rounding creates no new tie
    for name in ("moe_decode_t512", "moe_zipf_t1024"):
        c = workloads.CONFIGS[name]
        z = workloads.router_logits(c["T"], c["E"], c["routing"], 0, c.get("zipf_s", 1.1), c.get("zero_experts", 0))
        ids_ref, w_ref = workloads.config_routing(name)
        ids, w = oracle.route_topk(z.astype(np.float32), c["k"])
        same = np.all(ids == ids_ref, axis=1)
        assert same.mean() > 0.999
        assert np.allclose(w[same], w_ref[same], rtol=1e-5, atol=1e-7)

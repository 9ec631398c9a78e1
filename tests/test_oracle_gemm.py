"""Pins for the oracle's grouped GEMM, SwiGLU epilogue, routing and combine.

The GEMM is checked by exact rational brute force (fractions.Fraction) with an
independent decoder, closed forms and structural cases (which half is gate,
which expert a row uses, empty experts). Routing is checked against numpy's
stable argsort / bincount; the combine against one-hot and exact-weight cases
and a numpy einsum.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def e2m1_table():
    t = {}
    for line in open(os.path.join(GOLDEN, "e2m1_values.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            c, v = line.split()
            t[int(c)] = Fraction(float(v))
    return t


E2M1 = e2m1_table()
E4M3 = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def exact_value(q_row, sf_row, k):
    code = (int(q_row[k // 2]) >> (4 * (k % 2))) & 0xF
    return E2M1[code] * Fraction(float(E4M3[int(sf_row[k // 16])]))


def random_codes(rng, rows, K, sf_hi=127):
    q = rng.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)
    # finite scales only (0x7F / 0xFF are NaN)
    sf = rng.integers(0, sf_hi, size=(rows, K // 16), dtype=np.uint8)
    return q, sf


def silu(v):
    return v / (1 + math.exp(-v)) if v > -700 else -0.0


@pytest.mark.parametrize("swiglu", [False, True])
def test_bruteforce_fraction_tiny(swiglu):
    rng = np.random.default_rng(7)
    E, N, K = 3, 4, 32
    off = np.array([0, 3, 3, 5], dtype=np.int32)        # expert 1 empty
    sf_hi = 0x40 if swiglu else 127     # keep SwiGLU arguments where the gate is not saturated
    a_q, a_sf = random_codes(rng, 5, K, sf_hi)
    w_q, w_sf = random_codes(rng, E * N, K, sf_hi)
    w_q = w_q.reshape(E, N, K // 2)
    w_sf = w_sf.reshape(E, N, K // 16)
    a_g = np.float32(0.37)
    w_g = np.array([0.05, 3.0, 0.011], dtype=np.float32)
    got = oracle.grouped_gemm(a_q, a_sf, a_g, w_q, w_sf, w_g, off, N, K, swiglu)
    nout = N // 2 if swiglu else N
    assert got.shape == (5, nout)
    for m in range(5):
        e = 0 if m < 3 else 2
        alpha = Fraction(float(a_g)) * Fraction(float(w_g[e]))
        for n in range(nout):
            acc = sum(exact_value(a_q[m], a_sf[m], k) * exact_value(w_q[e, n], w_sf[e, n], k) for k in range(K))
            v = float(alpha * acc)
            if swiglu:
                u = float(alpha * sum(exact_value(a_q[m], a_sf[m], k) * exact_value(w_q[e, N // 2 + n], w_sf[e, N // 2 + n], k)
                                      for k in range(K)))
                v = silu(v) * u
            assert got[m, n] == pytest.approx(v, rel=1e-12, abs=1e-300)
    # the sampled entry point agrees with the full one
    rows = np.array([0, 1, 2, 3, 4, 4], dtype=np.int64)
    cols = np.array([0, 1, nout - 1, 0, 1, nout - 1], dtype=np.int64)
    at = oracle.grouped_gemm_at(a_q, a_sf, a_g, w_q, w_sf, w_g, off, N, K, swiglu, rows, cols)
    assert np.array_equal(at, got[rows, cols])


def test_all_ones_closed_form():
    K, N = 256, 8
    ones = np.full((4, K), 0x3F80, dtype=np.uint16)
    a_q, a_sf, a_g = oracle.quantize(ones)
    w_q, w_sf, w_g = oracle.quantize(np.full((N, K), 0x3F80, dtype=np.uint16))
    out = oracle.grouped_gemm(a_q, a_sf, a_g, w_q[None], w_sf[None], np.array([w_g]), np.array([0, 4]), N, K, False)
    assert np.all(oracle.bf16_round(out) == oracle.bf16_from_double(256.0))


def test_single_block_closed_form():
    K = 64
    a_q = np.zeros((1, K // 2), dtype=np.uint8)
    a_sf = np.zeros((1, K // 16), dtype=np.uint8)
    # block 1 (elements 16..31): codes 1..15 then 7, scale 0x38 (= 1.0)
    codes = list(range(1, 16)) + [7]
    for i, c in enumerate(codes):
        k = 16 + i
        a_q[0, k // 2] |= c << (4 * (k % 2))
    a_sf[0, 1] = 0x38
    w_q = np.full((1, 1, K // 2), 0x22, dtype=np.uint8)      # every weight element 1.0
    w_sf = np.full((1, 1, K // 16), 0x38, dtype=np.uint8)     # scale 1.0
    out = oracle.grouped_gemm(a_q, a_sf, 1.0, w_q, w_sf, np.array([1.0], np.float32), np.array([0, 1]), 1, K, False)
    want = sum([0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6, 6])
    assert out[0, 0] == want == 6.0


def test_swiglu_gate_is_first_half_and_limits():
    K, N = 32, 4            # gate rows 0..1, up rows 2..3
    a_q = np.full((1, K // 2), 0x22, dtype=np.uint8)          # all 1.0
    a_sf = np.full((1, K // 16), 0x38, dtype=np.uint8)
    w_q = np.zeros((1, N, K // 2), dtype=np.uint8)
    w_sf = np.full((1, N, K // 16), 0x38, dtype=np.uint8)
    w_q[0, 0, 0] = 0xA          # gate row 0: one element -1.0 -> acc -1
    w_q[0, 2, :] = 0x22         # up row 0: 32 elements of 1.0 -> acc 32
    # gate row 1: zero -> output 0 whatever up is
    w_q[0, 3, :] = 0x77
    out = oracle.grouped_gemm(a_q, a_sf, 1.0, w_q, w_sf, np.array([1.0], np.float32), np.array([0, 1]), N, K, True)
    assert out[0, 0] == pytest.approx((-1 / (1 + math.e)) * 32, rel=1e-15)   # silu(-1) * 32
    assert out[0, 1] == 0.0
    # large gate: silu(v) -> v
    w_q[0, 0, :] = 0x77         # gate acc = 32 * 6 = 192
    out = oracle.grouped_gemm(a_q, a_sf, 1.0, w_q, w_sf, np.array([1.0], np.float32), np.array([0, 1]), N, K, True)
    assert out[0, 0] == pytest.approx(192.0 * 32, rel=1e-12)


def test_rows_use_their_own_expert():
    K, N, E = 32, 2, 4
    a_q = np.full((6, K // 2), 0x22, dtype=np.uint8)
    a_sf = np.full((6, K // 16), 0x38, dtype=np.uint8)
    w_q = np.full((E, N, K // 2), 0x22, dtype=np.uint8)
    w_sf = np.full((E, N, K // 16), 0x38, dtype=np.uint8)
    w_g = np.array([1, 2, 4, 8], dtype=np.float32)
    off = np.array([0, 2, 2, 5, 6], dtype=np.int32)
    out = oracle.grouped_gemm(a_q, a_sf, 1.0, w_q, w_sf, w_g, off, N, K, False)
    assert out[:, 0].tolist() == [32, 32, 128, 128, 128, 256]


def test_permute_matches_numpy_stable_sort():
    ids, _ = workloads.routing(300, 32, 4, "zipf", seed=3, zero_experts=3)
    off, src, inv = oracle.permute(ids, 32)
    counts = np.bincount(ids.ravel(), minlength=32)
    assert np.array_equal(off, np.concatenate([[0], np.cumsum(counts)]))
    order = np.argsort(ids.ravel(), kind="stable")
    assert np.array_equal(src, order // 4)
    assert np.array_equal(inv[order], np.arange(ids.size))
    assert (counts == 0).sum() >= 3            # the three zero-probability experts stay empty


def test_permute_rejects_out_of_range():
    with pytest.raises(ValueError):
        oracle.permute(np.array([[0, 5]], dtype=np.int32), 4)


def test_gather_rows_is_fancy_indexing():
    rng = np.random.default_rng(0)
    src = rng.integers(0, 256, size=(10, 48), dtype=np.uint8)
    idx = rng.integers(0, 10, size=25).astype(np.int32)
    assert np.array_equal(oracle.gather_rows(src, idx), src[idx])


def test_combine_one_hot_and_exact_weights():
    T, k, H = 5, 4, 24
    ids, _ = workloads.routing(T, 8, k, "uniform", seed=1)
    off, src, inv = oracle.permute(ids, 8)
    y = workloads.random_bf16_bits((T * k, H), seed=2)
    w = np.zeros((T, k), dtype=np.float32)
    w[:, 2] = 1.0
    out = oracle.bf16_round(oracle.combine(y, inv, w))
    assert np.array_equal(out, y[inv.reshape(T, k)[:, 2]])
    # identical expert outputs and weights summing exactly to one reproduce the row
    yrow = workloads.random_bf16_bits((1, H), seed=3)
    y_same = np.repeat(yrow, T * k, axis=0)
    w = np.tile(np.array([0.5, 0.25, 0.125, 0.125], dtype=np.float32), (T, 1))
    out = oracle.bf16_round(oracle.combine(y_same, inv, w))
    assert np.array_equal(out, np.repeat(yrow, T, axis=0))


def test_combine_matches_einsum():
    T, k, H, E = 7, 3, 40, 6
    ids, w = workloads.routing(T, E, k, "uniform", seed=4)
    _, _, inv = oracle.permute(ids, E)
    y = workloads.random_bf16_bits((T * k, H), seed=5)
    yf = oracle.bf16_bits_to_f64(y)
    want = np.einsum("tj,tjh->th", w.astype(np.float64), yf[inv.reshape(T, k)])
    assert np.allclose(oracle.combine(y, inv, w), want, rtol=1e-14, atol=1e-300)

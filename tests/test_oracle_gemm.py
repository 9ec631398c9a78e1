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



def test_combine_skips_pairs_without_a_row():
    # a -1 slot (the permute's marker for a pair with an invalid expert) adds nothing: the combine equals the
    # einsum over the remaining slots, and a token whose slots are all -1 gets zeros
    T, k, H, E = 6, 3, 32, 6
    ids, w = workloads.routing(T, E, k, "uniform", seed=6)
    _, _, inv = oracle.permute(ids, E)
    inv = inv.copy()
    inv[1] = -1
    inv[3 * k: 4 * k] = -1
    y = workloads.random_bf16_bits((T * k, H), seed=7)
    yf = oracle.bf16_bits_to_f64(y)
    inv2 = inv.reshape(T, k)
    keep = (inv2 >= 0).astype(np.float64)
    want = np.einsum("tj,tjh->th", w.astype(np.float64) * keep, yf[np.maximum(inv2, 0)])
    got = oracle.combine(y, inv, w)
    assert np.allclose(got, want, rtol=1e-14, atol=1e-300)
    assert np.all(got[3] == 0.0)

# ---- the FP32-path error bound used to recognise rounding ties -------------------------------------------

def _decoded(q, sf):
    """Decoded block-scaled values (no global scale) with the oracle's own codecs, in FP64."""
    e2 = np.array([oracle.e2m1_decode(c) for c in range(16)])
    e4 = np.array([oracle.e4m3_decode(b) for b in range(256)])
    codes = np.stack([q & 15, q >> 4], axis=-1).reshape(q.shape[0], -1)
    return e2[codes] * np.repeat(e4[sf], 16, axis=1)


def _fp32_model(a, w, alpha, order_rng):
    """One FP32 computation of the kind the bound covers: exact 16-element block partials, accumulated in
    FP32 in a random order, times FP32 alpha, rounded in FP32."""
    P = (a.reshape(a.shape[0], -1, 16)[:, None, :, :] * w.reshape(w.shape[0], -1, 16)[None, :, :, :]).sum(-1)
    Pf = P.astype(np.float32)
    assert np.array_equal(Pf.astype(np.float64), P)        # block partials are exact in FP32
    acc = np.zeros(P.shape[:2], dtype=np.float32)
    for b in order_rng.permutation(P.shape[2]):
        acc = (acc + Pf[:, :, b]).astype(np.float32)
    return (np.float32(alpha) * acc).astype(np.float32)


@pytest.mark.parametrize("K", [256, 2048])
def test_fp32_bound_covers_fp32_accumulation(K):
    rng = np.random.default_rng(K)
    M, N = 6, 8
    a_bits = workloads.random_bf16_bits((M, K), seed=K)
    w_bits = workloads.random_bf16_bits((N, K), seed=K + 1, std=0.02)
    aq, asf, ag = oracle.quantize(a_bits)
    wq, wsf, wg = oracle.quantize(w_bits)
    off = np.array([0, M], np.int32)
    exact = oracle.grouped_gemm(aq, asf, ag, wq[None], wsf[None], np.array([wg]), off, N, K, False)
    bound = oracle.grouped_gemm_bound(aq, asf, ag, wq[None], wsf[None], np.array([wg]), off, N, K, False)
    alpha = np.float32(np.float32(ag) * np.float32(wg))
    A, W = _decoded(aq, asf), _decoded(wq, wsf)
    worst = 0.0
    for trial in range(20):
        got = _fp32_model(A, W, alpha, rng).astype(np.float64)
        assert np.all(np.abs(got - exact) <= bound)
        worst = max(worst, float(np.max(np.abs(got - exact) / bound)))
    assert worst > 1e-4      # the bound is not vacuous: some orders use a visible share of it
    # the sampled form gives the same bound at the same points
    rr, cc = np.array([0, 3, 5]), np.array([7, 0, 2])
    assert np.array_equal(oracle.grouped_gemm_bound(aq, asf, ag, wq[None], wsf[None], np.array([wg]), off, N, K,
                                                    False, rr, cc), bound[rr, cc])


def test_fp32_bound_swiglu_covers_fp32_epilogue():
    rng = np.random.default_rng(5)
    M, N, K = 5, 8, 512
    a_bits = workloads.random_bf16_bits((M, K), seed=50)
    w_bits = workloads.random_bf16_bits((N, K), seed=51, std=0.05)
    aq, asf, ag = oracle.quantize(a_bits)
    wq, wsf, wg = oracle.quantize(w_bits)
    off = np.array([0, M], np.int32)
    exact = oracle.grouped_gemm(aq, asf, ag, wq[None], wsf[None], np.array([wg]), off, N, K, True)
    bound = oracle.grouped_gemm_bound(aq, asf, ag, wq[None], wsf[None], np.array([wg]), off, N, K, True)
    alpha = np.float32(np.float32(ag) * np.float32(wg))
    A, W = _decoded(aq, asf), _decoded(wq, wsf)
    for trial in range(10):
        y = _fp32_model(A, W, alpha, rng)
        g, u = y[:, : N // 2], y[:, N // 2:]
        h = (g / (np.float32(1) + np.exp(-g))).astype(np.float32) * u      # single-precision SiLU and product
        assert np.all(np.abs(h.astype(np.float64) - exact) <= bound)
    assert np.all(bound > 0) and np.all(bound < 1e-3 * np.sqrt(np.mean(exact ** 2)))

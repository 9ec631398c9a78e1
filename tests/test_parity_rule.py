"""The BF16 parity rule itself (tests/helpers.compare_bf16), on planted cases: a one-ulp disagreement is a
rounding tie only when the exact value lies within the element's derived bound of the midpoint; anything
else is held to the stated max-abs and relative-Frobenius bounds."""
import numpy as np
import pytest

import oracle
from tests.helpers import compare_bf16


def bits(v):
    return oracle.bf16_round(np.asarray(v, dtype=np.float64))


def case(n=4000, seed=0):
    ex = np.random.default_rng(seed).standard_normal(n)
    return ex, bits(ex)


def test_exact_match_passes():
    ex, ref = case()
    st = compare_bf16(ref.copy(), ref, "exact", exact=ex, band=np.full(ex.shape, 1e-9))
    assert st["exact_frac"] == 1.0 and st["tie_flips"] == 0


def test_flip_at_midpoint_within_band_is_a_tie():
    ex, ref = case()
    i = int(np.argmax(np.abs(ex)))                      # a large element: one ulp is far above 1e-2 RMS
    lo = np.float64(np.frombuffer((ref[i:i + 1].astype(np.uint32) << 16).astype(np.uint32).tobytes(), np.float32)[0])
    hi_bits = ref[i] + np.uint16(1)
    hi = np.float64(np.frombuffer((np.array([hi_bits], np.uint32) << 16).astype(np.uint32).tobytes(), np.float32)[0])
    mid = 0.5 * (lo + hi)
    ex2 = ex.copy()
    ex2[i] = mid - 1e-12 * np.sign(mid)                 # exact value a hair on the reference's side of the midpoint
    ref2 = bits(ex2)
    gpu = ref2.copy()
    gpu[i] = hi_bits if ref2[i] == ref[i] else ref[i]   # the other neighbour
    band = np.full(ex.shape, 1e-9)
    st = compare_bf16(gpu, ref2, "tie", exact=ex2, band=band)
    assert st["tie_flips"] == 1
    # the same flip with the exact value far from the midpoint (outside its band) fails
    band_small = np.full(ex.shape, 1e-15)
    with pytest.raises(AssertionError):
        compare_bf16(gpu, ref2, "not a tie", exact=ex2, band=band_small)


def test_two_ulp_error_on_a_large_element_fails():
    ex, ref = case()
    i = int(np.argmax(np.abs(ex)))
    gpu = ref.copy()
    gpu[i] = ref[i] + np.uint16(2)
    with pytest.raises(AssertionError):
        compare_bf16(gpu, ref, "two ulp", exact=ex, band=np.full(ex.shape, 1.0))


def test_small_errors_within_max_abs_pass_without_ties():
    ex, ref = case()
    small = np.argsort(np.abs(ex))[:50]                 # tiny elements: one ulp is far below 1e-2 RMS
    gpu = ref.copy()
    gpu[small] = ref[small] ^ np.uint16(1)
    st = compare_bf16(gpu, ref, "small", exact=ex, band=np.zeros(ex.shape))
    assert st["tie_flips"] == 0 and st["exact_frac"] < 1.0


def test_a_tie_needs_a_band():
    ex, ref = case()
    with pytest.raises(AssertionError):
        compare_bf16(ref, ref, "no band", exact=ex)

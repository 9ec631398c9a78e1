"""Pins for the oracle's NVFP4 quantiser: closed forms, special cases,
round-trip invariants and an error bound that follows from the grid alone."""
import numpy as np
import pytest
import torch

import oracle
import workloads

ONE = 0x3F80    # BF16 1.0
ZERO = 0x0000


def bf16(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_all_ones_closed_form():
    x = np.full((3, 64), ONE, dtype=np.uint16)
    q, sf, g = oracle.quantize(x)
    # amax = 1 -> g_enc = 2688, s = (1/6)*2688 = 448 -> S = 0x7E, f = 2688/448 = 6 -> code 6 = 0x7
    assert np.all(q == 0x77)
    assert np.all(sf == 0x7E)
    assert g == np.float32(1.0) / np.float32(2688.0)
    deq = oracle.dequantize(q, sf, 1.0)            # without the global scale: 6 * 448
    assert np.all(deq == 2688.0)


def test_all_zero_tensor():
    x = np.zeros((2, 32), dtype=np.uint16)
    q, sf, g = oracle.quantize(x)
    assert np.all(q == 0) and np.all(sf == 0) and g == np.float32(1.0)


def test_global_scale_value():
    x = bf16([[5.0] + [0.0] * 15])
    _, _, g = oracle.quantize(x)
    assert g == np.float32(5.0) / np.float32(2688.0)


def test_tensor_amax_element_encodes_to_six():
    x = workloads.random_bf16_bits((8, 128), seed=5)
    xf = oracle.bf16_bits_to_f64(x)
    r, c = np.unravel_index(np.argmax(np.abs(xf)), xf.shape)
    q, sf, g = oracle.quantize(x)
    code = (q[r, c // 2] >> (4 * (c % 2))) & 0xF
    assert code & 0x7 == 0x7
    assert (code >> 3) == (1 if xf[r, c] < 0 else 0)
    assert sf[r, c // 16] == 0x7E


def test_fixed_scale_block_scale_and_roundtrip():
    # With the global scale given as 1, a block whose amax is 6 gets s = 1 -> S = 0x38,
    # f = 1, so every value already on the E2M1 grid encodes to its own code.
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]
    x = bf16([grid])
    q, sf, g = oracle.quantize(x, global_scale=1.0)
    assert g == 1.0 and sf[0, 0] == 0x38
    codes = [(q[0, i // 2] >> (4 * (i % 2))) & 0xF for i in range(16)]
    assert codes == list(range(16))
    # block amax 3 -> s = 0.5 -> S = 0x30 (E4M3 exponent field 6, mantissa 0)
    q, sf, _ = oracle.quantize(bf16([[3.0] + [1.0] * 15]), global_scale=1.0)
    assert sf[0, 0] == 0x30


def test_negative_value_rounding_to_zero_keeps_sign():
    vals = [[6.0, -0.01, 0.01] + [0.0] * 13]
    q, _, _ = oracle.quantize(bf16(vals), global_scale=1.0)
    codes = [(q[0, i // 2] >> (4 * (i % 2))) & 0xF for i in range(3)]
    assert codes == [0x7, 0x8, 0x0]


def test_nibble_order_even_element_low():
    vals = [[6.0, 1.0] + [0.0] * 14]
    q, _, _ = oracle.quantize(bf16(vals), global_scale=1.0)
    assert q[0, 0] == (0x7 | (0x2 << 4))


def test_zero_block_gives_zero_scale_and_codes():
    vals = [[0.0] * 16 + [1.0] * 16]
    q, sf, _ = oracle.quantize(bf16(vals))
    assert sf[0, 0] == 0 and np.all(q[0, :8] == 0)
    assert sf[0, 1] == 0x7E


@pytest.mark.parametrize("seed,std", [(0, 1.0), (1, 0.02), (2, 100.0)])
def test_error_bound_from_grid(seed, std):
    x = workloads.random_bf16_bits((16, 256), seed=seed, std=std)
    q, sf, g = oracle.quantize(x)
    xf = oracle.bf16_bits_to_f64(x)
    deq = oracle.dequantize(q, sf, g)
    scale = np.repeat(np.array([[oracle.e4m3_decode(int(b)) for b in row] for row in sf]), 16, axis=1) * float(g)
    y = np.abs(xf) / scale
    half_step = np.where(y < 2, 0.25, np.where(y < 4, 0.5, 1.0))
    err = np.abs(deq - xf)
    sat = y > 6 * (1 + 1e-6)
    assert np.all(err[~sat] <= half_step[~sat] * scale[~sat] * (1 + 1e-5))
    assert np.all(np.abs(deq[sat]) == 6 * scale[sat])
    # a block scale never exceeds the E4M3 maximum and the largest block hits it
    assert sf.max() == 0x7E


def test_static_global_scale_saturates():
    x = bf16([[12.0] + [0.0] * 15])
    q, sf, g = oracle.quantize(x, global_scale=1.0 / 448.0)   # g_enc = 448: s = 2*448 -> 448 (satfinite)
    assert sf[0, 0] == 0x7E
    assert (q[0, 0] & 0xF) == 0x7                              # y = 12 * 448/448 = 12 -> saturates to 6


def test_quantize_with_amax_is_quantize_of_the_whole_tensor():
    # one global scale per tensor: rows quantised with the tensor's amax equal the tensor's own quantisation,
    # also when the rows are split into parts (expert-parallel ranks) that each see only their part
    x = workloads.random_bf16_bits((96, 256), seed=21, std=2.0)
    q, sf, g = oracle.quantize(x)
    q1, sf1, g1 = oracle.quantize_with_amax(x, oracle.amax(x))
    assert np.array_equal(q1, q) and np.array_equal(sf1, sf) and g1 == g
    a, b = x[:40], x[40:]
    assert oracle.amax(a) != oracle.amax(b)            # the parts alone would get different scales
    for part, lo in ((a, 0), (b, 40)):
        qp, sfp, gp = oracle.quantize_with_amax(part, oracle.amax(x))
        assert np.array_equal(qp, q[lo: lo + len(part)]) and np.array_equal(sfp, sf[lo: lo + len(part)])
        assert gp == g
    # and the part without the tensor's max element has a different scale of its own (not vacuous)
    small = a if oracle.amax(a) < oracle.amax(x) else b
    assert oracle.quantize(small)[2] != g

"""Pins for the oracle's scalar codecs (E2M1, E4M3, BF16 rounding).

Each check compares the oracle against something other than itself: the
format's printed value table, torch's float8_e4m3fn / bfloat16 conversions
(library routines), closed forms, or brute force over all codes.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load_e2m1_table():
    table = {}
    with open(os.path.join(GOLDEN, "e2m1_values.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            c, v = line.split()
            table[int(c)] = float(v)
    assert len(table) == 16
    return table


E2M1 = load_e2m1_table()


def test_e2m1_decode_matches_value_table():
    for code, v in E2M1.items():
        got = oracle.e2m1_decode(code)
        assert got == v and math.copysign(1, got) == math.copysign(1, v), (code, got, v)


@pytest.mark.parametrize("y,code", [
    (0.0, 0x0), (-0.0, 0x8), (0.25, 0x0), (0.2500001, 0x1), (0.75, 0x2), (1.25, 0x2),
    (1.75, 0x4), (2.5, 0x4), (3.5, 0x6), (5.0, 0x6), (5.0000005, 0x7), (6.0, 0x7),
    (7.0, 0x7), (1e30, 0x7), (-0.25, 0x8), (-0.1, 0x8), (-0.75, 0xA), (-5.0, 0xE), (-100.0, 0xF),
    (0.24999999, 0x0), (2.4999998, 0x4), (2.5000002, 0x5),
])
def test_e2m1_ties_saturation_sign(y, code):
    assert oracle.e2m1_encode(y) == code


def test_e2m1_encode_is_nearest_with_even_ties_bruteforce():
    rng = np.random.default_rng(1)
    ys = np.concatenate([
        rng.uniform(-8, 8, 20000),
        rng.standard_normal(5000) * 3,
        # exact tie points and their float32 neighbours
        np.array([m for t in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)
                  for m in (t, np.nextafter(np.float32(t), np.float32(0)), np.nextafter(np.float32(t), np.float32(9)))]),
    ]).astype(np.float32)
    mags = [E2M1[c] for c in range(8)]
    for y in ys:
        a = abs(float(y))
        d = [abs(m - a) for m in mags]
        best = min(d)
        cands = [c for c in range(8) if d[c] == best]
        if a > 6.0:
            want = 7
        elif len(cands) == 1:
            want = cands[0]
        else:
            want = [c for c in cands if c % 2 == 0][0]   # even mantissa bit wins the tie
        want |= 0x8 if math.copysign(1, float(y)) < 0 else 0
        assert oracle.e2m1_encode(float(y)) == want, (float(y), want)


def e4m3_closed_form(b):
    s = -1.0 if b & 0x80 else 1.0
    e = (b >> 3) & 0xF
    m = b & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * m * 2.0 ** -9
    return s * (1 + m / 8) * 2.0 ** (e - 7)


def test_e4m3_decode_all_codes_closed_form_and_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    via_torch = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for b in range(256):
        got = oracle.e4m3_decode(b)
        cf = e4m3_closed_form(b)
        if math.isnan(cf):
            assert math.isnan(got) and math.isnan(via_torch[b])
            continue
        assert got == cf == via_torch[b], (b, got, cf, via_torch[b])
    assert oracle.e4m3_decode(0x7E) == 448.0
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(2)
    finite = np.array([e4m3_closed_form(b) for b in range(127)])
    mids = (finite[:-1] + finite[1:]) / 2
    s = np.concatenate([
        rng.uniform(0, 448, 20000),
        np.exp(rng.uniform(np.log(2.0 ** -12), np.log(448.0), 20000)),
        mids, finite,
        np.nextafter(mids.astype(np.float32), np.float32(0)), np.nextafter(mids.astype(np.float32), np.float32(1e9)),
    ]).astype(np.float32)
    s = s[(s >= 0) & (s <= 448)]
    want = torch.from_numpy(s).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for v, w in zip(s, want):
        assert oracle.e4m3_encode(float(v)) == int(w), (float(v), int(w))


@pytest.mark.parametrize("s,code", [(448.0, 0x7E), (464.0, 0x7E), (1e6, 0x7E), (0.0, 0x00),
                                    (2.0 ** -10, 0x00), (2.0 ** -10 * 1.0001, 0x01), (0.5, 0x30)])
def test_e4m3_saturation_and_ties(s, code):
    assert oracle.e4m3_encode(s) == code


def test_bf16_rounding_matches_torch_on_float32_inputs():
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.standard_normal(50000) * 10.0 ** rng.uniform(-30, 30, 50000),
                        rng.standard_normal(1000)]).astype(np.float32)
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.bf16_round(v.astype(np.float64))
    assert np.array_equal(got, want)


def test_bf16_rounding_single_step_from_double():
    # 1 + 2^-8 + 2^-40 lies just above the BF16 midpoint between 1 and 1 + 2^-7;
    # a detour through FP32 would land on the midpoint and round down to 1.0.
    assert oracle.bf16_from_double(1 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81
    assert oracle.bf16_from_double(1 + 2.0 ** -8) == 0x3F80          # tie -> even
    assert oracle.bf16_from_double(1 + 3 * 2.0 ** -8) == 0x3F82      # tie -> even (up)
    assert oracle.bf16_from_double(-2.0) == 0xC000
    assert oracle.bf16_from_double(-0.0) == 0x8000
    assert oracle.bf16_from_double(1e39) == 0x7F80

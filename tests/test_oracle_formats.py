"""Pins of the oracle's number formats (bf16, E4M3, E8M0) against hand-worked
values, library conversions and an exact brute-force search.

Format sources: pytorch/ao PR #4743 "[mxfp8 training] Add a fused gated-activation
(SwiGLU) + MXFP8 quantization kernel", section "Summary" (RCEIL MXFP8 cast with
E4M3 data and E8M0 scales over 1x32 / 32x1 blocks).
"""
import math
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import naive_ref
from conftest import read_golden


def _f32(x):
    return float(np.float32(x))


# ------------------------------------------------------------------ bf16
def test_bf16_rounding_matches_torch_on_random_and_edge_bits():
    rng = np.random.default_rng(123)
    bits = rng.integers(0, 2 ** 32, size=20000, dtype=np.uint64).astype(np.uint32)
    # ties and near-ties at every exponent: low 16 bits 0x8000, 0x7FFF, 0x8001
    hi = rng.integers(0, 2 ** 16, size=3000, dtype=np.uint64).astype(np.uint32) << 16
    edge = np.concatenate([hi | 0x8000, hi | 0x7FFF, hi | 0x8001, hi,
                           np.array([0x7F7FFFFF, 0x7F7F8000, 0x7F7F7FFF, 0x00000001,
                                     0x80008000, 0x00018000, 0x00008000], np.uint32)])
    allb = np.concatenate([bits, edge])
    f = allb.view(np.float32)
    f = f[~np.isnan(f)]
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.f32_to_bf16(float(v)) for v in f], np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_nan_and_inf():
    assert oracle.f32_to_bf16(float("nan")) & 0x7FFF > 0x7F80
    assert oracle.f32_to_bf16(float("inf")) == 0x7F80
    assert oracle.f32_to_bf16(float("-inf")) == 0xFF80
    assert oracle.f32_to_bf16(_f32(3.4028234663852886e38)) == 0x7F80  # rounds past max


# ------------------------------------------------------------------ E4M3
@pytest.mark.parametrize("row", read_golden("e4m3_hand.txt"))
def test_e4m3_hand_table(row):
    value, code = eval(row[0]), int(row[1], 16)
    assert oracle.e4m3_encode(float(value)) == code, row


def test_e4m3_decode_encode_roundtrip_all_codes():
    for c in range(256):
        v = oracle.e4m3_decode(c)
        if (c & 0x7F) == 0x7F:
            assert math.isnan(v)
            continue
        assert oracle.e4m3_encode(v) == c, hex(c)


def test_e4m3_decode_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_decode(c) for c in range(256)])
    same = (ref == got) | (np.isnan(ref) & np.isnan(got))
    assert same.all()


def test_e4m3_midpoints_round_to_even_and_neighbours_to_nearest():
    finite = sorted({oracle.e4m3_decode(c) for c in range(0x7F)})
    for lo, hi in zip(finite[:-1], finite[1:]):
        mid = (lo + hi) / 2  # exact in binary64
        c_lo, c_hi = oracle.e4m3_encode(lo), oracle.e4m3_encode(hi)
        even = c_lo if c_lo % 2 == 0 else c_hi
        assert oracle.e4m3_encode(mid) == even
        assert oracle.e4m3_encode(math.nextafter(mid, -math.inf)) == c_lo
        assert oracle.e4m3_encode(math.nextafter(mid, math.inf)) == c_hi
        assert oracle.e4m3_encode(-mid) == even | 0x80


def test_e4m3_matches_torch_float8_cast_on_fp32_values():
    # torch's fp32 -> float8_e4m3fn cast is round-to-nearest-even but not
    # saturating (overflow gives NaN), so compare on |x| < 464.
    rng = np.random.default_rng(7)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(64),
        (rng.standard_normal(20000) * 2.0 ** rng.integers(-14, 9, 20000)).astype(np.float32),
    ])
    x = x[np.abs(x) < 464]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in x], np.uint8)
    assert np.array_equal(got, ref)


def test_e4m3_matches_exact_brute_force_search():
    rng = np.random.default_rng(11)
    xs = list((rng.standard_normal(3000) * 2.0 ** rng.integers(-12, 10, 3000)))
    xs += [v for c in range(0x7F) for v in
           (naive_ref.E4M3_VALUES[c][0] * Fraction(3, 2),)]
    for x in xs:
        x = float(x)
        assert oracle.e4m3_encode(x) == naive_ref.e4m3_encode(x), x


# ------------------------------------------------------------------ E8M0
@pytest.mark.parametrize("row", read_golden("e8m0_hand.txt"))
def test_e8m0_hand_table(row):
    amax, b = np.float32(eval(row[0])), int(row[1])
    assert oracle.e8m0_rceil(float(amax)) == b, row


def _e8m0_by_frexp(a: float) -> int:
    """Independent computation: ceil(log2(a/448)) from frexp of the exact
    rational a/448, clamped to [-127, 127]."""
    if math.isnan(a):
        return 255
    if math.isinf(a):
        return 254
    if a == 0:
        return 0
    q = Fraction(a) / 448
    m, e = math.frexp(float(q))  # q may round in binary64; fix up exactly
    k = e if Fraction(m) != Fraction(1, 2) else e - 1  # candidate ceil(log2 q)
    while Fraction(2) ** (k - 1) >= q:
        k -= 1
    while Fraction(2) ** k < q:
        k += 1
    return max(-127, min(127, k)) + 127


def test_e8m0_against_frexp_on_random_and_boundary_amax():
    rng = np.random.default_rng(5)
    bits = rng.integers(0, 0x7F800000, size=30000, dtype=np.int64).astype(np.uint32)
    vals = list(bits.view(np.float32))
    for k in range(-127, 120):  # every fp32 threshold 448*2^k and its neighbours
        t = np.float32(448.0 * 2.0 ** k)
        vals += [t, np.nextafter(t, np.float32(np.inf)), np.nextafter(t, np.float32(0))]
    for v in vals:
        v = float(v)
        assert oracle.e8m0_rceil(v) == _e8m0_by_frexp(v), v


def test_e8m0_invariant_scaled_amax_in_upper_half_of_e4m3_range():
    # for 0 < b < 254: 224 < amax * 2^(127-b) <= 448
    rng = np.random.default_rng(9)
    for v in np.abs(rng.standard_normal(5000) * 2.0 ** rng.integers(-100, 100, 5000)):
        v = float(np.float32(v))
        b = oracle.e8m0_rceil(v)
        if 0 < b < 254:
            q = Fraction(v) * Fraction(2) ** (127 - b)
            assert 224 < q <= 448, (v, b)


def test_e8m0_power_of_two_rule():
    for k in range(-100, 120):
        assert oracle.e8m0_rceil(float(2.0 ** k)) == k + 119

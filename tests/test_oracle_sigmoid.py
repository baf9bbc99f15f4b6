"""Pins of the oracle's sigmoid: the correctly rounded fp32 value of
1/(1+exp(-g)) for every bf16 input g.

The pages characterise the activation by an exhaustive sweep over the finite
bf16 inputs (pytorch/ao PR #4743, review reply on the sigmoid: the fast sigmoid
differs from fp32 torch.sigmoid at 795 of 65,280 finite bf16 codes); the oracle
takes the exact reading of that sweep and rounds the true sigmoid once.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import naive_ref


@pytest.fixture(scope="module")
def table():
    return oracle.sigmoid_table()


def test_all_65536_inputs_match_decimal_reference(table):
    # independent: 60-digit decimal exp, exact rational rounding to fp32
    for b in range(65536):
        ref = naive_ref.sigmoid_f32(b)
        got = float(table[b])
        if math.isnan(ref):
            assert math.isnan(got), hex(b)
        else:
            assert got == ref, (hex(b), got, ref)


def test_against_torch_sigmoid_fp64_rounded(table):
    # torch's fp64 sigmoid rounded to fp32 must agree wherever binary64 can
    # decide the rounding: skip only inputs whose fp64 value lies within
    # 8 fp64 ulps of an fp32 rounding midpoint (tiny g, where sigma ~ 0.5 + g/4
    # sits on a midpoint and the -g^3/48 term is below binary64 resolution).
    g = torch.arange(65536, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    s64 = torch.sigmoid(g.to(torch.float64)).numpy()
    ref = s64.astype(np.float32)
    f = ref.astype(np.float64)
    up = np.nextafter(ref, np.float32(np.inf)).astype(np.float64)
    dn = np.nextafter(ref, np.float32(-np.inf)).astype(np.float64)
    dist = np.minimum(np.abs(s64 - (f + up) / 2), np.abs(s64 - (f + dn) / 2))
    decisive = dist > 8 * np.spacing(np.abs(s64))
    ok = (ref == table) | (np.isnan(ref) & np.isnan(table)) | ~decisive
    assert ok.all(), np.nonzero(~ok)[0][:10]
    assert decisive.sum() > 64000


def test_identities(table):
    def s(x):
        b = int(torch.tensor(x, dtype=torch.bfloat16).view(torch.int16)) & 0xFFFF
        return float(table[b])
    assert s(0.0) == 0.5 and s(-0.0) == 0.5
    assert s(float("inf")) == 1.0 and s(float("-inf")) == 0.0
    assert math.isnan(s(float("nan")))
    # sigma(g) + sigma(-g) = 1 within 2 ulps of the larger term
    for b in range(0, 0x7F80):
        sp, sn = float(table[b]), float(table[b | 0x8000])
        assert abs(sp + sn - 1.0) <= 2 * 2.0 ** -24, hex(b)


def test_saturation_regions(table):
    bits = np.arange(65536, dtype=np.uint32)
    g = (bits << 16).view(np.float32)
    fin = np.isfinite(g)
    # g >= 17.33 (1 - sigma < 2^-25): exactly 1
    assert (table[fin & (g >= 17.34)] == 1.0).all()
    # |g| < 2^-24: exactly 0.5
    assert (table[fin & (np.abs(g) < 2.0 ** -24)] == 0.5).all()
    # g < -103.98 (sigma below half the smallest subnormal): exactly 0
    assert (table[fin & (g < -104.0)] == 0.0).all()
    # subnormal sigmas exist (the CUDA path must not flush them)
    sub = table[fin & (g < -87.5) & (g > -103.0)]
    assert (sub > 0).all() and (sub < np.float32(2.0 ** -126)).all()


def test_silu_and_dsilu_special_points(table):
    b0 = 0
    sig = np.float32(table[b0])
    silu = np.float32(0.0) * sig
    dsilu = naive_ref.ffma(float(silu), float(np.float32(1) - sig), float(sig))
    assert silu == 0.0 and dsilu == 0.5
    # dsilu crosses zero near g = -1.2785 (root of 1 + g(1 - sigma(g)) = 0)
    vals = []
    for x in (-1.3125, -1.25):
        b = int(torch.tensor(x, dtype=torch.bfloat16).view(torch.int16)) & 0xFFFF
        s = float(table[b])
        si = float(np.float32(x) * np.float32(s))
        vals.append(naive_ref.ffma(si, float(np.float32(1.0) - np.float32(s)), s))
    assert vals[0] < 0 < vals[1]

"""Pins of the oracle's forward and backward (dense) against an independent
naive implementation on tiny grids, closed forms, invariants and finite
differences.

Method sources: pytorch/ao PR #4743 (Summary: SwiGLU fused with the RCEIL MXFP8
cast, rowwise 1x32 / colwise 32x1 / both; API: [gate | up] input, [dGate | dUp]
gradient; review reply: dact = fma(silu, 1 - s, s)); TransformerEngine PR #3238
(Greptile summary: per-row-scaled SReLU / SwiGLU and the scale gradient);
VeOmni PR #1340 (SiLU rounded to the activation dtype before the multiply).
"""
import math

import numpy as np
import pytest
import torch

import naive_ref
import oracle
from moe_gated_activation_b200.workloads import bf16_bits, random_case

BOTH = oracle.ROWWISE | oracle.COLWISE


def _special_case(M, N, seed, act):
    """Tiny grid mixing ordinary values with zeros, negatives, large values
    (near-overflow products), tiny values and ties."""
    width = 2 * N if act == oracle.SWIGLU else N
    c = random_case(M, N, seed, width=width, std=3.0)
    x = c["x"].float()
    g = torch.Generator().manual_seed(seed + 99)
    pick = torch.rand(x.shape, generator=g)
    x = torch.where(pick < 0.05, torch.zeros_like(x), x)
    x = torch.where((pick > 0.05) & (pick < 0.08), x * 1e-30, x)
    x = torch.where((pick > 0.08) & (pick < 0.10), x * 1e4, x)
    s = c["s"].clone()
    s[0] = 0.0          # a zero scale: codes become signed zeros
    s[1] = 2.0 ** -100  # tiny scale: tiny block amax
    return bf16_bits(x.to(torch.bfloat16)), c["s"].numpy(), s.numpy(), bf16_bits(c["dy"])


def _nested(a):
    return [list(map(int, r)) for r in a]


@pytest.mark.parametrize("act", [oracle.SWIGLU, oracle.SRELU])
@pytest.mark.parametrize("staged", [False, True])
@pytest.mark.parametrize("M,N", [(32, 32), (45, 64)])
def test_forward_matches_naive_reference(act, staged, M, N):
    if act == oracle.SRELU and staged:
        pytest.skip("staged rounding applies to SwiGLU only")
    xb, _, s, _ = _special_case(M, N, 10 + M + N, act)
    got = oracle.act_fwd(xb, s, N, BOTH, act=act, staged=staged)
    y = naive_ref.fwd_values(_nested(xb), [float(v) for v in s], N,
                             act="swiglu" if act == oracle.SWIGLU else "srelu", staged=staged)
    yo = oracle.act_values(xb, s, N, act=act, staged=staged)
    for i in range(M):
        for j in range(N):
            a, b = float(yo[i, j]), y[i][j]
            assert (a == b and math.copysign(1, a) == math.copysign(1, b)) or \
                (math.isnan(a) and math.isnan(b)), (i, j, a, b)
    ref = naive_ref.mxfp8(y, BOTH)
    for k in ("row_codes", "row_scales", "col_codes", "col_scales"):
        assert np.array_equal(got[k], np.array(ref[k], np.uint8)), k


@pytest.mark.parametrize("act", [oracle.SWIGLU, oracle.SRELU])
@pytest.mark.parametrize("M,N", [(32, 32), (37, 64)])
def test_backward_matches_naive_reference(act, M, N):
    xb, _, s, dyb = _special_case(M, N, 20 + M + N, act)
    got = oracle.act_bwd(dyb, xb, s, N, BOTH, act=act)
    dx, dsc = naive_ref.bwd_values(_nested(dyb), _nested(xb), [float(v) for v in s], N,
                                   act="swiglu" if act == oracle.SWIGLU else "srelu")
    W = len(dx[0])
    dxo = got["dx"]
    for i in range(M):
        for j in range(W):
            a = naive_ref.bf16_value(int(dxo[i, j]))
            b = dx[i][j]
            assert (a == b and math.copysign(1, a) == math.copysign(1, b)) or \
                (math.isnan(a) and math.isnan(b)), (i, j, a, b)
    for i in range(M):
        a, b = float(got["dscale"][i]), dsc[i]
        if math.isnan(b):
            assert math.isnan(a)
        else:
            assert abs(a - b) <= 1e-6 * abs(b) + 1e-30, (i, a, b)
    ref = naive_ref.mxfp8(dx, BOTH)
    for k in ("row_codes", "row_scales", "col_codes", "col_scales"):
        assert np.array_equal(got[k], np.array(ref[k], np.uint8)), k


def test_cross_mode_consistency():
    c = random_case(96, 128, 3)
    xb, s = bf16_bits(c["x"]), c["s"].numpy()
    both = oracle.act_fwd(xb, s, 128, BOTH)
    row = oracle.act_fwd(xb, s, 128, oracle.ROWWISE)
    col = oracle.act_fwd(xb, s, 128, oracle.COLWISE)
    for k in ("row_codes", "row_scales"):
        assert np.array_equal(both[k], row[k])
    for k in ("col_codes", "col_scales"):
        assert np.array_equal(both[k], col[k])
    assert row["col_codes"] is None and col["row_codes"] is None


def test_colwise_is_rowwise_of_transpose():
    rng = np.random.default_rng(4)
    y = (rng.standard_normal((64, 96)) * 2.0 ** rng.integers(-8, 8, (64, 96))).astype(np.float32)
    col = oracle.mxfp8_quantize(y, oracle.COLWISE)
    rowT = oracle.mxfp8_quantize(np.ascontiguousarray(y.T), oracle.ROWWISE)
    assert np.array_equal(col["col_codes"], rowT["row_codes"].T)
    assert np.array_equal(col["col_scales"], rowT["row_scales"].T)


def test_power_of_two_blocks_and_signs():
    k = np.arange(-20, 12)
    y = np.zeros((32, 32), np.float32)
    for i in range(32):
        sign = np.where(np.arange(32) % 3 == 0, -1.0, 1.0)
        y[i] = (sign * 2.0 ** k[i]).astype(np.float32)
    out = oracle.mxfp8_quantize(y, oracle.ROWWISE)
    assert np.array_equal(out["row_scales"][:, 0], (k + 119).astype(np.uint8))
    exp = np.where(np.arange(32) % 3 == 0, 0xF8, 0x78).astype(np.uint8)
    assert (out["row_codes"] == exp[None, :]).all()


def test_zero_nan_inf_blocks():
    y = np.zeros((32, 128), np.float32)
    y[:, 32:64] = -0.0
    y[:, 64:96] = 1.0
    y[5, 70] = np.nan
    y[:, 96:128] = 3.0
    y[7, 100] = np.inf
    y[8, 101] = -np.inf
    out = oracle.mxfp8_quantize(y, oracle.ROWWISE)
    rs, rq = out["row_scales"], out["row_codes"]
    assert (rs[:, 0] == 0).all() and (rq[:, 0:32] == 0x00).all()
    assert (rs[:, 1] == 0).all() and (rq[:, 32:64] == 0x80).all()
    assert rs[5, 2] == 255 and (rq[5, 64:96] == 0x7F).all()
    assert rs[4, 2] == 119 and (rq[4, 64:96] == 0x78).all()
    assert rs[7, 3] == 254 and rq[7, 100] == 0x7E and (rq[7, 96:100] == 0).all()
    assert rs[8, 3] == 254 and rq[8, 101] == 0xFE


def test_max_code_and_dequantisation_error():
    rng = np.random.default_rng(8)
    y = (rng.standard_normal((64, 256)) * 2.0 ** rng.integers(-30, 30, (64, 1))).astype(np.float32)
    out = oracle.mxfp8_quantize(y, oracle.ROWWISE | oracle.COLWISE)
    dec = np.vectorize(oracle.e4m3_decode)
    for q, sc, axis in ((out["row_codes"], np.repeat(out["row_scales"], 32, axis=1), 1),
                        (out["col_codes"], np.repeat(out["col_scales"], 32, axis=0), 0)):
        mag = q & 0x7F
        blocks = mag.reshape(64, 8, 32).max(axis=2) if axis == 1 else \
            mag.reshape(2, 32, 256).max(axis=1)
        assert ((blocks >= 0x76) & (blocks <= 0x7E)).all()
        v = dec(q) * np.exp2(sc.astype(np.float64) - 127)
        # error at most half an E4M3 step at the value's magnitude
        mant = np.maximum(np.abs(y.astype(np.float64)) * np.exp2(127 - sc.astype(np.float64)),
                          2.0 ** -6)
        half_step = np.exp2(np.floor(np.log2(mant)) - 4) * np.exp2(sc.astype(np.float64) - 127)
        assert (np.abs(v - y) <= half_step * (1 + 1e-12)).all()


def _fwd64(g, u, s):
    return g / (1.0 + np.exp(-g)) * u * s[:, None]


@pytest.mark.parametrize("act", [oracle.SWIGLU, oracle.SRELU])
def test_backward_against_finite_differences(act):
    M, N = 8, 32
    c = random_case(M, N, 77, width=2 * N if act == oracle.SWIGLU else N)
    xb, s, dyb = bf16_bits(c["x"]), c["s"].numpy(), bf16_bits(c["dy"])
    out = oracle.act_bwd(dyb, xb, s, N, oracle.ROWWISE, act=act)
    x = c["x"].double().numpy()
    dy = c["dy"].double().numpy()
    sd = s.astype(np.float64)
    h = 1e-6
    if act == oracle.SWIGLU:
        g, u = x[:, :N], x[:, N:]
        L = lambda g_, u_, s_: (dy * _fwd64(g_, u_, s_)).sum()
        dg = np.zeros_like(g); du = np.zeros_like(u)
        for i in range(M):
            for j in range(N):
                e = np.zeros_like(g); e[i, j] = h
                dg[i, j] = (L(g + e, u, sd) - L(g - e, u, sd)) / (2 * h)
                du[i, j] = (L(g, u + e, sd) - L(g, u - e, sd)) / (2 * h)
        ref = np.concatenate([dg, du], axis=1)
        dsc = np.array([(dy[i] * (g[i] / (1 + np.exp(-g[i])) * u[i])).sum() for i in range(M)])
    else:
        r = np.maximum(x, 0)
        ref = dy * sd[:, None] * 2 * r
        dsc = (dy * r * r).sum(axis=1)
    got = np.array([[oracle.bf16_to_f32(int(b)) for b in row] for row in out["dx"]])
    # bf16 rounding of the result: relative 2^-8 plus fp32 chain error
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6)
    assert np.allclose(out["dscale"], dsc, rtol=1e-5, atol=1e-6)


def test_dscale_identity_with_dup():
    M, N = 16, 64
    c = random_case(M, N, 5, s_low=0.1, s_high=1.0)
    xb, s, dyb = bf16_bits(c["x"]), c["s"].numpy(), bf16_bits(c["dy"])
    out = oracle.act_bwd(dyb, xb, s, N, oracle.ROWWISE)
    dup = np.array([[oracle.bf16_to_f32(int(b)) for b in row[N:]] for row in out["dx"]])
    u = c["x"][:, N:].double().numpy()
    est = (dup * u).sum(axis=1) / s
    assert np.allclose(est, out["dscale"], rtol=2e-2, atol=2e-2)

"""Pins of the oracle's ClampedSwiGLU (reading: gc = min(g, L), uc =
clamp(u, -L, L), sigma of RN(alpha * gc) correctly rounded, h =
RN(RN(gc * sigma) * RN(uc + 1)); backward in the SwiGLU form with slope
alpha and zero gradient where an input was clamped).

Pinned against: the SwiGLU oracle (alpha = 1, L = +Inf, up values with u + 1
exact in bf16 -- a different sigma path: the bf16 table instead of sigma of an
fp32 argument), an independent exact-arithmetic reference on tiny grids with
clamped, NaN and tiny inputs, the clamp's plateau and zero gradients, and fp64
finite differences of the definition."""
import math

import numpy as np
import pytest
import torch

import naive_ref
import oracle
from moe_gated_activation_b200.workloads import bf16_bits, random_case

BOTH = oracle.ROWWISE | oracle.COLWISE
INF = float("inf")


def _bits(t):
    return bf16_bits(t.to(torch.bfloat16))


def _case(M, N, seed, scale=4.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, 2 * N, generator=g) * scale
    s = torch.rand(M, generator=g) + 0.05
    dy = torch.randn(M, N, generator=g)
    return x, s, dy


def test_reduces_to_swiglu_with_up_plus_one():
    M, N = 32, 64
    g = torch.Generator().manual_seed(3)
    gate = torch.randn(M, N, generator=g) * 5
    k = torch.randint(-64, 65, (M, N), generator=g).float()
    u = k / 8                                  # u + 1 is exact in bf16
    x = torch.cat([gate, u], dim=1)
    x_sw = torch.cat([gate, u + 1], dim=1)
    xb, xb_sw = _bits(x), _bits(x_sw)
    assert np.array_equal(xb_sw[:, N:], _bits(u + 1))
    s = (torch.rand(M, generator=g) + 0.1).numpy()
    dyb = _bits(torch.randn(M, N, generator=g))
    y = oracle.clamped_values(xb, s, N, alpha=1.0, limit=INF)
    y_sw = oracle.act_values(xb_sw, s, N)
    assert np.array_equal(y.view(np.uint32), y_sw.view(np.uint32))
    a = oracle.clamped_bwd(dyb, xb, s, N, BOTH, alpha=1.0, limit=INF)
    b = oracle.act_bwd(dyb, xb_sw, s, N, BOTH)
    for k_ in ("dx", "row_codes", "row_scales", "col_codes", "col_scales"):
        assert np.array_equal(a[k_], b[k_]), k_
    assert np.array_equal(a["dscale"].view(np.uint32), b["dscale"].view(np.uint32))


@pytest.mark.parametrize("alpha,L", [(1.702, 7.0), (1.0, 2.5), (2.0, 0.75), (0.8125, INF)])
def test_matches_the_exact_reference_on_tiny_grids(alpha, L):
    M, N = 16, 32
    x, s, dy = _case(M, N, seed=int(alpha * 100 + (L if L != INF else 99)))
    x[0, :N] = L + 3.0            # clamped gates (a plateau, zero gradient)
    x[1, N:] = L + 1.0            # clamped ups
    x[2, N:] = -L - 1.0
    x[3, 5] = float("nan")
    x[4, N + 6] = float("nan")
    x[5, :N] *= 1e-30             # tiny gates: sigma = 0.5
    x[6, :N] = 0.0
    xb, sv, dyb = _bits(x), s.numpy(), _bits(dy)
    alpha32 = float(np.float32(alpha))
    L32 = float(np.float32(L))
    y = oracle.clamped_values(xb, sv, N, alpha=alpha32, limit=L32)
    ref = naive_ref.clamped_fwd_values([list(map(int, r)) for r in xb], [float(v) for v in sv],
                                       N, alpha32, L32)
    for i in range(M):
        for j in range(N):
            a, b = float(y[i, j]), ref[i][j]
            assert (a == b and math.copysign(1, a) == math.copysign(1, b)) or \
                (math.isnan(a) and math.isnan(b)), (i, j, a, b)
    out = oracle.clamped_bwd(dyb, xb, sv, N, BOTH, alpha=alpha32, limit=L32)
    dx, dsc = naive_ref.clamped_bwd_values([list(map(int, r)) for r in dyb],
                                           [list(map(int, r)) for r in xb],
                                           [float(v) for v in sv], N, alpha32, L32)
    for i in range(M):
        for j in range(2 * N):
            a, b = naive_ref.bf16_value(int(out["dx"][i, j])), dx[i][j]
            assert (a == b and math.copysign(1, a) == math.copysign(1, b)) or \
                (math.isnan(a) and math.isnan(b)), (i, j, a, b)
        if math.isnan(dsc[i]):
            assert math.isnan(out["dscale"][i])
        else:
            assert abs(float(out["dscale"][i]) - dsc[i]) <= 1e-6 * abs(dsc[i]) + 1e-30
    mx = naive_ref.mxfp8(dx, BOTH)
    for k in ("row_codes", "row_scales", "col_codes", "col_scales"):
        assert np.array_equal(out[k], np.array(mx[k], np.uint8)), k


def test_clamp_plateau_and_zero_gradients():
    M, N, L = 4, 32, 7.0
    x, s, dy = _case(M, N, seed=5, scale=1.0)
    x[:, 0] = 7.0
    x[:, 1] = 9.0          # clamped to 7: same value as column 0's gate
    x[:, N + 0] = 0.5
    x[:, N + 1] = 0.5
    x[:, N + 2] = 20.0     # up clamped to +7
    x[:, N + 3] = 7.0
    x[:, N + 4] = -30.0    # up clamped to -7
    x[:, N + 5] = -7.0
    x[:, 2] = x[:, 3] = x[:, 4] = x[:, 5] = 1.5
    xb, sv, dyb = _bits(x), s.numpy(), _bits(dy)
    y = oracle.clamped_values(xb, sv, N, limit=L)
    assert np.array_equal(y[:, 0], y[:, 1])
    assert np.array_equal(y[:, 2], y[:, 3]) and np.array_equal(y[:, 4], y[:, 5])
    d = oracle.clamped_bwd(dyb, xb, sv, N, oracle.ROWWISE, limit=L)["dx"]
    assert (d[:, 1] == 0).all()                       # dgate of a clamped gate
    assert (d[:, 0] != 0).any()                       # g == L still has a gradient
    assert (d[:, N + 2] == 0).all() and (d[:, N + 4] == 0).all()
    assert (d[:, N + 3] != 0).any() and (d[:, N + 5] != 0).any()


def _h64(g, u, alpha, L):
    gc = np.minimum(g, L)
    uc = np.clip(u, -L, L)
    return gc / (1.0 + np.exp(-alpha * gc)) * (uc + 1.0)


def test_backward_against_finite_differences():
    M, N, alpha, L = 6, 32, 1.702, 7.0
    c = random_case(M, N, 41, std=1.0)
    c["x"] = c["x"].clamp(-6.5, 6.5)
    xb, s, dyb = bf16_bits(c["x"]), c["s"].numpy(), bf16_bits(c["dy"])
    out = oracle.clamped_bwd(dyb, xb, s, N, oracle.ROWWISE, alpha=alpha, limit=L)
    x = c["x"].double().numpy()
    dy = c["dy"].double().numpy()
    sd = s.astype(np.float64)
    g, u = x[:, :N], x[:, N:]
    assert (np.abs(g) < L - 0.1).all() and (np.abs(u) < L - 0.1).all()
    loss = lambda g_, u_: (dy * _h64(g_, u_, alpha, L) * sd[:, None]).sum()
    hh = 1e-6
    dg, du = np.zeros_like(g), np.zeros_like(u)
    for i in range(M):
        for j in range(N):
            e = np.zeros_like(g); e[i, j] = hh
            dg[i, j] = (loss(g + e, u) - loss(g - e, u)) / (2 * hh)
            du[i, j] = (loss(g, u + e) - loss(g, u - e)) / (2 * hh)
    ref = np.concatenate([dg, du], axis=1)
    got = np.array([[oracle.bf16_to_f32(int(b)) for b in row] for row in out["dx"]])
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6)
    dsc = (dy * _h64(g, u, alpha, L)).sum(axis=1)
    assert np.allclose(out["dscale"], dsc, rtol=1e-5, atol=1e-6)


def test_argument_range():
    xb = np.zeros((32, 64), np.uint16)
    s = np.ones(32, np.float32)
    for alpha, L in ((0.5, 7.0), (2.5, 7.0), (1.0, 0.0), (1.0, -1.0), (1.0, float("nan"))):
        with pytest.raises(ValueError):
            oracle.clamped_fwd(xb, s, 32, BOTH, alpha=alpha, limit=L)


def test_sigmoid_table_of_a_slope():
    """sigma(RN(alpha * g)) over bf16 g: alpha = 1 gives the SwiGLU table;
    for alpha = 1.702 a sample of gates (every 97th pattern, and the window
    edges) against the exact reference."""
    t1 = oracle.clamped_sigmoid_table(1.0)
    ref = oracle.sigmoid_table()
    fin = ~np.isnan(ref)
    assert np.array_equal(t1.view(np.uint32)[fin], ref.view(np.uint32)[fin])
    alpha = float(np.float32(1.702))
    t = oracle.clamped_sigmoid_table(alpha)
    sample = sorted(set(range(0, 65536, 97)) | {0x3300, 0x32FF, 0x42FF, 0x4300, 0xB300, 0xC2FF})
    for b in sample:
        g = naive_ref.bf16_value(b)
        if math.isnan(g):
            continue
        want = naive_ref.sigmoid_of(naive_ref.fmul(alpha, g))
        assert float(t[b]) == want, (hex(b), float(t[b]), want)

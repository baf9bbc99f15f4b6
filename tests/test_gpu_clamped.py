"""ClampedSwiGLU on the GPU against the oracle: the per-slope sigmoid table on
all bf16 gates, forward and backward parity (dense, grouped, ragged, special
values, both scale layouts), at several (alpha, limit)."""

import numpy as np
import pytest
import torch

import oracle
import moe_gated_activation_b200 as mg
from moe_gated_activation_b200 import _capi
from moe_gated_activation_b200.workloads import bf16_bits
from parity import assert_bf16_close, assert_dscale, bf16_u16, compare_mx

pytestmark = pytest.mark.gpu

INF = float("inf")
# 3.3 is not a bf16 value: a bf16 gate or up lies above it exactly when it
# lies above 3.296875, the bf16 below it
PARAMS = [(1.702, 7.0), (1.0, 2.5), (2.0, 0.75), (0.8125, INF), (1.0, 3.3)]
SHAPES = [(32, 32), (96, 224), (100, 192), (257, 320)]


def _f32(v):
    return float(np.float32(v))


def _case(M, N, seed, scale=4.0):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(M, 2 * N, generator=g) * scale).to(torch.bfloat16)
    s = torch.rand(M, generator=g) + 0.05
    dy = torch.randn(M, N, generator=g).to(torch.bfloat16)
    return x, s, dy


def _dscale_bound(dyb, xb, s, N, alpha, L):
    """sum_j |dY * h| per row in float64, h from the oracle's definition."""
    y = oracle.clamped_values(xb, np.ones_like(s), N, alpha=alpha, limit=L).astype(np.float64)
    dy = torch.from_numpy(dyb.view(np.int16)).view(torch.bfloat16).double().numpy()[:, :N]
    return np.abs(dy * y).sum(axis=1)


@pytest.mark.parametrize("alpha", [1.702, 1.0, 0.8125, 2.0])
def test_sigmoid_table_of_a_slope_on_all_bf16(cuda_device, alpha):
    a = _f32(alpha)
    got = mg.clamped_sigmoid_table(a, device=cuda_device).cpu().numpy()
    ref = oracle.clamped_sigmoid_table(a)
    bits = np.arange(65536, dtype=np.uint32)
    is_nan = ((bits & 0x7F80) == 0x7F80) & ((bits & 0x7F) != 0)
    same = got.view(np.uint32) == ref.view(np.uint32)
    assert same[~is_nan].all(), np.nonzero(~same & ~is_nan)[0][:10]


@pytest.mark.parametrize("alpha,L", [(1.702, 7.0), (2.0, 0.75), (0.8125, 0.015625)])
def test_sigmoid_table_with_the_gate_clamp_on_all_bf16(cuda_device, alpha, L):
    """The table a call with a finite limit looks up: sigma(RN(alpha * min(g,
    L))), i.e. the oracle's unclamped entry of the gate, or of L (a bf16
    value here) for every gate above L."""
    a = _f32(alpha)
    got = mg.clamped_sigmoid_table(a, L, device=cuda_device).cpu().numpy()
    ref = oracle.clamped_sigmoid_table(a)
    bits = np.arange(65536, dtype=np.uint32)
    g = (bits << 16).view(np.float32)
    lbits = int(np.array([L], np.float32).view(np.uint32)[0] >> 16)
    want = np.where(g > L, ref[lbits], ref)
    is_nan = np.isnan(g)
    same = got.view(np.uint32) == want.view(np.uint32)
    assert same[~is_nan].all(), np.nonzero(~same & ~is_nan)[0][:10]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("alpha,L", PARAMS)
def test_forward_and_backward_parity(cuda_device, alpha, L, shape):
    M, N = shape
    a, l = _f32(alpha), _f32(L)
    x, s, dy = _case(M, N, seed=M * 3 + N + int(alpha * 10))
    xb, sn, dyb = bf16_bits(x), s.numpy(), bf16_bits(dy)
    xg, sg, dyg = x.to(cuda_device), s.to(cuda_device), dy.to(cuda_device)
    got = mg.scaled_clamped_swiglu_mxfp8_fwd(xg, sg, alpha=a, limit=l)
    gotb = mg.scaled_clamped_swiglu_mxfp8_bwd(dyg, xg, sg, alpha=a, limit=l)
    torch.cuda.synchronize()
    what = f"clamped a={a} L={l} {shape}"
    ref = oracle.clamped_fwd(xb, sn, N, 3, alpha=a, limit=l)
    compare_mx(got, ref, what + " fwd", exact=True)
    refb = oracle.clamped_bwd(dyb, xb, sn, N, 3, alpha=a, limit=l)
    compare_mx(gotb.mx, refb, what + " bwd", exact=True)
    assert np.array_equal(bf16_u16(gotb.dx), refb["dx"]), what + " dx"
    assert_dscale(gotb.dscale, refb["dscale"], _dscale_bound(dyb, xb, sn, N, a, l), what + " dscale")


def test_special_values(cuda_device):
    M, N, a, l = 64, 128, _f32(1.702), 7.0
    x, s, dy = _case(M, N, seed=9)
    x = x.float()
    x[0, :N] = 9.0                   # clamped gates
    x[1, N:] = 30.0                  # clamped ups
    x[2, N:] = -30.0
    x[3, :N] = 7.0                   # exactly at the limit
    x[4, 5] = float("nan")
    x[5, N + 6] = float("nan")
    x[6, 7] = float("inf")
    x[7, 8] = float("-inf")
    x[8, N + 9] = float("inf")
    x[9, :N] = 0.0
    x[10, :N] *= 1e-30
    x[11, :N] = -200.0
    x = x.to(torch.bfloat16)
    s = s.clone()
    s[12] = 0.0
    s[13] = -0.5
    # non-finite dY where the gate (row 0) or the up (rows 1, 2) is clamped:
    # the clamped input's gradient is +0 all the same
    dy = dy.float()
    dy[0, 3], dy[0, 4], dy[1, 5], dy[2, 6] = float("nan"), float("inf"), float("nan"), -float("inf")
    dy = dy.to(torch.bfloat16)
    xb, sn, dyb = bf16_bits(x), s.numpy(), bf16_bits(dy)
    xg, sg, dyg = x.to(cuda_device), s.to(cuda_device), dy.to(cuda_device)
    got = mg.scaled_clamped_swiglu_mxfp8_fwd(xg, sg, alpha=a, limit=l)
    gotb = mg.scaled_clamped_swiglu_mxfp8_bwd(dyg, xg, sg, alpha=a, limit=l)
    torch.cuda.synchronize()
    compare_mx(got, oracle.clamped_fwd(xb, sn, N, 3, alpha=a, limit=l), "special fwd", exact=True)
    refb = oracle.clamped_bwd(dyb, xb, sn, N, 3, alpha=a, limit=l)
    compare_mx(gotb.mx, refb, "special bwd", exact=True)
    # NaN results may carry another sign or payload (inf * 0 gives the
    # host's default NaN in the oracle): NaN positions must match
    assert_bf16_close(bf16_u16(gotb.dx), refb["dx"], "special dx", ulps=0)
    gd, rd = gotb.dscale.cpu().numpy(), refb["dscale"]
    assert np.array_equal(np.isnan(gd), np.isnan(rd)) and np.array_equal(np.isinf(gd), np.isinf(rd))
    fin = np.isfinite(rd)
    assert_dscale(gd[fin], rd[fin], _dscale_bound(dyb, xb, sn, N, a, l)[fin], "special dscale")


@pytest.mark.parametrize("gemm", [False, True])
def test_grouped_parity(cuda_device, gemm):
    N, a, l = 128, _f32(1.702), 7.0
    m = np.array([256, 0, 128, 384], np.int64) if gemm else np.array([5, 40, 0, 33, 1, 49, 0, 17])
    M = int(m.sum())
    x, s, dy = _case(M, N, seed=21)
    xb, sn, dyb = bf16_bits(x), s.numpy(), bf16_bits(dy)
    _, ro, cb = oracle.splits_to_offsets(m, M)
    gro, gcb, _ = mg.splits_to_offsets(torch.from_numpy(m).to(cuda_device), M)
    xg, sg, dyg = x.to(cuda_device), s.to(cuda_device), dy.to(cuda_device)
    S = int(cb[-1])
    got, st = mg.grouped_scaled_clamped_swiglu_mxfp8_fwd(xg, sg, gro, gcb, alpha=a, limit=l,
                                                         col_scale_rows=S, gemm_scales=gemm)
    gotb, stb = mg.grouped_scaled_clamped_swiglu_mxfp8_bwd(dyg, xg, sg, gro, gcb, alpha=a, limit=l,
                                                           col_scale_rows=S, gemm_scales=gemm)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and int(stb.item()) == 0
    ref = oracle.grouped_clamped_fwd(xb, sn, N, 3, ro, cb, alpha=a, limit=l)
    refb = oracle.grouped_clamped_bwd(dyb, xb, sn, N, 3, ro, cb, alpha=a, limit=l)
    if gemm:
        for r, W in ((ref, N), (refb, 2 * N)):
            r["row_scales"] = oracle.scales_gemm_layout(r["row_scales"]).reshape(M, W // 32)
            r["col_scales"] = oracle.col_scales_gemm_layout(r["col_scales"], W, ro, cb).reshape(
                S, W)
    compare_mx(got, ref, f"grouped clamped fwd gemm={gemm}", exact=True)
    compare_mx(gotb.mx, refb, f"grouped clamped bwd gemm={gemm}", exact=True)
    assert np.array_equal(bf16_u16(gotb.dx), refb["dx"])
    assert_dscale(gotb.dscale, refb["dscale"], _dscale_bound(dyb, xb, sn, N, a, l),
                  "grouped clamped dscale")


def test_backward_without_dx_matches(cuda_device):
    """dX not requested: the tile stays in registers (the other kernel
    variant); the MXFP8 of the gradient and dscale must not change."""
    M, N, a, l = 96, 224, _f32(1.702), 7.0
    x, s, dy = _case(M, N, seed=33)
    xb, sn, dyb = bf16_bits(x), s.numpy(), bf16_bits(dy)
    got = mg.scaled_clamped_swiglu_mxfp8_bwd(dy.to(cuda_device), x.to(cuda_device),
                                             s.to(cuda_device), alpha=a, limit=l, want_dx=False)
    torch.cuda.synchronize()
    refb = oracle.clamped_bwd(dyb, xb, sn, N, 3, alpha=a, limit=l)
    compare_mx(got.mx, refb, "clamped bwd without dx", exact=True)
    assert got.dx is None


def test_argument_errors(cuda_device):
    x = torch.zeros(32, 64, dtype=torch.bfloat16, device=cuda_device)
    s = torch.ones(32, device=cuda_device)
    for alpha, limit in ((0.5, 7.0), (2.5, 7.0), (1.0, 0.0), (1.0, float("nan"))):
        with pytest.raises(_capi.MoeactError) as e:
            mg.scaled_clamped_swiglu_mxfp8_fwd(x, s, alpha=alpha, limit=limit)
        assert e.value.status == _capi.EINVAL

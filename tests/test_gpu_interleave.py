"""Interleaved gate / up columns (glu_interleave = G) on the GPU against the
oracle, bitwise: dense and grouped, SwiGLU (plain and staged) and
ClampedSwiGLU, G = 32, 64, 128, 256 and G = N, a ragged last column tile,
ragged groups, the backward with and without dX, and the GEMM-ready scale
layout."""
import numpy as np
import pytest
import torch

import oracle
import moe_gated_activation_b200 as mg
from moe_gated_activation_b200 import _capi
from moe_gated_activation_b200.workloads import bf16_bits, random_case
from parity import (assert_bf16_close, assert_dscale, bf16_u16, compare_mx, dscale_abs_bound,
                    u8)

pytestmark = pytest.mark.gpu


def _case(M, N, seed, dev):
    c = random_case(M, N, seed, std=2.0)
    host = bf16_bits(c["x"]), c["s"].numpy(), bf16_bits(c["dy"])
    return host, (c["x"].to(dev), c["s"].to(dev), c["dy"].to(dev))


def _dx_compare(got, ref, act, what):
    if act == "clamped":
        assert_bf16_close(bf16_u16(got), ref, what, ulps=0)
    else:
        assert np.array_equal(bf16_u16(got), ref), what


def _fwd(act, x, s, G, **kw):
    if act == "clamped":
        return mg.scaled_clamped_swiglu_mxfp8_fwd(x, s, glu_interleave=G, **kw)
    return mg.scaled_swiglu_mxfp8_fwd(x, s, glu_interleave=G, **kw)


def _bwd(act, dy, x, s, G, **kw):
    if act == "clamped":
        return mg.scaled_clamped_swiglu_mxfp8_bwd(dy, x, s, glu_interleave=G, **kw)
    return mg.scaled_swiglu_mxfp8_bwd(dy, x, s, glu_interleave=G, **kw)


@pytest.mark.parametrize("act", ["swiglu", "clamped"])
@pytest.mark.parametrize("M,N,G", [(200, 512, 32), (200, 512, 64), (200, 512, 128),
                                   (200, 512, 256), (96, 512, 512), (70, 224, 32),
                                   (70, 192, 64), (33, 1024, 32)])
def test_dense(cuda_device, act, M, N, G):
    (xb, s, dyb), (x, sg, dy) = _case(M, N, M + N + G, cuda_device)
    got = _fwd(act, x, sg, G)
    gotb = _bwd(act, dy, x, sg, G)
    torch.cuda.synchronize()
    what = f"{act} {M}x{N} G={G}"
    compare_mx(got, oracle.interleaved_fwd(xb, s, N, 3, G, act=act), what + " fwd")
    ref = oracle.interleaved_bwd(dyb, xb, s, N, 3, G, act=act)
    compare_mx(gotb.mx, ref, what + " bwd")
    _dx_compare(gotb.dx, ref["dx"], act, what + " dx")
    assert_dscale(gotb.dscale, ref["dscale"],
                  dscale_abs_bound(dyb, oracle.glu_halves(xb, N, G), s, N), what + " dscale")


@pytest.mark.parametrize("G", [32, 128])
@pytest.mark.parametrize("dirs", [1, 2, 3])
def test_backward_without_dx(cuda_device, G, dirs):
    """dX not requested: the backward keeps the whole tile in registers."""
    M, N = 100, 384
    (xb, s, dyb), (x, sg, dy) = _case(M, N, 5 + G, cuda_device)
    gotb = mg.scaled_swiglu_mxfp8_bwd(dy, x, sg, rowwise=bool(dirs & 1),
                                      colwise=bool(dirs & 2), want_dx=False, glu_interleave=G)
    torch.cuda.synchronize()
    ref = oracle.interleaved_bwd(dyb, xb, s, N, dirs, G)
    compare_mx(gotb.mx, ref, f"bwd no dx G={G} dirs={dirs}")
    assert gotb.dx is None


def test_staged_forward(cuda_device):
    M, N, G = 64, 256, 32
    (xb, s, _), (x, sg, _) = _case(M, N, 77, cuda_device)
    got = mg.scaled_swiglu_mxfp8_fwd(x, sg, staged_rounding=True, glu_interleave=G)
    torch.cuda.synchronize()
    compare_mx(got, oracle.interleaved_fwd(xb, s, N, 3, G, staged=True), "staged G=32")


@pytest.mark.parametrize("act", ["swiglu", "clamped"])
@pytest.mark.parametrize("G", [32, 64, 256])
def test_grouped(cuda_device, act, G):
    N = 512
    m = np.array([70, 0, 33, 128, 1, 64], np.int64)
    M = int(m.sum())
    (xb, s, dyb), (x, sg, dy) = _case(M, N, 300 + G, cuda_device)
    _, ro, cb = oracle.splits_to_offsets(m, M)
    gro, gcb, _ = mg.splits_to_offsets(torch.from_numpy(m).to(cuda_device), M)
    S = int(cb[-1])
    if act == "clamped":
        got, st = mg.grouped_scaled_clamped_swiglu_mxfp8_fwd(x, sg, gro, gcb, col_scale_rows=S,
                                                             glu_interleave=G)
        gotb, stb = mg.grouped_scaled_clamped_swiglu_mxfp8_bwd(dy, x, sg, gro, gcb,
                                                               col_scale_rows=S, glu_interleave=G)
    else:
        got, st = mg.grouped_scaled_swiglu_mxfp8_fwd(x, sg, gro, gcb, col_scale_rows=S,
                                                     glu_interleave=G)
        gotb, stb = mg.grouped_scaled_swiglu_mxfp8_bwd(dy, x, sg, gro, gcb, col_scale_rows=S,
                                                       glu_interleave=G)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and int(stb.item()) == 0
    what = f"grouped {act} G={G}"
    compare_mx(got, oracle.interleaved_fwd(xb, s, N, 3, G, act=act, row_offs=ro,
                                           colblk_offs=cb), what + " fwd")
    ref = oracle.interleaved_bwd(dyb, xb, s, N, 3, G, act=act, row_offs=ro, colblk_offs=cb)
    compare_mx(gotb.mx, ref, what + " bwd")
    _dx_compare(gotb.dx, ref["dx"], act, what + " dx")


@pytest.mark.parametrize("G", [32, 64, 128])
def test_gemm_layout(cuda_device, G):
    N = 256
    m = np.array([128, 0, 256, 128], np.int64)
    M = int(m.sum())
    (xb, s, dyb), (x, sg, dy) = _case(M, N, 900 + G, cuda_device)
    _, ro, cb = oracle.splits_to_offsets(m, M)
    gro, gcb, _ = mg.splits_to_offsets(torch.from_numpy(m).to(cuda_device), M)
    S = int(cb[-1])
    got, st = mg.grouped_scaled_swiglu_mxfp8_fwd(x, sg, gro, gcb, col_scale_rows=S,
                                                 gemm_scales=True, glu_interleave=G)
    gotb, stb = mg.grouped_scaled_swiglu_mxfp8_bwd(dy, x, sg, gro, gcb, col_scale_rows=S,
                                                   gemm_scales=True, glu_interleave=G)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and int(stb.item()) == 0
    for res, ref, W in ((got, oracle.interleaved_fwd(xb, s, N, 3, G, row_offs=ro,
                                                     colblk_offs=cb), N),
                        (gotb.mx, oracle.interleaved_bwd(dyb, xb, s, N, 3, G, row_offs=ro,
                                                         colblk_offs=cb), 2 * N)):
        rs = oracle.scales_gemm_layout(ref["row_scales"])
        cs = oracle.col_scales_gemm_layout(ref["col_scales"], W, ro, cb)
        assert np.array_equal(u8(res.row_scales).reshape(-1), rs), f"G={G} W={W} row scales"
        assert np.array_equal(u8(res.col_scales).reshape(-1)[:cs.size], cs), f"G={G} col scales"
        assert np.array_equal(u8(res.row_codes), ref["row_codes"])
        assert np.array_equal(u8(res.col_codes), ref["col_codes"])


def test_bad_interleave(cuda_device):
    (_, _, _), (x, sg, dy) = _case(32, 384, 1, cuda_device)
    for G in (16, 96, 100, -32, 256):   # 96 and 256 do not qualify for N = 384
        with pytest.raises(_capi.MoeactError):
            mg.scaled_swiglu_mxfp8_fwd(x, sg, glu_interleave=G)
        with pytest.raises(_capi.MoeactError):
            mg.scaled_swiglu_mxfp8_bwd(dy, x, sg, glu_interleave=G)


def test_strided_input_and_g_equal_n(cuda_device):
    """x with a row stride wider than 2N, and G = N (the halves layout)."""
    M, N, G = 64, 256, 32
    (xb, s, dyb), (x, sg, dy) = _case(M, N, 404, cuda_device)
    wide = torch.zeros(M, 2 * N + 64, dtype=torch.bfloat16, device=cuda_device)
    wide[:, :2 * N] = x
    xs = wide[:, :2 * N]
    got = mg.scaled_swiglu_mxfp8_fwd(xs, sg, glu_interleave=G)
    gotb = mg.scaled_swiglu_mxfp8_bwd(dy, xs, sg, glu_interleave=G)
    halves = mg.scaled_swiglu_mxfp8_fwd(x, sg, glu_interleave=N)
    torch.cuda.synchronize()
    compare_mx(got, oracle.interleaved_fwd(xb, s, N, 3, G), "strided fwd")
    ref = oracle.interleaved_bwd(dyb, xb, s, N, 3, G)
    compare_mx(gotb.mx, ref, "strided bwd")
    assert np.array_equal(bf16_u16(gotb.dx), ref["dx"])
    compare_mx(halves, oracle.act_fwd(xb, s, N, 3), "G = N")


def test_noop_flag_and_empty_input(cuda_device):
    """A set no-op flag writes nothing with an interleaved input either; an
    empty input launches nothing."""
    M, N, G = 64, 256, 64
    (_, _, _), (x, sg, dy) = _case(M, N, 505, cuda_device)
    flag = torch.ones(1, dtype=torch.int32, device=cuda_device)
    stream = torch.cuda.current_stream(cuda_device).cuda_stream
    ws = torch.zeros(mg.bwd_workspace_bytes(M, N), dtype=torch.uint8, device=cuda_device)
    for W in (N, 2 * N):
        u8_ = dict(dtype=torch.uint8, device=cuda_device)
        o = [torch.full((M, W), 0xA5, **u8_), torch.full((M, W // 32), 0xA5, **u8_),
             torch.full((M, W), 0xA5, **u8_), torch.full(((M + 31) // 32, W), 0xA5, **u8_)]
        dx = torch.full((M, 2 * N), -7.0, dtype=torch.bfloat16, device=cuda_device)
        dscale = torch.full((M,), -7.0, device=cuda_device)
        mx = _capi.MxOut(*(t.data_ptr() for t in o), _capi.SCALES_ROWMAJOR, flag.data_ptr())
        if W == N:
            _capi.call("scaled_swiglu_mxfp8_fwd", x.data_ptr(), 2 * N, sg.data_ptr(), M, N, 3, 0,
                       G, mx, stream)
        else:
            _capi.call("scaled_swiglu_mxfp8_bwd", dy.data_ptr(), N, x.data_ptr(), 2 * N,
                       sg.data_ptr(), M, N, 3, G, dx.data_ptr(), dscale.data_ptr(), mx,
                       ws.data_ptr(), ws.numel(), stream)
        torch.cuda.synchronize()
        assert all(bool((t == 0xA5).all()) for t in o)
        assert bool((dx == -7.0).all()) and bool((dscale == -7.0).all())
    e = mg.scaled_swiglu_mxfp8_fwd(x[:0], sg[:0], glu_interleave=G)
    torch.cuda.synchronize()
    assert e.row_codes.numel() == 0

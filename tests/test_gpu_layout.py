"""The GEMM-ready scale layout (MOEACT_SCALES_GEMM) on the GPU against the
oracle: small dense and grouped cases bitwise (scales laid out by the
oracle's layout functions; codes, dX and dscale as in the row-major layout),
the workload sizes whose groups are 128-aligned on sampled slabs, and the
alignment errors."""
import numpy as np
import pytest
import torch

import oracle
import moe_gated_activation_b200 as mg
from moe_gated_activation_b200 import _capi
from moe_gated_activation_b200.workloads import WORKLOADS, bf16_bits, make_inputs, random_case
from parity import (assert_codes, assert_dscale, assert_scales_exact, bf16_u16,
                    dscale_abs_bound, u8, unblock_cols, unblock_rows)

pytestmark = pytest.mark.gpu

ACTS = {"swiglu": oracle.SWIGLU, "srelu": oracle.SRELU}


def _case(M, N, act, seed):
    return random_case(M, N, seed, width=2 * N if act == "swiglu" else N, std=2.0)


def _expect(ref, W, m_splits, cb):
    """Oracle scales in the GEMM layout."""
    ro = np.concatenate([[0], np.cumsum(m_splits)]).astype(np.int64)
    return (oracle.scales_gemm_layout(ref["row_scales"]),
            oracle.col_scales_gemm_layout(ref["col_scales"], W, ro, cb))


def _compare(got, ref, W, m_splits, cb, what):
    rs, cs = _expect(ref, W, m_splits, cb)
    assert np.array_equal(u8(got.row_scales).reshape(-1), rs), what + " row scales"
    assert np.array_equal(u8(got.col_scales).reshape(-1)[:cs.size], cs), what + " col scales"
    assert_codes(got.row_codes, ref["row_codes"], what + " row codes", exact=True)
    assert_codes(got.col_codes, ref["col_codes"], what + " col codes", exact=True)


@pytest.mark.parametrize("act", ["swiglu", "srelu"])
@pytest.mark.parametrize("M,N", [(128, 128), (256, 384), (384, 256)])
def test_dense_forward_and_backward(cuda_device, act, M, N):
    c = _case(M, N, act, seed=M + N)
    xb, s, dyb = bf16_bits(c["x"]), c["s"].numpy(), bf16_bits(c["dy"])
    x, sg, dy = c["x"].to(cuda_device), c["s"].to(cuda_device), c["dy"].to(cuda_device)
    m = np.array([M], np.int64)
    cb = np.array([0, M // 32], np.int64)
    fwd = mg.scaled_swiglu_mxfp8_fwd if act == "swiglu" else mg.scaled_srelu_mxfp8_fwd
    bwd = mg.scaled_swiglu_mxfp8_bwd if act == "swiglu" else mg.scaled_srelu_mxfp8_bwd
    got = fwd(x, sg, gemm_scales=True)
    gotb = bwd(dy, x, sg, gemm_scales=True)
    torch.cuda.synchronize()
    ref = oracle.act_fwd(xb, s, N, 3, act=ACTS[act])
    _compare(got, ref, N, m, cb, f"{act} fwd {M}x{N}")
    refb = oracle.act_bwd(dyb, xb, s, N, 3, act=ACTS[act])
    W = 2 * N if act == "swiglu" else N
    _compare(gotb.mx, refb, W, m, cb, f"{act} bwd {M}x{N}")
    assert np.array_equal(bf16_u16(gotb.dx), refb["dx"])
    assert_dscale(gotb.dscale, refb["dscale"], dscale_abs_bound(dyb, xb, s, N, act == "swiglu"),
                  "dscale")


@pytest.mark.parametrize("act", ["swiglu", "srelu"])
def test_grouped_forward_and_backward(cuda_device, act):
    N = 256
    m = np.array([256, 0, 128, 384, 0, 128], np.int64)
    M = int(m.sum())
    c = _case(M, N, act, seed=41)
    xb, s, dyb = bf16_bits(c["x"]), c["s"].numpy(), bf16_bits(c["dy"])
    x, sg, dy = c["x"].to(cuda_device), c["s"].to(cuda_device), c["dy"].to(cuda_device)
    _, ro, cb = oracle.splits_to_offsets(m, M)
    gro, gcb, _ = mg.splits_to_offsets(torch.from_numpy(m).to(cuda_device), M)
    S = int(cb[-1])
    fwd = mg.grouped_scaled_swiglu_mxfp8_fwd if act == "swiglu" else mg.grouped_scaled_srelu_mxfp8_fwd
    bwd = mg.grouped_scaled_swiglu_mxfp8_bwd if act == "swiglu" else mg.grouped_scaled_srelu_mxfp8_bwd
    got, st = fwd(x, sg, gro, gcb, col_scale_rows=S, gemm_scales=True)
    gotb, stb = bwd(dy, x, sg, gro, gcb, col_scale_rows=S, gemm_scales=True)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and int(stb.item()) == 0
    ref = oracle.grouped_act_fwd(xb, s, N, 3, ro, cb, act=ACTS[act])
    _compare(got, ref, N, m, cb, f"grouped {act} fwd")
    refb = oracle.grouped_act_bwd(dyb, xb, s, N, 3, ro, cb, act=ACTS[act])
    W = 2 * N if act == "swiglu" else N
    _compare(gotb.mx, refb, W, m, cb, f"grouped {act} bwd")
    assert np.array_equal(bf16_u16(gotb.dx), refb["dx"])


def test_single_direction_calls(cuda_device):
    M, N = 256, 256
    c = _case(M, N, "swiglu", seed=3)
    xb, s = bf16_bits(c["x"]), c["s"].numpy()
    x, sg = c["x"].to(cuda_device), c["s"].to(cuda_device)
    for rw, cw in ((True, False), (False, True)):
        got = mg.scaled_swiglu_mxfp8_fwd(x, sg, rowwise=rw, colwise=cw, gemm_scales=True)
        torch.cuda.synchronize()
        ref = oracle.act_fwd(xb, s, N, 3)
        rs, cs = _expect(ref, N, np.array([M]), np.array([0, M // 32]))
        if rw:
            assert np.array_equal(u8(got.row_scales).reshape(-1), rs)
            assert got.col_scales.numel() == 0
        else:
            assert np.array_equal(u8(got.col_scales).reshape(-1), cs)
            assert got.row_scales.numel() == 0


def test_unaligned_groups_set_status_and_write_nothing(cuda_device):
    N = 128
    m = np.array([96, 160], np.int64)      # sums to 256, but 96 % 128 != 0
    M = int(m.sum())
    c = _case(M, N, "swiglu", seed=8)
    x, sg = c["x"].to(cuda_device), c["s"].to(cuda_device)
    gro, gcb, gst = mg.splits_to_offsets(torch.from_numpy(m).to(cuda_device), M)
    W = N
    outs = {k: torch.full(shape, 0xAB, dtype=torch.uint8, device=cuda_device)
            for k, shape in (("rq", (M, W)), ("rs", (M, W // 32)), ("cq", (M, W)),
                             ("cs", (M // 32 + 2, W)))}
    mx = _capi.MxOut(outs["rq"].data_ptr(), outs["rs"].data_ptr(), outs["cq"].data_ptr(),
                     outs["cs"].data_ptr(), _capi.SCALES_GEMM)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    stream = torch.cuda.current_stream(cuda_device).cuda_stream
    _capi.call("grouped_scaled_swiglu_mxfp8_fwd", x.data_ptr(), 2 * N, sg.data_ptr(), M, N, 3, 0,
               0, gro.data_ptr(), gcb.data_ptr(), len(m), st.data_ptr(), mx, stream)
    torch.cuda.synchronize()
    assert int(gst.item()) == 0
    assert int(st.item()) == _capi.DEV_UNALIGNED_GROUPS
    for o in outs.values():
        assert bool((o == 0xAB).all())


@pytest.mark.parametrize("key", ["c3", "c5"])
def test_workload_sampled_parity(cuda_device, key):
    """The 128-aligned grouped workloads at full size: scales read back from
    the GEMM layout (by tensor reshapes) on sampled slabs against the oracle."""
    wl = WORKLOADS[key]
    inp = make_inputs(wl, device=cuda_device)
    x, s, dy = inp["x"], inp["s"], inp["dy"]
    m = inp["m_splits"].numpy()
    assert (m % 128 == 0).all() and wl.N % 128 == 0
    M, N = wl.M, wl.N
    _, ro, cb = oracle.splits_to_offsets(m, M)
    gro, gcb, _ = mg.splits_to_offsets(inp["m_splits"].to(cuda_device), M)
    S = int(cb[-1])
    f, fst = mg.grouped_scaled_swiglu_mxfp8_fwd(x, s, gro, gcb, col_scale_rows=S, gemm_scales=True)
    b, bst = mg.grouped_scaled_swiglu_mxfp8_bwd(dy, x, s, gro, gcb, col_scale_rows=S,
                                                gemm_scales=True)
    torch.cuda.synchronize()
    assert int(fst.item()) == 0 and int(bst.item()) == 0
    f_rs = unblock_rows(u8(f.row_scales).reshape(-1), M, N // 32)
    f_cs = unblock_cols(u8(f.col_scales).reshape(-1)[:M * N // 32], N, m)
    b_rs = unblock_rows(u8(b.mx.row_scales).reshape(-1), M, 2 * N // 32)
    b_cs = unblock_cols(u8(b.mx.col_scales).reshape(-1)[:M * 2 * N // 32], 2 * N, m)
    rng = np.random.default_rng(wl.seed)
    nz = [e for e in range(len(m)) if m[e] > 0]
    for e in sorted({nz[0], nz[-1], *rng.choice(nz, 2, replace=False).tolist()}):
        for k in sorted({0, int(cb[e + 1] - cb[e]) - 1}):
            r0 = int(ro[e]) + 32 * k
            rows = slice(r0, r0 + 32)
            xb = bf16_bits(x[rows])
            sv = s[rows].cpu().numpy()
            ref = oracle.act_fwd(xb, sv, N, 3)
            what = f"{key} gemm-layout fwd rows {r0}"
            assert_scales_exact(f_rs[rows], ref["row_scales"], what + " row scales")
            assert_scales_exact(f_cs[cb[e] + k:cb[e] + k + 1], ref["col_scales"], what + " col scales")
            refb = oracle.act_bwd(bf16_bits(dy[rows]), xb, sv, N, 3)
            what = f"{key} gemm-layout bwd rows {r0}"
            assert_scales_exact(b_rs[rows], refb["row_scales"], what + " row scales")
            assert_scales_exact(b_cs[cb[e] + k:cb[e] + k + 1], refb["col_scales"], what + " col scales")
            assert_codes(b.mx.col_codes[rows], refb["col_codes"], what + " col codes", exact=True)
    del f, b, inp
    torch.cuda.empty_cache()

"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Every case feeds the same seeded inputs to both sides and compares element by
element under the contract in tests/parity.py; the small cases also assert
bitwise equality of every code, scale and bf16 gradient (the sigmoid reading
makes the path exact everywhere except the order of the dscale sum).
"""
import numpy as np
import pytest
import torch

import oracle
import moe_gated_activation_b200 as mg
from moe_gated_activation_b200 import _capi
from moe_gated_activation_b200.workloads import bf16_bits, random_case
from parity import (assert_bf16_close, assert_codes, assert_dscale, assert_scales_exact,
                    bf16_u16, compare_mx, dscale_abs_bound, u8)

pytestmark = pytest.mark.gpu

ACTS = {"swiglu": oracle.SWIGLU, "srelu": oracle.SRELU}
DIRS = {"row": oracle.ROWWISE, "col": oracle.COLWISE, "both": oracle.ROWWISE | oracle.COLWISE}
# several 128-column tiles, ragged last tiles (N % 128 in {32, 64, 96}),
# partial last 32-row slabs (M % 32 != 0) and a single-block case
SHAPES = [(32, 32), (96, 224), (100, 192), (257, 320), (64, 2048)]


def _case(M, N, act, seed, std=2.0):
    width = 2 * N if act == "swiglu" else N
    c = random_case(M, N, seed, width=width, std=std)
    return c


def _fwd(act, x, s, dirs, staged=False):
    kw = dict(rowwise=bool(dirs & 1), colwise=bool(dirs & 2))
    if act == "swiglu":
        return mg.scaled_swiglu_mxfp8_fwd(x, s, staged_rounding=staged, **kw)
    return mg.scaled_srelu_mxfp8_fwd(x, s, **kw)


def _bwd(act, dy, x, s, dirs, want_dx=True, want_dscale=True):
    kw = dict(rowwise=bool(dirs & 1), colwise=bool(dirs & 2), want_dx=want_dx,
              want_dscale=want_dscale)
    if act == "swiglu":
        return mg.scaled_swiglu_mxfp8_bwd(dy, x, s, **kw)
    return mg.scaled_srelu_mxfp8_bwd(dy, x, s, **kw)


def test_sigmoid_table_matches_oracle_on_all_bf16(cuda_device):
    """Bitwise on every non-NaN bf16 input (infinities included).  For a NaN
    gate the kernels never use sigma itself: silu = g * sigma is NaN, which the
    special-value tests check."""
    got = mg.sigmoid_table(cuda_device).cpu().numpy()
    ref = oracle.sigmoid_table()
    bits = np.arange(65536, dtype=np.uint32)
    is_nan = ((bits & 0x7F80) == 0x7F80) & ((bits & 0x7F) != 0)
    same = got.view(np.uint32) == ref.view(np.uint32)
    assert same[~is_nan].all(), np.nonzero(~same & ~is_nan)[0][:10]
    assert is_nan.sum() == 254


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("dirs", list(DIRS))
@pytest.mark.parametrize("act,staged", [("swiglu", False), ("swiglu", True), ("srelu", False)])
def test_forward_parity(cuda_device, act, staged, dirs, shape):
    M, N = shape
    c = _case(M, N, act, seed=M * 7 + N)
    xb, s = bf16_bits(c["x"]), c["s"].numpy()
    ref = oracle.act_fwd(xb, s, N, DIRS[dirs], act=ACTS[act], staged=staged)
    got = _fwd(act, c["x"].to(cuda_device), c["s"].to(cuda_device), DIRS[dirs], staged)
    torch.cuda.synchronize()
    compare_mx(got, ref, f"{act} fwd {dirs} {shape}", exact=True)


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("dirs", ["none", "row", "col", "both"])
@pytest.mark.parametrize("act", ["swiglu", "srelu"])
def test_backward_parity(cuda_device, act, dirs, shape):
    M, N = shape
    d = 0 if dirs == "none" else DIRS[dirs]
    c = _case(M, N, act, seed=M * 11 + N)
    xb, s, dyb = bf16_bits(c["x"]), c["s"].numpy(), bf16_bits(c["dy"])
    ref = oracle.act_bwd(dyb, xb, s, N, d, act=ACTS[act])
    got = _bwd(act, c["dy"].to(cuda_device), c["x"].to(cuda_device), c["s"].to(cuda_device), d)
    torch.cuda.synchronize()
    what = f"{act} bwd {dirs} {shape}"
    compare_mx(got.mx, ref, what, exact=True)
    assert np.array_equal(bf16_u16(got.dx), ref["dx"]), what + " dx"
    bound = dscale_abs_bound(dyb, xb, s, N, act == "swiglu")
    assert_dscale(got.dscale, ref["dscale"], bound, what + " dscale")


@pytest.mark.parametrize("grouped", [False, True])
def test_backward_parity_many_tiles_per_warp(cuda_device, grouped):
    """The shapes above give each warp of the persistent backward one or two
    32x128 tiles; this one gives it more than four, so that the ring of each
    warp wraps several times, with ragged rows, columns and groups."""
    M, N = 16392, 1056
    c = _case(M, N, "swiglu", seed=91)
    xb, s, dyb = bf16_bits(c["x"]), c["s"].numpy(), bf16_bits(c["dy"])
    x, sg, dy = c["x"].to(cuda_device), c["s"].to(cuda_device), c["dy"].to(cuda_device)
    if grouped:
        g = np.random.default_rng(5)
        cut = np.sort(g.integers(0, M, 15))
        m = np.diff(np.concatenate([[0], cut, [M]])).astype(np.int64)
        _, ro, cb = oracle.splits_to_offsets(m, M)
        gro, gcb, _ = mg.splits_to_offsets(torch.from_numpy(m).to(cuda_device), M)
        got, st = mg.grouped_scaled_swiglu_mxfp8_bwd(dy, x, sg, gro, gcb, col_scale_rows=int(cb[-1]))
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        ref = oracle.grouped_act_bwd(dyb, xb, s, N, 3, ro, cb)
    else:
        got = _bwd("swiglu", dy, x, sg, 3)
        torch.cuda.synchronize()
        ref = oracle.act_bwd(dyb, xb, s, N, 3)
    what = f"swiglu bwd many tiles grouped={grouped}"
    compare_mx(got.mx, ref, what, exact=True)
    assert np.array_equal(bf16_u16(got.dx), ref["dx"]), what + " dx"
    assert_dscale(got.dscale, ref["dscale"], dscale_abs_bound(dyb, xb, s, N), what + " dscale")


@pytest.mark.parametrize("want_dx,want_dscale", [(False, True), (True, False), (False, False)])
def test_backward_optional_outputs(cuda_device, want_dx, want_dscale):
    M, N = 96, 224
    c = _case(M, N, "swiglu", seed=5)
    xb, s, dyb = bf16_bits(c["x"]), c["s"].numpy(), bf16_bits(c["dy"])
    ref = oracle.act_bwd(dyb, xb, s, N, 3)
    got = _bwd("swiglu", c["dy"].to(cuda_device), c["x"].to(cuda_device), c["s"].to(cuda_device),
               3, want_dx, want_dscale)
    torch.cuda.synchronize()
    compare_mx(got.mx, ref, "bwd optional", exact=True)
    assert (got.dx is None) == (not want_dx) and (got.dscale is None) == (not want_dscale)


def _special_grid(M, N, act, seed):
    """Inputs that reach every numeric regime: zeros (all-zero blocks), NaN and
    Inf (NaN / Inf blocks), tiny values (subnormal products, E4M3 underflow to
    signed zeros), huge values (fp32 overflow of u * silu), negative scales,
    E4M3-boundary magnitudes."""
    width = 2 * N if act == "swiglu" else N
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, width, generator=g) * 3
    pick = torch.rand(M, width, generator=g)
    x = torch.where(pick < 0.03, torch.zeros_like(x), x)
    x = torch.where((pick > 0.03) & (pick < 0.05), x * 1e-35, x)
    x = torch.where((pick > 0.05) & (pick < 0.06), x * 1e36, x)
    x[0, :32] = 0.0                    # an all-zero rowwise block
    x[1, 5] = float("nan")
    x[2, 7] = float("inf")
    x[3, 9] = float("-inf")
    x[4, :] = 448.0 / 2 ** 7           # exact E4M3-boundary values
    x[5, :N] = -200.0                  # sigma underflows to 0
    x[6, :N] = -95.0                   # subnormal sigma
    xb = x.to(torch.bfloat16)
    s = torch.rand(M, generator=g)
    s[7] = 0.0
    s[8] = -0.5
    s[9] = 2.0 ** -126
    s[10] = 3e38
    dy = (torch.randn(M, N, generator=g)).to(torch.bfloat16)
    dy[11, :] = 0.0
    return xb, s.float(), dy


@pytest.mark.parametrize("act", ["swiglu", "srelu"])
def test_special_values_forward_and_backward(cuda_device, act):
    M, N = 64, 128
    x, s, dy = _special_grid(M, N, act, 17)
    xb, sn, dyb = bf16_bits(x), s.numpy(), bf16_bits(dy)
    for staged in ([False, True] if act == "swiglu" else [False]):
        ref = oracle.act_fwd(xb, sn, N, 3, act=ACTS[act], staged=staged)
        got = _fwd(act, x.to(cuda_device), s.to(cuda_device), 3, staged)
        torch.cuda.synchronize()
        compare_mx(got, ref, f"{act} special fwd staged={staged}", exact=True)
    ref = oracle.act_bwd(dyb, xb, sn, N, 3, act=ACTS[act])
    got = _bwd(act, dy.to(cuda_device), x.to(cuda_device), s.to(cuda_device), 3)
    torch.cuda.synchronize()
    compare_mx(got.mx, ref, f"{act} special bwd", exact=True)
    assert_bf16_close(bf16_u16(got.dx), ref["dx"], "special dx", ulps=0)
    gd, rd = got.dscale.cpu().numpy(), ref["dscale"]
    fin = np.isfinite(rd)
    assert np.array_equal(np.isnan(gd), np.isnan(rd))
    assert np.array_equal(np.isinf(gd), np.isinf(rd))
    bound = dscale_abs_bound(dyb, xb, sn, N, act == "swiglu")
    assert_dscale(gd[fin], rd[fin], bound[fin], "special dscale")


def test_ragged_last_column_tile_sees_no_up_values(cuda_device):
    """With N % 128 != 0 the last 128-column tile of the gate reaches past
    column N-1.  Those columns must read as zero, not as the first up values:
    here row 3's up half is +Inf in its first 96 columns and its dY is
    positive, so its dscale is +Inf, which a NaN from an Inf gate times a zero
    up would turn into NaN."""
    M, N = 64, 160
    c = _case(M, N, "swiglu", seed=23)
    x, s, dy = c["x"].clone(), c["s"], c["dy"].clone()
    x[3, N:N + 96] = float("inf")
    x[3, :N] = 1.0
    dy[3] = dy[3].abs() + 0.5
    xb, sn, dyb = bf16_bits(x), s.numpy(), bf16_bits(dy)
    ref = oracle.act_bwd(dyb, xb, sn, N, 3)
    got = _bwd("swiglu", dy.to(cuda_device), x.to(cuda_device), s.to(cuda_device), 3)
    torch.cuda.synchronize()
    assert np.isposinf(ref["dscale"][3])
    compare_mx(got.mx, ref, "ragged tile bwd", exact=True)
    assert np.array_equal(bf16_u16(got.dx), ref["dx"])
    gd = got.dscale.cpu().numpy()
    assert np.isposinf(gd[3]), gd[3]
    fin = np.isfinite(ref["dscale"])
    assert_dscale(gd[fin], ref["dscale"][fin], dscale_abs_bound(dyb, xb, sn, N)[fin], "ragged dscale")
    reff = oracle.act_fwd(xb, sn, N, 3)
    gotf = _fwd("swiglu", x.to(cuda_device), s.to(cuda_device), 3)
    torch.cuda.synchronize()
    compare_mx(gotf, reff, "ragged tile fwd", exact=True)


def test_strided_input_is_read_in_place_and_inputs_are_not_mutated(cuda_device):
    M, N, ld = 96, 160, 2 * 160 + 64
    c = _case(M, N, "swiglu", seed=9)
    big = torch.randn(M, ld).to(torch.bfloat16)
    big[:, :2 * N] = c["x"]
    xg = big.to(cuda_device)
    view = xg[:, :2 * N]
    assert view.stride(0) == ld
    before = xg.clone()
    sg, dyg = c["s"].to(cuda_device), c["dy"].to(cuda_device)
    s_before, dy_before = sg.clone(), dyg.clone()
    got = mg.scaled_swiglu_mxfp8_fwd(view, sg)
    gb = mg.scaled_swiglu_mxfp8_bwd(dyg, view, sg)
    torch.cuda.synchronize()
    ref = oracle.act_fwd(bf16_bits(c["x"]), c["s"].numpy(), N, 3)
    compare_mx(got, ref, "strided fwd", exact=True)
    refb = oracle.act_bwd(bf16_bits(c["dy"]), bf16_bits(c["x"]), c["s"].numpy(), N, 3)
    compare_mx(gb.mx, refb, "strided bwd", exact=True)
    assert torch.equal(xg.view(torch.int16), before.view(torch.int16))
    assert torch.equal(sg, s_before) and torch.equal(dyg.view(torch.int16), dy_before.view(torch.int16))


def test_outputs_stay_inside_their_buffers(cuda_device):
    """Guard bands: every output is placed inside a larger canary-filled buffer;
    the bytes around it must be unchanged."""
    M, N = 100, 224
    c = _case(M, N, "swiglu", seed=21)
    x, s, dy = c["x"].to(cuda_device), c["s"].to(cuda_device), c["dy"].to(cuda_device)
    pad = 256

    def guarded(nbytes):
        buf = torch.full((nbytes + 2 * pad,), 0xA5, dtype=torch.uint8, device=cuda_device)
        return buf, buf.data_ptr() + pad

    W = 2 * N
    sizes = dict(rq=M * W, rs=M * W // 32, cq=M * W, cs=((M + 31) // 32) * W)
    bufs = {k: guarded(v) for k, v in sizes.items()}
    dxb = guarded(M * W * 2)
    dsb = guarded(M * 4)
    ws = torch.zeros(mg.bwd_workspace_bytes(M, N), dtype=torch.uint8, device=cuda_device)
    mx = _capi.MxOut(bufs["rq"][1], bufs["rs"][1], bufs["cq"][1], bufs["cs"][1])
    stream = torch.cuda.current_stream(cuda_device).cuda_stream
    _capi.call("scaled_swiglu_mxfp8_bwd", dy.data_ptr(), N, x.data_ptr(), 2 * N, s.data_ptr(),
               M, N, 3, 0, dxb[1], dsb[1], mx, ws.data_ptr(), ws.numel(), stream)
    torch.cuda.synchronize()
    for name, (buf, _), n in [(k, bufs[k], sizes[k]) for k in sizes] + \
            [("dx", dxb, M * W * 2), ("dscale", dsb, M * 4)]:
        h = buf.cpu().numpy()
        assert (h[:pad] == 0xA5).all() and (h[pad + n:] == 0xA5).all(), name
    ref = oracle.act_bwd(bf16_bits(c["dy"]), bf16_bits(c["x"]), c["s"].numpy(), N, 3)
    got_rq = bufs["rq"][0][pad:pad + sizes["rq"]].cpu().numpy().reshape(M, W)
    assert np.array_equal(got_rq, ref["row_codes"])
    # the same workspace serves the next call (its counters are back at zero)
    dsb2 = guarded(M * 4)
    _capi.call("scaled_swiglu_mxfp8_bwd", dy.data_ptr(), N, x.data_ptr(), 2 * N, s.data_ptr(),
               M, N, 0, 0, None, dsb2[1], _capi.MxOut(None, None, None, None), ws.data_ptr(),
               ws.numel(), stream)
    torch.cuda.synchronize()
    a = dsb[0][pad:pad + 4 * M].cpu()
    b = dsb2[0][pad:pad + 4 * M].cpu()
    assert torch.equal(a, b)


def test_dscale_is_deterministic(cuda_device):
    M, N = 256, 1024
    c = _case(M, N, "swiglu", seed=33)
    x, s, dy = c["x"].to(cuda_device), c["s"].to(cuda_device), c["dy"].to(cuda_device)
    a = mg.scaled_swiglu_mxfp8_bwd(dy, x, s).dscale.clone()
    b = mg.scaled_swiglu_mxfp8_bwd(dy, x, s).dscale.clone()
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))


def test_cross_mode_consistency_on_gpu(cuda_device):
    M, N = 128, 512
    c = _case(M, N, "swiglu", seed=41)
    x, s = c["x"].to(cuda_device), c["s"].to(cuda_device)
    both = mg.scaled_swiglu_mxfp8_fwd(x, s)
    row = mg.scaled_swiglu_mxfp8_fwd(x, s, colwise=False)
    col = mg.scaled_swiglu_mxfp8_fwd(x, s, rowwise=False)
    assert torch.equal(u8t(both.row_codes), u8t(row.row_codes))
    assert torch.equal(both.row_scales, row.row_scales)
    assert torch.equal(u8t(both.col_codes), u8t(col.col_codes))
    assert torch.equal(both.col_scales, col.col_scales)
    assert row.col_codes.numel() == 0 and col.row_scales.numel() == 0


def u8t(t):
    return t.view(torch.uint8)


# ------------------------------------------------------------------ grouped
SPLITS = {
    "aligned_with_empties": [64, 0, 96, 32, 0, 64, 0],
    "uniform": [32] * 8,
    "ragged": [5, 40, 0, 33, 1, 49, 0, 17],
    "single": [160],
}


@pytest.mark.parametrize("name", list(SPLITS))
def test_splits_to_offsets_parity(cuda_device, name):
    m = np.array(SPLITS[name], np.int64)
    M = int(m.sum())
    st, ro, cb = oracle.splits_to_offsets(m, M)
    gro, gcb, gst = mg.splits_to_offsets(torch.from_numpy(m).to(cuda_device), M)
    torch.cuda.synchronize()
    assert int(gst.item()) == st == 0
    assert np.array_equal(gro.cpu().numpy(), ro) and np.array_equal(gcb.cpu().numpy(), cb)


@pytest.mark.parametrize("splits,M,status", [([4, -1, 5], 8, 1), ([4, 5], 8, 2), ([4, 3], 8, 2),
                                             ([], 0, 0), ([2 ** 40, 2 ** 40], 8, 2)])
def test_splits_to_offsets_status(cuda_device, splits, M, status):
    m = np.array(splits, np.int64)
    assert oracle.splits_to_offsets(m, M)[0] == status
    _, _, gst = mg.splits_to_offsets(torch.from_numpy(m).to(cuda_device), M)
    assert int(gst.item()) == status


def test_failed_splits_leave_no_usable_offsets(cuda_device):
    """Offsets buffers reused across calls: after a valid splits_to_offsets and
    a grouped forward, bad splits (negative, or not summing to M) into the same
    buffers must make the next grouped forward report bad offsets and write
    nothing, not run on the earlier call's offsets."""
    N, m = 64, np.array([32, 64, 0, 32], np.int64)
    M = int(m.sum())
    c = _case(M, N, "swiglu", seed=31)
    x, s = c["x"].to(cuda_device), c["s"].to(cuda_device)
    md = torch.from_numpy(m).to(cuda_device)
    ro = torch.empty(len(m) + 1, dtype=torch.int64, device=cuda_device)
    cb = torch.empty_like(ro)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    lib = _capi.lib()
    stream = torch.cuda.current_stream(cuda_device).cuda_stream
    _capi.call("splits_to_offsets", md.data_ptr(), len(m), M, ro.data_ptr(), cb.data_ptr(),
               st.data_ptr(), stream)
    good, gst = mg.grouped_scaled_swiglu_mxfp8_fwd(x, s, ro, cb, col_scale_rows=M // 32)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and int(gst.item()) == 0
    for bad, code in (([32, -32, 64, 32], 1), ([32, 64, 0, 0], 2)):
        mb = torch.tensor(bad, dtype=torch.int64, device=cuda_device)
        _capi.call("splits_to_offsets", mb.data_ptr(), len(bad), M, ro.data_ptr(),
                   cb.data_ptr(), st.data_ptr(), stream)
        torch.cuda.synchronize()
        assert int(st.item()) == code
        outs = {k: torch.full_like(getattr(good, k).view(torch.uint8), 0xAB)
                for k in ("row_codes", "row_scales", "col_codes", "col_scales")}
        mx = _capi.MxOut(*(outs[k].data_ptr() for k in ("row_codes", "row_scales", "col_codes",
                                                          "col_scales")))
        st2 = torch.zeros(1, dtype=torch.int32, device=cuda_device)
        _capi.call("grouped_scaled_swiglu_mxfp8_fwd", x.data_ptr(), 2 * N, s.data_ptr(), M, N, 3,
                   0, 0, ro.data_ptr(), cb.data_ptr(), len(m), st2.data_ptr(), mx, stream)
        torch.cuda.synchronize()
        assert int(st2.item()) == _capi.DEV_BAD_OFFSETS
        for o in outs.values():
            assert bool((o == 0xAB).all())


def test_splits_to_offsets_many_groups(cuda_device):
    g = np.random.default_rng(3)
    m = (g.integers(0, 5, 2040) * 32 + g.integers(0, 3, 2040)).astype(np.int64)
    M = int(m.sum())
    st, ro, cb = oracle.splits_to_offsets(m, M)
    gro, gcb, gst = mg.splits_to_offsets(torch.from_numpy(m).to(cuda_device), M)
    assert int(gst.item()) == 0
    assert np.array_equal(gro.cpu().numpy(), ro) and np.array_equal(gcb.cpu().numpy(), cb)


@pytest.mark.parametrize("name", list(SPLITS))
@pytest.mark.parametrize("act", ["swiglu", "srelu"])
def test_grouped_forward_backward_parity(cuda_device, act, name):
    N = 96
    m = np.array(SPLITS[name], np.int64)
    M = int(m.sum())
    c = _case(M, N, act, seed=len(name) + N)
    xb, s, dyb = bf16_bits(c["x"]), c["s"].numpy(), bf16_bits(c["dy"])
    _, ro, cb = oracle.splits_to_offsets(m, M)
    gro, gcb, _ = mg.splits_to_offsets(torch.from_numpy(m).to(cuda_device), M)
    x, sg, dy = c["x"].to(cuda_device), c["s"].to(cuda_device), c["dy"].to(cuda_device)
    S = int(cb[-1])
    fwd = mg.grouped_scaled_swiglu_mxfp8_fwd if act == "swiglu" else mg.grouped_scaled_srelu_mxfp8_fwd
    bwd = mg.grouped_scaled_swiglu_mxfp8_bwd if act == "swiglu" else mg.grouped_scaled_srelu_mxfp8_bwd
    got, st = fwd(x, sg, gro, gcb, col_scale_rows=S)
    gotb, stb = bwd(dy, x, sg, gro, gcb, col_scale_rows=S)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and int(stb.item()) == 0
    ref = oracle.grouped_act_fwd(xb, s, N, 3, ro, cb, act=ACTS[act])
    compare_mx(got, ref, f"grouped {act} fwd {name}", exact=True)
    refb = oracle.grouped_act_bwd(dyb, xb, s, N, 3, ro, cb, act=ACTS[act])
    compare_mx(gotb.mx, refb, f"grouped {act} bwd {name}", exact=True)
    assert np.array_equal(bf16_u16(gotb.dx), refb["dx"])
    assert_dscale(gotb.dscale, refb["dscale"], dscale_abs_bound(dyb, xb, s, N, act == "swiglu"),
                  "grouped dscale")


@pytest.mark.parametrize("act", ["swiglu", "srelu"])
def test_grouped_parity_at_the_group_limit(cuda_device, act):
    """MOEACT_MAX_GROUPS groups (the most offsets the kernels stage in shared
    memory: in the sigmoid table's gap for SwiGLU, after the rings for SReLU),
    ragged sizes 0..40 with many empty groups."""
    N = 64
    g = np.random.default_rng(17)
    m = g.integers(0, 41, _capi.MAX_GROUPS).astype(np.int64)
    m[g.random(_capi.MAX_GROUPS) < 0.3] = 0
    M = int(m.sum())
    c = _case(M, N, act, seed=19)
    xb, s, dyb = bf16_bits(c["x"]), c["s"].numpy(), bf16_bits(c["dy"])
    _, ro, cb = oracle.splits_to_offsets(m, M)
    gro, gcb, gst = mg.splits_to_offsets(torch.from_numpy(m).to(cuda_device), M)
    x, sg, dy = c["x"].to(cuda_device), c["s"].to(cuda_device), c["dy"].to(cuda_device)
    S = int(cb[-1])
    fwd = mg.grouped_scaled_swiglu_mxfp8_fwd if act == "swiglu" else mg.grouped_scaled_srelu_mxfp8_fwd
    bwd = mg.grouped_scaled_swiglu_mxfp8_bwd if act == "swiglu" else mg.grouped_scaled_srelu_mxfp8_bwd
    got, st = fwd(x, sg, gro, gcb, col_scale_rows=S)
    gotb, stb = bwd(dy, x, sg, gro, gcb, col_scale_rows=S)
    torch.cuda.synchronize()
    assert int(gst.item()) == 0 and int(st.item()) == 0 and int(stb.item()) == 0
    ref = oracle.grouped_act_fwd(xb, s, N, 3, ro, cb, act=ACTS[act])
    compare_mx(got, ref, f"{act} fwd at {_capi.MAX_GROUPS} groups", exact=True)
    refb = oracle.grouped_act_bwd(dyb, xb, s, N, 3, ro, cb, act=ACTS[act])
    compare_mx(gotb.mx, refb, f"{act} bwd at {_capi.MAX_GROUPS} groups", exact=True)
    assert np.array_equal(bf16_u16(gotb.dx), refb["dx"])
    assert_dscale(gotb.dscale, refb["dscale"], dscale_abs_bound(dyb, xb, s, N, act == "swiglu"),
                  "dscale at the group limit")


def test_grouped_equals_dense_for_aligned_splits(cuda_device):
    N = 128
    m = np.array([96, 0, 32, 128, 0, 64], np.int64)
    M = int(m.sum())
    c = _case(M, N, "swiglu", seed=77)
    x, s = c["x"].to(cuda_device), c["s"].to(cuda_device)
    gro, gcb, _ = mg.splits_to_offsets(torch.from_numpy(m).to(cuda_device), M)
    g, _ = mg.grouped_scaled_swiglu_mxfp8_fwd(x, s, gro, gcb, col_scale_rows=M // 32)
    d = mg.scaled_swiglu_mxfp8_fwd(x, s)
    for a, b in zip(g, d):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))


@pytest.mark.parametrize("corrupt", ["row_last", "row_decreasing", "colblk"])
def test_grouped_bad_offsets_set_status_and_write_nothing(cuda_device, corrupt):
    N = 64
    m = np.array([32, 64, 32], np.int64)
    M = int(m.sum())
    c = _case(M, N, "swiglu", seed=1)
    x, s = c["x"].to(cuda_device), c["s"].to(cuda_device)
    gro, gcb, _ = mg.splits_to_offsets(torch.from_numpy(m).to(cuda_device), M)
    if corrupt == "row_last":
        gro[-1] = M - 1
    elif corrupt == "row_decreasing":
        gro[1] = 100
    else:
        gcb[2] = 7
    got, st = mg.grouped_scaled_swiglu_mxfp8_fwd(x, s, gro, gcb)
    torch.cuda.synchronize()
    assert int(st.item()) == _capi.DEV_BAD_OFFSETS
    # outputs were allocated uninitialised: compare against a second call on
    # pre-filled buffers through the C ABI to check nothing is written
    rq = torch.full((M, N), 0x5A, dtype=torch.uint8, device=cuda_device)
    rs = torch.full((M, N // 32), 0x5A, dtype=torch.uint8, device=cuda_device)
    stt = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    _capi.call("grouped_scaled_swiglu_mxfp8_fwd", x.data_ptr(), 2 * N, s.data_ptr(), M, N, 1, 0,
               0, gro.data_ptr(), gcb.data_ptr(), 3, stt.data_ptr(),
               _capi.MxOut(rq.data_ptr(), rs.data_ptr(), None, None),
               torch.cuda.current_stream(cuda_device).cuda_stream)
    torch.cuda.synchronize()
    assert int(stt.item()) == _capi.DEV_BAD_OFFSETS
    assert bool((rq == 0x5A).all()) and bool((rs == 0x5A).all())


def test_empty_inputs_through_the_python_api(cuda_device):
    """M = 0 through the tensor API (empty tensors may have null data
    pointers): empty outputs, no error, and a grouped call's status word 0."""
    N = 128
    x = torch.empty(0, 2 * N, dtype=torch.bfloat16, device=cuda_device)
    s = torch.empty(0, dtype=torch.float32, device=cuda_device)
    dy = torch.empty(0, N, dtype=torch.bfloat16, device=cuda_device)
    f = mg.scaled_swiglu_mxfp8_fwd(x, s)
    b = mg.scaled_swiglu_mxfp8_bwd(dy, x, s)
    m = torch.zeros(3, dtype=torch.int64, device=cuda_device)
    ro, cb, st = mg.splits_to_offsets(m, 0)
    gf, gst = mg.grouped_scaled_swiglu_mxfp8_fwd(x, s, ro, cb, glu_interleave=32)
    gb, gbst = mg.grouped_scaled_swiglu_mxfp8_bwd(dy, x, s, ro, cb)
    torch.cuda.synchronize()
    assert f.row_codes.shape == (0, N) and f.col_scales.shape[0] == 0
    assert b.dx.shape == (0, 2 * N) and b.dscale.shape == (0,)
    assert int(st.item()) == 0 and int(gst.item()) == 0 and int(gbst.item()) == 0
    assert gf.row_codes.numel() == 0 and gb.mx.row_codes.numel() == 0

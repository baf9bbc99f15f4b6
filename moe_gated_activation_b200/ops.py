"""PyTorch-facing calls of the fused scaled gated activation + MXFP8 path.

These functions only allocate outputs with torch, check dtypes/strides and pass
pointers and the current CUDA stream to libmoeact (include/moeact.h); every
step of the computation runs in the library's sm_100a kernels.

Every fused call takes ``out=``: caller-owned buffers (an ``MXFP8`` for the
forward, a ``Backward`` for the backward) that the kernels write in place,
for CUDA-graph replay without pointer changes.

Return convention (pytorch/ao PR #4743, section "API"): an ``MXFP8`` tuple
(row_codes, col_codes, row_scales, col_scales); a disabled direction comes back
zero-sized.  Codes are ``torch.float8_e4m3fn`` [M, W] (same row-major layout
for both directions), scales ``torch.uint8`` E8M0 bytes, row scales [M, W/32],
col scales [S, W].
"""
from __future__ import annotations

import ctypes
import threading
from typing import NamedTuple, Optional

import torch

from . import _capi

ROWWISE = _capi.ROWWISE
COLWISE = _capi.COLWISE


class MXFP8(NamedTuple):
    row_codes: torch.Tensor
    col_codes: torch.Tensor
    row_scales: torch.Tensor
    col_scales: torch.Tensor


class Backward(NamedTuple):
    mx: MXFP8                     # MXFP8 of dX ("grouped_dy")
    dx: Optional[torch.Tensor]    # bf16 [M, W] ("dense_dy")
    dscale: Optional[torch.Tensor]  # fp32 [M] ("grad_scales")


def _dirs(rowwise, colwise):
    return (ROWWISE if rowwise else 0) | (COLWISE if colwise else 0)


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _check_rows(t, name, dtype, width):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be 2-D with unit column stride")
    if t.shape[1] < width:
        raise ValueError(f"{name} has {t.shape[1]} columns, {width} needed")


def _check_s(s, M, device):
    if s.dtype != torch.float32 or not s.is_cuda or s.dim() != 1 or s.shape[0] != M:
        raise ValueError(f"s must be a CUDA float32 vector of length {M}")
    if s.stride(0) != 1:
        raise ValueError("s must be contiguous")


def _alloc_mx(M, W, dirs, device, col_rows):
    e = torch.empty(0, dtype=torch.uint8, device=device)
    rq = torch.empty((M, W), dtype=torch.uint8, device=device) if dirs & ROWWISE else e
    rs = torch.empty((M, W // 32), dtype=torch.uint8, device=device) if dirs & ROWWISE else e
    cq = torch.empty((M, W), dtype=torch.uint8, device=device) if dirs & COLWISE else e
    cs = torch.empty((col_rows, W), dtype=torch.uint8, device=device) if dirs & COLWISE else e
    return rq, rs, cq, cs


def _take_mx(out, M, W, dirs, device, col_rows):
    """Caller-owned MXFP8 buffers (`out=`): the requested directions' tensors,
    contiguous on `device`, codes uint8 or float8_e4m3fn [M, W], row scales
    uint8 [M, W/32], col scales uint8 [>= col_rows, W].  The library writes
    into them in place, so a captured CUDA graph can replay into the same
    buffers (TE PR #3238: an output= argument for graph-replayed quantization)."""
    e = torch.empty(0, dtype=torch.uint8, device=device)

    def take(t, name, shape, min_rows=False):
        if t is None:
            raise ValueError(f"out.{name} is required for the requested direction")
        if t.device != device or not t.is_contiguous():
            raise ValueError(f"out.{name} must be contiguous on {device}")
        if t.dtype == torch.float8_e4m3fn:
            t = t.view(torch.uint8)
        if t.dtype != torch.uint8:
            raise TypeError(f"out.{name} must be uint8 (or float8_e4m3fn codes)")
        ok = (t.dim() == 2 and t.shape[1] == shape[1] and t.shape[0] >= shape[0]) if min_rows \
            else tuple(t.shape) == tuple(shape)
        if not ok:
            raise ValueError(f"out.{name} has shape {tuple(t.shape)}, {tuple(shape)} needed")
        return t

    rq = take(out.row_codes, "row_codes", (M, W)) if dirs & ROWWISE else e
    rs = take(out.row_scales, "row_scales", (M, W // 32)) if dirs & ROWWISE else e
    cq = take(out.col_codes, "col_codes", (M, W)) if dirs & COLWISE else e
    cs = take(out.col_scales, "col_scales", (col_rows, W), min_rows=True) if dirs & COLWISE else e
    return rq, rs, cq, cs


def _mx_struct(rq, rs, cq, cs, dirs, gemm_scales=False, noop_flag=None):
    if dirs & ROWWISE:
        r = (rq.data_ptr(), rs.data_ptr())
    else:
        r = (None, None)
    if dirs & COLWISE:
        c = (cq.data_ptr(), cs.data_ptr())
    else:
        c = (None, None)
    layout = _capi.SCALES_GEMM if gemm_scales else _capi.SCALES_ROWMAJOR
    if noop_flag is not None and (noop_flag.dtype != torch.int32 or not noop_flag.is_cuda):
        raise ValueError("noop_flag must be an int32 CUDA tensor")
    return _capi.MxOut(r[0], r[1], c[0], c[1], layout,
                       noop_flag.data_ptr() if noop_flag is not None else None)


def _mx_result(rq, rs, cq, cs, col_rows_view=None):
    if col_rows_view is not None and cs.numel():
        cs = cs[:col_rows_view]
    return MXFP8(rq.view(torch.float8_e4m3fn), cq.view(torch.float8_e4m3fn), rs, cs)


def _ilv(glu_interleave, gated):
    """The glu_interleave argument: 0 for [gate | up] halves, else the block
    size G of interleaved gate / up columns (gated activations only)."""
    g = 0 if glu_interleave is None else int(glu_interleave)
    if g and not gated:
        raise ValueError("glu_interleave applies to gated activations only")
    return g


# ------------------------------------------------------------------ offsets
def splits_to_offsets(m_splits: torch.Tensor, total_rows: int):
    """(row_offs, colblk_offs, status) int64/int64/int32 device tensors for the
    per-expert row counts `m_splits` (int64, on the device)."""
    if m_splits.dtype != torch.int64 or not m_splits.is_cuda or m_splits.dim() != 1:
        raise ValueError("m_splits must be a 1-D int64 CUDA tensor")
    m_splits = m_splits.contiguous()
    dev = m_splits.device
    E = m_splits.shape[0]
    ro = torch.empty(E + 1, dtype=torch.int64, device=dev)
    cb = torch.empty(E + 1, dtype=torch.int64, device=dev)
    st = torch.empty(1, dtype=torch.int32, device=dev)
    _capi.call("splits_to_offsets", _ptr(m_splits), E, int(total_rows), _ptr(ro), _ptr(cb),
               _ptr(st), _stream(dev))
    return ro, cb, st


# ------------------------------------------------------------------ forward
def _fwd(act, x, s, N, rowwise, colwise, staged, grouped=None, gemm_scales=False, clamp=None,
         noop_flag=None, glu_interleave=0, out=None):
    swiglu = act != "srelu"        # gated: x = [gate | up]
    if N is None:
        N = x.shape[1] // 2 if swiglu else x.shape[1]
    _check_rows(x, "x", torch.bfloat16, 2 * N if swiglu else N)
    M = x.shape[0]
    _check_s(s, M, x.device)
    dirs = _dirs(rowwise, colwise)
    if grouped is None:
        col_rows, view = (M + 31) // 32, None
    else:
        ro, cb, E, st, view = grouped
        col_rows = (M + 31) // 32 + E
    if out is None:
        rq, rs, cq, cs = _alloc_mx(M, N, dirs, x.device, col_rows)
    else:
        rq, rs, cq, cs = _take_mx(out, M, N, dirs, x.device, col_rows)
    mx = _mx_struct(rq, rs, cq, cs, dirs, gemm_scales, noop_flag)
    stream = _stream(x.device)
    ldx = x.stride(0) if M > 1 else max(x.stride(0), x.shape[1])
    ilv = _ilv(glu_interleave, swiglu)
    if M == 0:
        # nothing to compute (the library launches nothing either); empty
        # tensors may have null data pointers, which the C ABI rejects
        if dirs == 0:
            raise ValueError("at least one of rowwise / colwise is required")
        if grouped is not None:
            st.zero_()
        return _mx_result(rq, rs, cq, cs, view)
    if act == "clamped":
        alpha, limit = clamp
        if grouped is None:
            _capi.call("scaled_clamped_swiglu_mxfp8_fwd", _ptr(x), ldx, _ptr(s), M, N, dirs,
                       alpha, limit, ilv, mx, stream)
        else:
            _capi.call("grouped_scaled_clamped_swiglu_mxfp8_fwd", _ptr(x), ldx, _ptr(s), M, N,
                       dirs, alpha, limit, ilv, _ptr(ro), _ptr(cb), E, _ptr(st), mx, stream)
    elif grouped is None:
        if swiglu:
            _capi.call("scaled_swiglu_mxfp8_fwd", _ptr(x), ldx, _ptr(s), M, N, dirs, int(staged),
                       ilv, mx, stream)
        else:
            _capi.call("scaled_srelu_mxfp8_fwd", _ptr(x), ldx, _ptr(s), M, N, dirs, mx, stream)
    else:
        if swiglu:
            _capi.call("grouped_scaled_swiglu_mxfp8_fwd", _ptr(x), ldx, _ptr(s), M, N, dirs,
                       int(staged), ilv, _ptr(ro), _ptr(cb), E, _ptr(st), mx, stream)
        else:
            _capi.call("grouped_scaled_srelu_mxfp8_fwd", _ptr(x), ldx, _ptr(s), M, N, dirs,
                       _ptr(ro), _ptr(cb), E, _ptr(st), mx, stream)
    return _mx_result(rq, rs, cq, cs, view)


def scaled_swiglu_mxfp8_fwd(x, s, *, rowwise=True, colwise=True, staged_rounding=False, N=None,
                            gemm_scales=False, noop_flag=None, glu_interleave=None, out=None):
    """MXFP8 of SwiGLU(x) * s; x bf16 [M, >=2N] packs [gate | up].
    gemm_scales: scales in the GEMM-ready tiled layout (moeact.h,
    MOEACT_SCALES_GEMM; M and N multiples of 128).
    glu_interleave: G > 0 reads x as G gate columns, then their G up
    columns, repeated (G = 32, 64 or a multiple of 128 dividing N); the
    backward writes dx and its MXFP8 in the same column order."""
    return _fwd("swiglu", x, s, N, rowwise, colwise, staged_rounding, gemm_scales=gemm_scales,
                noop_flag=noop_flag, out=out, glu_interleave=glu_interleave)


def scaled_srelu_mxfp8_fwd(x, s, *, rowwise=True, colwise=True, N=None, gemm_scales=False,
                           noop_flag=None, out=None):
    """MXFP8 of relu(x)^2 * s; x bf16 [M, >=N]."""
    return _fwd("srelu", x, s, N, rowwise, colwise, False, gemm_scales=gemm_scales,
                noop_flag=noop_flag, out=out)


def _grouped_args(row_offs, colblk_offs, status, col_scale_rows, device):
    E = row_offs.shape[0] - 1
    if status is None:
        status = torch.empty(1, dtype=torch.int32, device=device)
    return (row_offs, colblk_offs, E, status, col_scale_rows), status


def grouped_scaled_swiglu_mxfp8_fwd(x, s, row_offs, colblk_offs, *, rowwise=True, colwise=True,
                                    staged_rounding=False, status=None, col_scale_rows=None,
                                    N=None, gemm_scales=False, noop_flag=None,
                                    glu_interleave=None, out=None):
    """Grouped forward: experts own the rows given by `row_offs` (from
    splits_to_offsets).  Returns (MXFP8, status).  Col scales hold
    ceil(M/32) + E rows unless `col_scale_rows` (sum of ceil(m_e/32), known on
    the host) is given."""
    g, status = _grouped_args(row_offs, colblk_offs, status, col_scale_rows, x.device)
    return _fwd("swiglu", x, s, N, rowwise, colwise, staged_rounding, g,
                gemm_scales=gemm_scales, noop_flag=noop_flag, out=out,
                glu_interleave=glu_interleave), status


def grouped_scaled_srelu_mxfp8_fwd(x, s, row_offs, colblk_offs, *, rowwise=True, colwise=True,
                                   status=None, col_scale_rows=None, N=None, gemm_scales=False,
                                   noop_flag=None, out=None):
    g, status = _grouped_args(row_offs, colblk_offs, status, col_scale_rows, x.device)
    return _fwd("srelu", x, s, N, rowwise, colwise, False, g, gemm_scales=gemm_scales,
                noop_flag=noop_flag, out=out), status


# ------------------------------------------------------------------ backward
_ws_lock = threading.Lock()
_ws_cache = {}


def bwd_workspace_bytes(M, N, num_groups=1):
    return int(_capi.lib().scaled_act_mxfp8_bwd_workspace_size(M, N, num_groups))


def _workspace(device, nbytes):
    """A workspace per (device, stream), reused across calls (the kernels need
    no initial content in it)."""
    key = (device.index, torch.cuda.current_stream(device).cuda_stream)
    with _ws_lock:
        ws = _ws_cache.get(key)
        if ws is None or ws.numel() < nbytes:
            ws = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)
            _ws_cache[key] = ws
    return ws


def _bwd(act, dy, x, s, N, rowwise, colwise, want_dx, want_dscale, workspace, grouped=None,
         gemm_scales=False, clamp=None, noop_flag=None, glu_interleave=0, out=None):
    swiglu = act != "srelu"        # gated: x = [gate | up], W = 2N
    if N is None:
        N = dy.shape[1]
    _check_rows(x, "x", torch.bfloat16, 2 * N if swiglu else N)
    _check_rows(dy, "dy", torch.bfloat16, N)
    M = x.shape[0]
    if dy.shape[0] != M:
        raise ValueError("dy and x must have the same number of rows")
    _check_s(s, M, x.device)
    dirs = _dirs(rowwise, colwise)
    W = 2 * N if swiglu else N
    dev = x.device
    if grouped is None:
        E, col_rows, view = 1, (M + 31) // 32, None
    else:
        ro, cb, E, st, view = grouped
        col_rows = (M + 31) // 32 + E
    if out is None:
        rq, rs, cq, cs = _alloc_mx(M, W, dirs, dev, col_rows)
        dx = torch.empty((M, W), dtype=torch.bfloat16, device=dev) if want_dx else None
        dscale = torch.empty(M, dtype=torch.float32, device=dev) if want_dscale else None
    else:
        # caller-owned buffers: dx / dscale are computed when given
        rq, rs, cq, cs = _take_mx(out.mx, M, W, dirs, dev, col_rows)
        dx, dscale = out.dx, out.dscale
        if dx is not None and (dx.dtype != torch.bfloat16 or tuple(dx.shape) != (M, W)
                               or not dx.is_contiguous() or dx.device != dev):
            raise ValueError(f"out.dx must be a contiguous bf16 [{M}, {W}] tensor on {dev}")
        if dscale is not None and (dscale.dtype != torch.float32 or tuple(dscale.shape) != (M,)
                                   or not dscale.is_contiguous() or dscale.device != dev):
            raise ValueError(f"out.dscale must be a contiguous fp32 [{M}] tensor on {dev}")
        want_dx, want_dscale = dx is not None, dscale is not None
    mx = _mx_struct(rq, rs, cq, cs, dirs, gemm_scales, noop_flag)
    nbytes = bwd_workspace_bytes(M, N, E)
    ws = None
    if want_dscale:
        ws = workspace if workspace is not None else _workspace(dev, nbytes)
    stream = _stream(dev)
    ldx = x.stride(0) if M > 1 else max(x.stride(0), x.shape[1])
    lddy = dy.stride(0) if M > 1 else max(dy.stride(0), dy.shape[1])
    if M == 0:
        _ilv(glu_interleave, swiglu)
        if dirs == 0 and not want_dx and not want_dscale:
            raise ValueError("nothing requested: no direction, dx or dscale")
        if grouped is not None:
            st.zero_()
        return Backward(_mx_result(rq, rs, cq, cs, view), dx, dscale)
    common = (_ptr(dy), lddy, _ptr(x), ldx, _ptr(s), M, N, dirs)
    tail = (mx, _ptr(ws), ws.numel() if ws is not None else 0, stream)
    if swiglu:
        clamp_args = tuple(clamp) if act == "clamped" else ()
        common = common + clamp_args + (_ilv(glu_interleave, True),)
    if act == "clamped":
        if grouped is None:
            _capi.call("scaled_clamped_swiglu_mxfp8_bwd", *common, _ptr(dx), _ptr(dscale), *tail)
        else:
            _capi.call("grouped_scaled_clamped_swiglu_mxfp8_bwd", *common, _ptr(ro), _ptr(cb), E,
                       _ptr(st), _ptr(dx), _ptr(dscale), *tail)
    elif grouped is None:
        name = "scaled_swiglu_mxfp8_bwd" if swiglu else "scaled_srelu_mxfp8_bwd"
        _capi.call(name, *common, _ptr(dx), _ptr(dscale), *tail)
    else:
        name = "grouped_scaled_swiglu_mxfp8_bwd" if swiglu else "grouped_scaled_srelu_mxfp8_bwd"
        _capi.call(name, *common, _ptr(ro), _ptr(cb), E, _ptr(st), _ptr(dx), _ptr(dscale), *tail)
    return Backward(_mx_result(rq, rs, cq, cs, view), dx, dscale)


def scaled_swiglu_mxfp8_bwd(dy, x, s, *, rowwise=True, colwise=True, want_dx=True,
                            want_dscale=True, workspace=None, N=None, gemm_scales=False,
                            noop_flag=None, glu_interleave=None, out=None):
    """Backward of the scaled SwiGLU: MXFP8 of [dgate | dup], bf16 dx, fp32 dscale."""
    return _bwd("swiglu", dy, x, s, N, rowwise, colwise, want_dx, want_dscale, workspace,
                gemm_scales=gemm_scales, noop_flag=noop_flag, out=out,
                glu_interleave=glu_interleave)


def scaled_srelu_mxfp8_bwd(dy, x, s, *, rowwise=True, colwise=True, want_dx=True,
                           want_dscale=True, workspace=None, N=None, gemm_scales=False,
                           noop_flag=None, out=None):
    return _bwd("srelu", dy, x, s, N, rowwise, colwise, want_dx, want_dscale, workspace,
                gemm_scales=gemm_scales, noop_flag=noop_flag, out=out)


def grouped_scaled_swiglu_mxfp8_bwd(dy, x, s, row_offs, colblk_offs, *, rowwise=True,
                                    colwise=True, want_dx=True, want_dscale=True,
                                    workspace=None, status=None, col_scale_rows=None, N=None,
                                    gemm_scales=False, noop_flag=None, glu_interleave=None,
                                    out=None):
    g, status = _grouped_args(row_offs, colblk_offs, status, col_scale_rows, x.device)
    return _bwd("swiglu", dy, x, s, N, rowwise, colwise, want_dx, want_dscale, workspace,
                g, gemm_scales=gemm_scales, noop_flag=noop_flag, out=out,
                glu_interleave=glu_interleave), status


def grouped_scaled_srelu_mxfp8_bwd(dy, x, s, row_offs, colblk_offs, *, rowwise=True,
                                   colwise=True, want_dx=True, want_dscale=True,
                                   workspace=None, status=None, col_scale_rows=None, N=None,
                                   gemm_scales=False, noop_flag=None, out=None):
    g, status = _grouped_args(row_offs, colblk_offs, status, col_scale_rows, x.device)
    return _bwd("srelu", dy, x, s, N, rowwise, colwise, want_dx, want_dscale, workspace,
                g, gemm_scales=gemm_scales, noop_flag=noop_flag, out=out), status


# ------------------------------------------------------------------ ClampedSwiGLU
CLAMPED_ALPHA = 1.702   # defaults of the reading (the public gpt-oss clamped SwiGLU)
CLAMPED_LIMIT = 7.0


def scaled_clamped_swiglu_mxfp8_fwd(x, s, *, alpha=CLAMPED_ALPHA, limit=CLAMPED_LIMIT,
                                    rowwise=True, colwise=True, N=None, gemm_scales=False,
                                    noop_flag=None, glu_interleave=None, out=None):
    """MXFP8 of ClampedSwiGLU(x) * s (moeact.h); x bf16 [M, >=2N] packs [gate | up]."""
    return _fwd("clamped", x, s, N, rowwise, colwise, False, gemm_scales=gemm_scales,
                clamp=(alpha, limit), noop_flag=noop_flag, out=out,
                glu_interleave=glu_interleave)


def grouped_scaled_clamped_swiglu_mxfp8_fwd(x, s, row_offs, colblk_offs, *, alpha=CLAMPED_ALPHA,
                                            limit=CLAMPED_LIMIT, rowwise=True, colwise=True,
                                            status=None, col_scale_rows=None, N=None,
                                            gemm_scales=False, noop_flag=None,
                                            glu_interleave=None, out=None):
    g, status = _grouped_args(row_offs, colblk_offs, status, col_scale_rows, x.device)
    return _fwd("clamped", x, s, N, rowwise, colwise, False, g, gemm_scales=gemm_scales,
                clamp=(alpha, limit), noop_flag=noop_flag, out=out,
                glu_interleave=glu_interleave), status


def scaled_clamped_swiglu_mxfp8_bwd(dy, x, s, *, alpha=CLAMPED_ALPHA, limit=CLAMPED_LIMIT,
                                    rowwise=True, colwise=True, want_dx=True, want_dscale=True,
                                    workspace=None, N=None, gemm_scales=False, noop_flag=None,
                                    glu_interleave=None, out=None):
    return _bwd("clamped", dy, x, s, N, rowwise, colwise, want_dx, want_dscale, workspace,
                gemm_scales=gemm_scales, clamp=(alpha, limit), noop_flag=noop_flag, out=out,
                glu_interleave=glu_interleave)


def grouped_scaled_clamped_swiglu_mxfp8_bwd(dy, x, s, row_offs, colblk_offs, *,
                                            alpha=CLAMPED_ALPHA, limit=CLAMPED_LIMIT,
                                            rowwise=True, colwise=True, want_dx=True,
                                            want_dscale=True, workspace=None, status=None,
                                            col_scale_rows=None, N=None, gemm_scales=False,
                                            noop_flag=None, glu_interleave=None, out=None):
    g, status = _grouped_args(row_offs, colblk_offs, status, col_scale_rows, x.device)
    return _bwd("clamped", dy, x, s, N, rowwise, colwise, want_dx, want_dscale, workspace, g,
                gemm_scales=gemm_scales, clamp=(alpha, limit), noop_flag=noop_flag, out=out,
                glu_interleave=glu_interleave), status


def init_clamped(alpha=CLAMPED_ALPHA, limit=CLAMPED_LIMIT):
    """Build the sigmoid table of a ClampedSwiGLU (slope, limit) on the current
    device (the first call with that pair would; this one may precede a
    capture)."""
    _capi.call("moeact_init_clamped", alpha, limit)


def clamped_sigmoid_table(alpha=CLAMPED_ALPHA, limit=float("inf"), device="cuda"):
    """fp32 sigma(RN(alpha * min(g, limit))) for all 65536 bf16 g, as the
    kernels look it up."""
    out = torch.empty(65536, dtype=torch.float32, device=device)
    _capi.call("moeact_clamped_sigmoid_dump", alpha, limit, _ptr(out), _stream(out.device))
    return out


# ------------------------------------------------------------------ misc
def init():
    """Set up the current device (sigmoid table); call before any stream capture."""
    _capi.call("moeact_init")


def sigmoid_table(device="cuda"):
    """fp32 sigma for all 65536 bf16 bit patterns, as the kernels compute it."""
    out = torch.empty(65536, dtype=torch.float32, device=device)
    _capi.call("moeact_sigmoid_dump", _ptr(out), _stream(out.device))
    return out


# ------------------------------------------------------------------ activation -> FC2
def grouped_scaled_swiglu_mxfp8_fc2(x, s, row_offs, w_codes, w_scales, *, status=None,
                                    staged_rounding=False, out=None, noop_flag=None):
    """The scaled SwiGLU + rowwise MXFP8 of each expert's rows fused with the
    expert's FC2 GEMM on the tensor cores (TE PR #3238: the quantized grouped
    activation feeds the grouped linear after it).

    x bf16 [M, 2N] ([gate | up]), s fp32 [M], row_offs int64 [E + 1] (from
    splits_to_offsets); w_codes E4M3 [E, H, N] (uint8 or float8_e4m3fn) whose
    bytes hold each expert's [H, N] code matrix (row h = output column h) in
    the tensor cores' tiled operand layout (128 x 128 tiles of 16 KiB, rows
    128-byte swizzled; see include/moeact.h), w_scales uint8 E8M0
    [E, H, N/32] whose bytes hold each expert's [H, N/32] scale matrix in the
    GEMM-ready tiled layout (128 x 4 tiles of 512 bytes, as gemm_scales=True
    writes).
    Returns (out bf16 [M, H], status); `out=` takes a caller-owned bf16
    [M, >= H] tensor with unit column stride."""
    N = x.shape[1] // 2
    _check_rows(x, "x", torch.bfloat16, 2 * N)
    M = x.shape[0]
    _check_s(s, M, x.device)
    dev = x.device
    if w_codes.dtype == torch.float8_e4m3fn:
        w_codes = w_codes.view(torch.uint8)
    if w_codes.dtype != torch.uint8 or w_codes.dim() != 3 or w_codes.shape[2] != N or \
            not w_codes.is_contiguous() or w_codes.device != dev:
        raise ValueError(f"w_codes must be a contiguous uint8 / float8_e4m3fn [E, H, {N}] tensor "
                         f"on {dev}")
    E, H = w_codes.shape[0], w_codes.shape[1]
    if w_scales.dtype != torch.uint8 or tuple(w_scales.shape) != (E, H, N // 32) or \
            not w_scales.is_contiguous() or w_scales.device != dev:
        raise ValueError(f"w_scales must be a contiguous uint8 [{E}, {H}, {N // 32}] tensor on {dev}")
    if row_offs.dtype != torch.int64 or tuple(row_offs.shape) != (E + 1,) or not row_offs.is_cuda:
        raise ValueError(f"row_offs must be an int64 CUDA tensor of {E + 1} offsets")
    if status is None:
        status = torch.empty(1, dtype=torch.int32, device=dev)
    if out is None:
        out = torch.empty((M, H), dtype=torch.bfloat16, device=dev)
    elif out.dtype != torch.bfloat16 or out.dim() != 2 or out.shape[0] != M or \
            out.shape[1] < H or out.stride(1) != 1 or out.device != dev:
        raise ValueError(f"out must be a bf16 [{M}, >= {H}] tensor with unit column stride on {dev}")
    if noop_flag is not None and (noop_flag.dtype != torch.int32 or not noop_flag.is_cuda):
        raise ValueError("noop_flag must be an int32 CUDA tensor")
    if M == 0:
        status.zero_()
        return out, status
    ldx = x.stride(0) if M > 1 else max(x.stride(0), x.shape[1])
    ldo = out.stride(0) if M > 1 else max(out.stride(0), H)
    _capi.call("grouped_scaled_swiglu_mxfp8_fc2", _ptr(x), ldx, _ptr(s), M, N,
               int(bool(staged_rounding)), _ptr(row_offs), E, _ptr(status), _ptr(w_codes),
               _ptr(w_scales), H, _ptr(out), ldo, _ptr(noop_flag), _stream(dev))
    return out, status

"""Plain CPU oracle for the scaled gated activation + MXFP8 path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(``moe_gated_activation_b200``) never imports, loads or calls it, and this
package never imports the product.

The arithmetic lives in ``moeact_oracle.c`` (plain C, IEEE binary32 steps in the
order the method states, binary128 for the sigmoid, binary64 for sums); this
module only compiles it with gcc and marshals numpy arrays through ctypes (and,
for inputs whose gate and up columns are interleaved, rearranges columns around
those calls).

Array conventions (all numpy, C-contiguous):
  bf16 data is passed as ``uint16`` bit patterns; fp32 as ``float32``;
  E4M3 codes and E8M0 scales as ``uint8``; offsets as ``int64``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

ROWWISE = 1
COLWISE = 2
SWIGLU = 0
SRELU = 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moeact_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-Wall", "-Wextra", "-std=gnu11"]

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` with gcc if it is missing or older than the source."""
    with _lock:
        stale = (not os.path.exists(_LIB)
                 or os.path.getmtime(_LIB) < os.path.getmtime(_SRC))
        if force or stale:
            tmp = _LIB + f".tmp{os.getpid()}"
            cmd = ["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lquadmath", "-lm", "-lpthread"]
            subprocess.run(cmd, check=True)
            os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    I32 = ctypes.c_int32
    I = ctypes.c_int
    lib.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
    lib.orc_bf16_to_f32.restype = ctypes.c_float
    lib.orc_f32_to_bf16.argtypes = [ctypes.c_float]
    lib.orc_f32_to_bf16.restype = ctypes.c_uint16
    lib.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.orc_e4m3_decode.restype = ctypes.c_double
    lib.orc_e4m3_encode.argtypes = [ctypes.c_double]
    lib.orc_e4m3_encode.restype = ctypes.c_uint8
    lib.orc_e8m0_rceil.argtypes = [ctypes.c_float]
    lib.orc_e8m0_rceil.restype = I
    lib.orc_sigma_init.argtypes = []
    lib.orc_sigma_init.restype = I
    lib.orc_sigmoid_bf16.argtypes = [ctypes.c_uint16]
    lib.orc_sigmoid_bf16.restype = ctypes.c_float
    lib.orc_act_fwd.argtypes = [I, P, I64, P, I64, I64, I, I, P, P, P, P]
    lib.orc_act_fwd.restype = I
    lib.orc_act_values.argtypes = [I, P, I64, P, I64, I64, I, P]
    lib.orc_act_values.restype = I
    lib.orc_mxfp8_quantize.argtypes = [P, I64, I64, I, P, P, P, P]
    lib.orc_mxfp8_quantize.restype = I
    lib.orc_act_bwd.argtypes = [I, P, I64, P, I64, P, I64, I64, I, P, P, P, P, P, P]
    lib.orc_act_bwd.restype = I
    lib.orc_splits_to_offsets.argtypes = [P, I32, I64, P, P]
    lib.orc_splits_to_offsets.restype = I
    lib.orc_grouped_act_fwd.argtypes = [I, P, I64, P, I64, I64, I, I, P, P, I32, P, P, P, P]
    lib.orc_grouped_act_fwd.restype = I
    lib.orc_grouped_act_bwd.argtypes = [I, P, I64, P, I64, P, I64, I64, I, P, P, I32,
                                        P, P, P, P, P, P]
    lib.orc_grouped_act_bwd.restype = I
    F = ctypes.c_float
    lib.orc_clamped_fwd.argtypes = [P, I64, P, I64, I64, I, F, F, P, P, P, P]
    lib.orc_clamped_fwd.restype = I
    lib.orc_clamped_values.argtypes = [P, I64, P, I64, I64, F, F, P]
    lib.orc_clamped_values.restype = I
    lib.orc_clamped_bwd.argtypes = [P, I64, P, I64, P, I64, I64, I, F, F, P, P, P, P, P, P]
    lib.orc_clamped_bwd.restype = I
    lib.orc_grouped_clamped_fwd.argtypes = [P, I64, P, I64, I64, I, F, F, P, P, I32,
                                            P, P, P, P]
    lib.orc_grouped_clamped_fwd.restype = I
    lib.orc_grouped_clamped_bwd.argtypes = [P, I64, P, I64, P, I64, I64, I, F, F, P, P, I32,
                                            P, P, P, P, P, P]
    lib.orc_grouped_clamped_bwd.restype = I
    lib.orc_clamped_sigmoid.argtypes = [F, ctypes.c_uint16, ctypes.POINTER(I)]
    lib.orc_clamped_sigmoid.restype = F
    lib.orc_scales_gemm_layout.argtypes = [P, I64, I64, P]
    lib.orc_scales_gemm_layout.restype = None
    lib.orc_col_scales_gemm_layout.argtypes = [P, I64, P, P, I32, P]
    lib.orc_col_scales_gemm_layout.restype = I
    if lib.orc_sigma_init() != 0:
        raise RuntimeError("oracle: sigmoid table has uncertified roundings")
    _lib = lib
    return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    return a


# ---------------------------------------------------------------- scalars
def bf16_to_f32(b: int) -> float:
    return _load().orc_bf16_to_f32(b)


def f32_to_bf16(f: float) -> int:
    return _load().orc_f32_to_bf16(f)


def e4m3_decode(c: int) -> float:
    return _load().orc_e4m3_decode(c)


def e4m3_encode(x: float) -> int:
    return _load().orc_e4m3_encode(x)


def e8m0_rceil(amax: float) -> int:
    return _load().orc_e8m0_rceil(amax)


def sigmoid_bf16(bits: int) -> float:
    return _load().orc_sigmoid_bf16(bits)


def sigmoid_table() -> np.ndarray:
    """fp32 sigma for every bf16 bit pattern 0..65535."""
    lib = _load()
    return np.array([lib.orc_sigmoid_bf16(b) for b in range(65536)], dtype=np.float32)


# ---------------------------------------------------------------- helpers
def mx_widths(M: int, W: int):
    """Shapes of (row codes, row scales, col codes, col scales) for [M, W]."""
    return (M, W), (M, W // 32), (M, W), ((M + 31) // 32, W)


def _alloc_mx(M, W, dirs, colblk_rows=None):
    rq, rs, cq, cs = mx_widths(M, W)
    if colblk_rows is not None:
        cs = (colblk_rows, W)
    out = {"row_codes": None, "row_scales": None, "col_codes": None, "col_scales": None}
    if dirs & ROWWISE:
        out["row_codes"] = np.zeros(rq, np.uint8)
        out["row_scales"] = np.zeros(rs, np.uint8)
    if dirs & COLWISE:
        out["col_codes"] = np.zeros(cq, np.uint8)
        out["col_scales"] = np.zeros(cs, np.uint8)
    return out


def _mx_ptrs(out):
    return (_ptr(out["row_codes"]), _ptr(out["row_scales"]),
            _ptr(out["col_codes"]), _ptr(out["col_scales"]))


# ---------------------------------------------------------------- forward
def act_fwd(x_bits: np.ndarray, s: np.ndarray, N: int, dirs: int, act: int = SWIGLU,
            staged: bool = False, ldx: int | None = None) -> dict:
    """Forward: MXFP8 of y = act(x) * s.  x_bits uint16 [M, ldx]."""
    x_bits = _c(x_bits, np.uint16)
    s = _c(s, np.float32)
    M = x_bits.shape[0]
    ldx = x_bits.shape[1] if ldx is None else ldx
    out = _alloc_mx(M, N, dirs)
    rc = _load().orc_act_fwd(act, _ptr(x_bits), ldx, _ptr(s), M, N, dirs, int(staged),
                             *_mx_ptrs(out))
    if rc:
        raise ValueError(f"oracle act_fwd failed ({rc})")
    return out


def act_values(x_bits: np.ndarray, s: np.ndarray, N: int, act: int = SWIGLU,
               staged: bool = False) -> np.ndarray:
    """The fp32 activation y = act(x) * s before quantization, [M, N]."""
    x_bits = _c(x_bits, np.uint16)
    s = _c(s, np.float32)
    M = x_bits.shape[0]
    y = np.zeros((M, N), np.float32)
    _load().orc_act_values(act, _ptr(x_bits), x_bits.shape[1], _ptr(s), M, N, int(staged),
                           _ptr(y))
    return y


def mxfp8_quantize(y: np.ndarray, dirs: int) -> dict:
    """Stand-alone MXFP8 quantizer of an fp32 [M, W] matrix."""
    y = _c(y, np.float32)
    M, W = y.shape
    out = _alloc_mx(M, W, dirs)
    rc = _load().orc_mxfp8_quantize(_ptr(y), M, W, dirs, *_mx_ptrs(out))
    if rc:
        raise ValueError(f"oracle mxfp8_quantize failed ({rc})")
    return out


# ---------------------------------------------------------------- backward
def act_bwd(dy_bits: np.ndarray, x_bits: np.ndarray, s: np.ndarray, N: int, dirs: int,
            act: int = SWIGLU, want_dx: bool = True, want_dscale: bool = True) -> dict:
    """Backward: dx (bf16 bits [M, W]), dscale (fp32 [M]) and MXFP8 of dx."""
    dy_bits = _c(dy_bits, np.uint16)
    x_bits = _c(x_bits, np.uint16)
    s = _c(s, np.float32)
    M = x_bits.shape[0]
    W = 2 * N if act == SWIGLU else N
    out = _alloc_mx(M, W, dirs)
    out["dx"] = np.zeros((M, W), np.uint16) if want_dx else None
    out["dscale"] = np.zeros(M, np.float32) if want_dscale else None
    rc = _load().orc_act_bwd(act, _ptr(dy_bits), dy_bits.shape[1], _ptr(x_bits),
                             x_bits.shape[1], _ptr(s), M, N, dirs,
                             _ptr(out["dx"]), _ptr(out["dscale"]), *_mx_ptrs(out))
    if rc:
        raise ValueError(f"oracle act_bwd failed ({rc})")
    return out


# ---------------------------------------------------------------- grouped
def splits_to_offsets(m_splits: np.ndarray, total_rows: int):
    """(status, row_offs[E+1], colblk_offs[E+1]); offsets are None on error."""
    m = _c(m_splits, np.int64)
    E = m.shape[0]
    ro = np.zeros(E + 1, np.int64)
    co = np.zeros(E + 1, np.int64)
    st = _load().orc_splits_to_offsets(_ptr(m), E, total_rows, _ptr(ro), _ptr(co))
    if st:
        return st, None, None
    return 0, ro, co


def grouped_act_fwd(x_bits, s, N, dirs, row_offs, colblk_offs, act=SWIGLU, staged=False):
    x_bits = _c(x_bits, np.uint16)
    s = _c(s, np.float32)
    ro = _c(row_offs, np.int64)
    co = _c(colblk_offs, np.int64)
    E = ro.shape[0] - 1
    M = x_bits.shape[0]
    out = _alloc_mx(M, N, dirs, colblk_rows=int(co[-1]))
    rc = _load().orc_grouped_act_fwd(act, _ptr(x_bits), x_bits.shape[1], _ptr(s), M, N, dirs,
                                     int(staged), _ptr(ro), _ptr(co), E, *_mx_ptrs(out))
    if rc:
        raise ValueError(f"oracle grouped_act_fwd failed ({rc})")
    return out


def grouped_act_bwd(dy_bits, x_bits, s, N, dirs, row_offs, colblk_offs, act=SWIGLU,
                    want_dx=True, want_dscale=True):
    dy_bits = _c(dy_bits, np.uint16)
    x_bits = _c(x_bits, np.uint16)
    s = _c(s, np.float32)
    ro = _c(row_offs, np.int64)
    co = _c(colblk_offs, np.int64)
    E = ro.shape[0] - 1
    M = x_bits.shape[0]
    W = 2 * N if act == SWIGLU else N
    out = _alloc_mx(M, W, dirs, colblk_rows=int(co[-1]))
    out["dx"] = np.zeros((M, W), np.uint16) if want_dx else None
    out["dscale"] = np.zeros(M, np.float32) if want_dscale else None
    rc = _load().orc_grouped_act_bwd(act, _ptr(dy_bits), dy_bits.shape[1], _ptr(x_bits),
                                     x_bits.shape[1], _ptr(s), M, N, dirs, _ptr(ro), _ptr(co), E,
                                     _ptr(out["dx"]), _ptr(out["dscale"]), *_mx_ptrs(out))
    if rc:
        raise ValueError(f"oracle grouped_act_bwd failed ({rc})")
    return out


# ---------------------------------------------------------------- GEMM-ready scales
def scales_gemm_layout(S: np.ndarray) -> np.ndarray:
    """E8M0 matrix [R, C] -> the 128 x 4 tiled GEMM layout (flat uint8,
    ceil(R/128) * ceil(C/4) * 512 bytes, padding 0)."""
    S = _c(S, np.uint8)
    R, C = S.shape
    out = np.zeros(((R + 127) // 128) * ((C + 3) // 4) * 512, np.uint8)
    _load().orc_scales_gemm_layout(_ptr(S), R, C, _ptr(out))
    return out


def codes_gemm_layout(W: np.ndarray) -> np.ndarray:
    """E4M3 codes [R, K] (R, K multiples of 128) -> the tensor cores' K-major
    operand tiles (flat uint8, R * K bytes): 128-row blocks in order, within a
    row block 128-byte k blocks in order, each a 16 KiB tile holding row r's
    128 bytes at offset 128 r with its 16-byte chunk c at chunk position
    c ^ (r mod 8) (the 128-byte swizzle).  A permutation of the bytes (any
    dtype is permuted alike, so an index matrix gives the permutation)."""
    W = np.ascontiguousarray(W)
    R, K = W.shape
    if R % 128 or K % 128:
        raise ValueError("codes_gemm_layout needs rows and columns in multiples of 128")
    src = W.reshape(R // 128, 128, K // 128, 8, 16)      # [row block, r, k block, chunk, byte]
    tiles = np.empty((R // 128, K // 128, 128, 8, 16), W.dtype)
    for r in range(128):
        for c in range(8):
            tiles[:, :, r, c ^ (r % 8), :] = src[:, r, :, c, :]
    return tiles.reshape(-1)


def col_scales_gemm_layout(cs: np.ndarray, W: int, row_offs, colblk_offs) -> np.ndarray:
    """Row-major colwise scales [S, W] of a grouped tensor -> per expert, the
    transposed [W, m_e/32] matrix in the GEMM layout, experts in order."""
    cs = _c(cs, np.uint8)
    ro = _c(row_offs, np.int64)
    co = _c(colblk_offs, np.int64)
    E = ro.shape[0] - 1
    out = np.zeros(max(1, int(ro[-1]) * W // 32), np.uint8)
    if _load().orc_col_scales_gemm_layout(_ptr(cs), W, _ptr(ro), _ptr(co), E, _ptr(out)):
        raise ValueError("GEMM layout needs W and every group's rows to be multiples of 128")
    return out[:int(ro[-1]) * W // 32]


# ---------------------------------------------------------------- ClampedSwiGLU
CLAMPED_ALPHA = 1.702   # defaults of the reading (the public gpt-oss clamped SwiGLU)
CLAMPED_LIMIT = 7.0


def _check_rc(rc, what):
    if rc == 3:
        raise ArithmeticError(f"oracle {what}: a sigma rounding could not be certified")
    if rc:
        raise ValueError(f"oracle {what} failed ({rc})")


def clamped_fwd(x_bits, s, N, dirs, alpha=CLAMPED_ALPHA, limit=CLAMPED_LIMIT):
    """Forward of the scaled ClampedSwiGLU: MXFP8 of h(x) * s, width N."""
    x_bits = _c(x_bits, np.uint16)
    s = _c(s, np.float32)
    M = x_bits.shape[0]
    out = _alloc_mx(M, N, dirs)
    _check_rc(_load().orc_clamped_fwd(_ptr(x_bits), x_bits.shape[1], _ptr(s), M, N, dirs,
                                      alpha, limit, *_mx_ptrs(out)), "clamped_fwd")
    return out


def clamped_values(x_bits, s, N, alpha=CLAMPED_ALPHA, limit=CLAMPED_LIMIT):
    x_bits = _c(x_bits, np.uint16)
    s = _c(s, np.float32)
    M = x_bits.shape[0]
    y = np.zeros((M, N), np.float32)
    _check_rc(_load().orc_clamped_values(_ptr(x_bits), x_bits.shape[1], _ptr(s), M, N, alpha,
                                         limit, _ptr(y)), "clamped_values")
    return y


def clamped_bwd(dy_bits, x_bits, s, N, dirs, alpha=CLAMPED_ALPHA, limit=CLAMPED_LIMIT,
                want_dx=True, want_dscale=True):
    dy_bits = _c(dy_bits, np.uint16)
    x_bits = _c(x_bits, np.uint16)
    s = _c(s, np.float32)
    M = x_bits.shape[0]
    out = _alloc_mx(M, 2 * N, dirs)
    out["dx"] = np.zeros((M, 2 * N), np.uint16) if want_dx else None
    out["dscale"] = np.zeros(M, np.float32) if want_dscale else None
    _check_rc(_load().orc_clamped_bwd(_ptr(dy_bits), dy_bits.shape[1], _ptr(x_bits),
                                      x_bits.shape[1], _ptr(s), M, N, dirs, alpha, limit,
                                      _ptr(out["dx"]), _ptr(out["dscale"]), *_mx_ptrs(out)),
              "clamped_bwd")
    return out


def grouped_clamped_fwd(x_bits, s, N, dirs, row_offs, colblk_offs, alpha=CLAMPED_ALPHA,
                        limit=CLAMPED_LIMIT):
    x_bits = _c(x_bits, np.uint16)
    s = _c(s, np.float32)
    ro = _c(row_offs, np.int64)
    co = _c(colblk_offs, np.int64)
    M = x_bits.shape[0]
    out = _alloc_mx(M, N, dirs, colblk_rows=int(co[-1]))
    _check_rc(_load().orc_grouped_clamped_fwd(_ptr(x_bits), x_bits.shape[1], _ptr(s), M, N,
                                              dirs, alpha, limit, _ptr(ro), _ptr(co),
                                              ro.shape[0] - 1, *_mx_ptrs(out)),
              "grouped_clamped_fwd")
    return out


def grouped_clamped_bwd(dy_bits, x_bits, s, N, dirs, row_offs, colblk_offs,
                        alpha=CLAMPED_ALPHA, limit=CLAMPED_LIMIT):
    dy_bits = _c(dy_bits, np.uint16)
    x_bits = _c(x_bits, np.uint16)
    s = _c(s, np.float32)
    ro = _c(row_offs, np.int64)
    co = _c(colblk_offs, np.int64)
    M = x_bits.shape[0]
    out = _alloc_mx(M, 2 * N, dirs, colblk_rows=int(co[-1]))
    out["dx"] = np.zeros((M, 2 * N), np.uint16)
    out["dscale"] = np.zeros(M, np.float32)
    _check_rc(_load().orc_grouped_clamped_bwd(_ptr(dy_bits), dy_bits.shape[1], _ptr(x_bits),
                                              x_bits.shape[1], _ptr(s), M, N, dirs, alpha,
                                              limit, _ptr(ro), _ptr(co), ro.shape[0] - 1,
                                              _ptr(out["dx"]), _ptr(out["dscale"]),
                                              *_mx_ptrs(out)), "grouped_clamped_bwd")
    return out


def clamped_sigmoid_table(alpha=CLAMPED_ALPHA) -> np.ndarray:
    """sigma(RN(alpha * g)) for all 65536 bf16 g (fp32, correctly rounded)."""
    lib = _load()
    ok = ctypes.c_int(1)
    out = np.array([lib.orc_clamped_sigmoid(alpha, b, ctypes.byref(ok)) for b in range(65536)],
                   np.float32)
    if not ok.value:
        raise ArithmeticError("a sigma rounding could not be certified")
    return out


# ---------------------------------------------------------------- interleaved gate / up
# TE PR #3238, Important Files Changed (swiglu.py row): the GLU interleave
# reshaping of the gated input moves into the scaled_swiglu / scaled_dswiglu
# kernels.  The block order and size are a reading: the 2N columns hold G gate
# columns, then the G up columns paired with them, repeated N / G times; dX
# comes back in the same order, and its MXFP8 blocks run along the stored
# columns.  The functions below only rearrange columns and then call the
# oracle's halves-layout functions and quantizer.
def glu_halves(x_bits, N, G):
    """An interleaved gated input [M, >= 2N] as [gate | up] halves [M, 2N]."""
    x = np.asarray(x_bits)
    M = x.shape[0]
    blocks = x[:, :2 * N].reshape(M, N // G, 2, G)
    return np.ascontiguousarray(np.concatenate(
        [blocks[:, :, 0, :].reshape(M, N), blocks[:, :, 1, :].reshape(M, N)], axis=1))


def glu_interleave(a, N, G):
    """[gate | up] halves [M, 2N] -> the interleaved column order."""
    a = np.asarray(a)
    M = a.shape[0]
    g = a[:, :N].reshape(M, N // G, 1, G)
    u = a[:, N:2 * N].reshape(M, N // G, 1, G)
    return np.ascontiguousarray(np.concatenate([g, u], axis=2).reshape(M, 2 * N))


def _quantize_grouped(y, dirs, row_offs=None, colblk_offs=None):
    """MXFP8 of y [M, W]; with offsets, each group's rows on their own
    (colwise blocks end at group boundaries, col scales at colblk_offs[e])."""
    if row_offs is None:
        return mxfp8_quantize(y, dirs)
    ro = _c(row_offs, np.int64)
    co = _c(colblk_offs, np.int64)
    M, W = y.shape
    out = _alloc_mx(M, W, dirs, colblk_rows=int(co[-1]))
    for e in range(ro.shape[0] - 1):
        r0, r1 = int(ro[e]), int(ro[e + 1])
        if r1 == r0:
            continue
        q = mxfp8_quantize(y[r0:r1], dirs)
        if dirs & ROWWISE:
            out["row_codes"][r0:r1] = q["row_codes"]
            out["row_scales"][r0:r1] = q["row_scales"]
        if dirs & COLWISE:
            out["col_codes"][r0:r1] = q["col_codes"]
            c0 = int(co[e])
            out["col_scales"][c0:c0 + q["col_scales"].shape[0]] = q["col_scales"]
    return out


def interleaved_fwd(x_bits, s, N, dirs, G, act="swiglu", staged=False, row_offs=None,
                    colblk_offs=None, alpha=CLAMPED_ALPHA, limit=CLAMPED_LIMIT):
    """Forward of a gated activation whose input interleaves gate and up in
    blocks of G columns (act "swiglu" or "clamped"; grouped with offsets)."""
    xc = glu_halves(x_bits, N, G)
    grouped = row_offs is not None
    if act == "clamped":
        if grouped:
            return grouped_clamped_fwd(xc, s, N, dirs, row_offs, colblk_offs, alpha, limit)
        return clamped_fwd(xc, s, N, dirs, alpha, limit)
    if grouped:
        return grouped_act_fwd(xc, s, N, dirs, row_offs, colblk_offs, SWIGLU, staged)
    return act_fwd(xc, s, N, dirs, SWIGLU, staged)


def interleaved_bwd(dy_bits, x_bits, s, N, dirs, G, act="swiglu", row_offs=None,
                    colblk_offs=None, alpha=CLAMPED_ALPHA, limit=CLAMPED_LIMIT):
    """Backward with interleaved gate / up: dx [M, 2N] in the interleaved
    order, dscale, and the MXFP8 of that dx (of its bf16 values)."""
    xc = glu_halves(x_bits, N, G)
    if act == "clamped":
        r = clamped_bwd(dy_bits, xc, s, N, 0, alpha, limit)
    else:
        r = act_bwd(dy_bits, xc, s, N, 0, SWIGLU)
    dx = glu_interleave(r["dx"], N, G)
    y = (dx.astype(np.uint32) << 16).view(np.float32)
    out = _quantize_grouped(y, dirs, row_offs, colblk_offs)
    out["dx"] = dx
    out["dscale"] = r["dscale"]
    return out



# ---------------------------------------------------------------- activation -> FC2 GEMM
# TE PR #3238, Greptile summary and sequence diagram: the grouped activation
# hands its quantized grouped tensor straight to the grouped linear that
# follows it (ForwardScaledActivationGroupedLinear).  Here that linear is the
# expert's FC2: out[i, h] = sum_k A[i, k] * W_e[h, k] for a row i of expert e,
# where A is the rowwise (1 x 32 along k) MXFP8 of the scaled SwiGLU output
# -- the forward above, rowwise only (rowwise blocks never depend on the
# grouping) -- and W_e [H, N] is the expert's weight, itself MXFP8 with 1 x 32
# blocks along k.  Both are taken at their exact dequantized values
# (code value x 2^(scale - 127)); the product is summed in binary64 by a
# library matmul, the one step a library routine performs.
def e4m3_values() -> np.ndarray:
    """The value of every E4M3 code (binary64, exact), NaN for 0x7F / 0xFF."""
    lib = _load()
    return np.array([lib.orc_e4m3_decode(c) for c in range(256)], np.float64)


def mxfp8_dequantize_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Exact values of rowwise MXFP8 data: codes uint8 [..., W], E8M0 scales
    uint8 [..., W/32] (255 is NaN)."""
    codes = np.asarray(codes, np.uint8)
    scales = np.asarray(scales, np.uint8)
    v = e4m3_values()[codes]
    mult = np.where(scales == 255, np.nan, np.ldexp(1.0, scales.astype(np.int64) - 127))
    return v * np.repeat(mult, 32, axis=-1)


def grouped_fc2(x_bits, s, N, row_offs, w_codes, w_scales, staged=False) -> np.ndarray:
    """out [M, H] (binary64) of the activation -> MXFP8 -> FC2 path: rows
    [row_offs[e], row_offs[e+1]) use expert e's weight (w_codes uint8
    [E, H, N] E4M3, w_scales uint8 [E, H, N/32] E8M0)."""
    a = act_fwd(x_bits, s, N, ROWWISE, SWIGLU, staged)
    a_val = mxfp8_dequantize_rows(a["row_codes"], a["row_scales"])
    ro = _c(row_offs, np.int64)
    E, H = w_codes.shape[0], w_codes.shape[1]
    out = np.zeros((a_val.shape[0], H), np.float64)
    for e in range(E):
        r0, r1 = int(ro[e]), int(ro[e + 1])
        if r1 > r0:
            w_val = mxfp8_dequantize_rows(w_codes[e], w_scales[e])
            out[r0:r1] = a_val[r0:r1] @ w_val.T
    return out

"""Comparison rules for the CUDA path against the oracle (test helper).

The bar (the stated contract for this path): offsets and E8M0 scales
bit-exact; E4M3 codes exact except at most one code step on at most 1e-4 of
the elements; bf16 gradients within 2 bf16 ulp; dscale relative error 1e-3
(with an absolute floor for rows whose sum cancels: |d| <= 1e-3 |ref| +
1e-6 sum_j |dY h|).  NaN compares equal to NaN.
"""
import numpy as np
import torch

CODE_FRAC = 1e-4


def u8(t):
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t
    return t.detach().view(torch.uint8).cpu().numpy() if t.dtype != torch.uint8 \
        else t.detach().cpu().numpy()


def bf16_u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def assert_scales_exact(got, ref, what):
    got, ref = u8(got), u8(ref)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    bad = np.nonzero(got != ref)
    assert bad[0].size == 0, f"{what}: {bad[0].size} scale bytes differ, first at " \
        f"{tuple(int(b[0]) for b in bad)}: got {got[tuple(b[0] for b in bad)]} " \
        f"ref {ref[tuple(b[0] for b in bad)]}"


def code_mismatches(got, ref):
    """(count, max step) of E4M3 code differences; a step is the distance in
    the ordered magnitude space of one sign."""
    got, ref = u8(got).astype(np.int32), u8(ref).astype(np.int32)
    diff = got != ref
    n = int(diff.sum())
    if n == 0:
        return 0, 0
    g, r = got[diff], ref[diff]
    same_sign = (g & 0x80) == (r & 0x80)
    step = np.where(same_sign, np.abs((g & 0x7F) - (r & 0x7F)), 256)
    return n, int(step.max())


def assert_codes(got, ref, what, exact=False):
    got, ref = u8(got), u8(ref)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    n, step = code_mismatches(got, ref)
    if exact:
        assert n == 0, f"{what}: {n} E4M3 codes differ (max step {step})"
    else:
        assert step <= 1 and n <= CODE_FRAC * got.size, \
            f"{what}: {n} E4M3 codes differ (max step {step}) of {got.size}"


def assert_bf16_close(got_u16, ref_u16, what, ulps=2):
    g = got_u16.astype(np.int32)
    r = ref_u16.astype(np.int32)
    gn = ((g & 0x7F80) == 0x7F80) & ((g & 0x7F) != 0)
    rn = ((r & 0x7F80) == 0x7F80) & ((r & 0x7F) != 0)
    assert np.array_equal(gn, rn), f"{what}: NaN positions differ"
    # ordered integer images: sign-magnitude -> two's complement order
    go = np.where(g & 0x8000, -(g & 0x7FFF), g & 0x7FFF)
    ro = np.where(r & 0x8000, -(r & 0x7FFF), r & 0x7FFF)
    d = np.abs(go - ro)[~gn]
    assert d.size == 0 or d.max() <= ulps, f"{what}: max {int(d.max())} bf16 ulps"


def assert_dscale(got, ref, bound_abs, what):
    got = got.detach().cpu().numpy() if isinstance(got, torch.Tensor) else got
    gn, rn = np.isnan(got), np.isnan(ref)
    assert np.array_equal(gn, rn), f"{what}: NaN positions differ"
    ok = ~gn
    err = np.abs(got[ok].astype(np.float64) - ref[ok].astype(np.float64))
    lim = 1e-3 * np.abs(ref[ok].astype(np.float64)) + 1e-6 * bound_abs[ok]
    assert (err <= lim).all(), f"{what}: max excess {float((err - lim).max())}"


def dscale_abs_bound(dy_bits, x_bits, s, N, act_swiglu=True):
    """sum_j |dY * h| per row in float64 (for the absolute floor)."""
    dy = torch.from_numpy(dy_bits.view(np.int16)).view(torch.bfloat16).double()[:, :N]
    x = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).double()
    if act_swiglu:
        g, u = x[:, :N], x[:, N:2 * N]
        h = g * torch.sigmoid(g) * u
    else:
        h = torch.clamp(x[:, :N], min=0) ** 2
    return (dy.abs() * h.abs()).sum(1).numpy()


def compare_mx(got, ref, what, exact=True):
    """got: ops.MXFP8; ref: oracle dict."""
    if ref["row_codes"] is not None:
        assert_scales_exact(got.row_scales, ref["row_scales"], what + " row scales")
        assert_codes(got.row_codes, ref["row_codes"], what + " row codes", exact)
    else:
        assert got.row_codes.numel() == 0 and got.row_scales.numel() == 0
    if ref["col_codes"] is not None:
        assert_scales_exact(got.col_scales, ref["col_scales"], what + " col scales")
        assert_codes(got.col_codes, ref["col_codes"], what + " col codes", exact)
    else:
        assert got.col_codes.numel() == 0 and got.col_scales.numel() == 0


# ------------------------------------------------------------------ GEMM scale layout
def unblock_rows(buf, R, C):
    """Inverse of the GEMM-ready tiled scale layout for an [R, C] matrix with
    R % 128 == 0 and C % 4 == 0 (tiles [R/128, C/4] of 32 x 4 x 4 bytes
    ordered (r0, r1, c), row r = 128 t + 32 r1 + r0), via tensor reshapes."""
    t = torch.as_tensor(np.asarray(buf)).reshape(R // 128, C // 4, 32, 4, 4)
    return t.permute(0, 3, 2, 1, 4).reshape(R, C).numpy()


def unblock_cols(buf, W, m_splits):
    """Row-major colwise scales [sum m_e/32, W] from the GEMM-ready layout:
    per group, tiles of the transposed [W, m_e/32] matrix."""
    buf = np.asarray(buf).reshape(-1)
    parts, pos = [], 0
    for me in m_splits:
        kb = int(me) // 32
        n = W * kb
        if n:
            blk = unblock_rows(buf[pos:pos + n], W, kb)   # [W, m_e/32]
            parts.append(np.ascontiguousarray(blk.T))
        pos += n
    return np.concatenate(parts) if parts else np.zeros((0, W), np.uint8)

"""Parity at the full workload sizes, in the launch configuration the
benchmark times: the whole forward and backward run on the GPU; sampled
32-row slabs (each one complete colwise block inside one expert, so the
oracle can compute it on its own) are compared with the oracle element by
element, and properties that hold at any size are checked on the whole output.
"""
import numpy as np
import pytest
import torch

import oracle
import moe_gated_activation_b200 as mg
from moe_gated_activation_b200.workloads import WORKLOADS, bf16_bits, make_inputs
from parity import (assert_codes, assert_dscale, assert_scales_exact, bf16_u16,
                    dscale_abs_bound, u8)

pytestmark = pytest.mark.gpu


def _slabs(wl, m_splits, seed):
    """(row0, nrows, col-scale row) of sampled slabs."""
    M = wl.M
    if not wl.grouped:
        S = (M + 31) // 32
        rng = np.random.default_rng(seed)
        idx = sorted({0, 1, S // 3, S // 2, S - 2, S - 1, *rng.integers(0, S, 3).tolist()})
        return [(32 * i, min(32, M - 32 * i), i) for i in idx if 0 <= i < S]
    m = m_splits.numpy()
    st, ro, cb = oracle.splits_to_offsets(m, M)
    assert st == 0
    nz = [e for e in range(len(m)) if m[e] > 0]
    rng = np.random.default_rng(seed)
    pick = {nz[0], nz[-1], max(nz, key=lambda e: m[e]), min(nz, key=lambda e: m[e]),
            *rng.choice(nz, 2, replace=False).tolist()}
    out = []
    for e in sorted(pick):
        nslab = int(cb[e + 1] - cb[e])
        for k in sorted({0, nslab - 1}):
            r0 = int(ro[e]) + 32 * k
            out.append((r0, min(32, int(ro[e + 1]) - r0), int(cb[e]) + k))
    return out


def _run(wl, inp, act, staged, device):
    x, s, dy = inp["x"], inp["s"], inp["dy"]
    if wl.grouped:
        ms = inp["m_splits"].to(device)
        ro, cb, st = mg.splits_to_offsets(ms, wl.M)
        S = int(((inp["m_splits"] + 31) // 32).sum())
        if act == "swiglu":
            f, fst = mg.grouped_scaled_swiglu_mxfp8_fwd(x, s, ro, cb, staged_rounding=staged,
                                                        col_scale_rows=S)
            b, bst = (mg.grouped_scaled_swiglu_mxfp8_bwd(dy, x, s, ro, cb, col_scale_rows=S)
                      if dy is not None else (None, None))
        else:
            f, fst = mg.grouped_scaled_srelu_mxfp8_fwd(x, s, ro, cb, col_scale_rows=S)
            b, bst = mg.grouped_scaled_srelu_mxfp8_bwd(dy, x, s, ro, cb, col_scale_rows=S)
        torch.cuda.synchronize()
        assert int(st.item()) == 0 and int(fst.item()) == 0
        assert bst is None or int(bst.item()) == 0
        return f, b
    if act == "swiglu":
        f = mg.scaled_swiglu_mxfp8_fwd(x, s, staged_rounding=staged)
        b = mg.scaled_swiglu_mxfp8_bwd(dy, x, s) if dy is not None else None
    else:
        f = mg.scaled_srelu_mxfp8_fwd(x, s)
        b = mg.scaled_srelu_mxfp8_bwd(dy, x, s)
    torch.cuda.synchronize()
    return f, b


def _check(wl, inp, f, b, act, staged, N):
    actc = oracle.SWIGLU if act == "swiglu" else oracle.SRELU
    W = 2 * N if act == "swiglu" else N
    for r0, n, cs_row in _slabs(wl, inp["m_splits"], wl.seed):
        rows = slice(r0, r0 + n)
        xb = bf16_bits(inp["x"][rows])
        sv = inp["s"][rows].cpu().numpy()
        ref = oracle.act_fwd(xb, sv, N, 3, act=actc, staged=staged)
        what = f"{wl.key} {act} fwd rows {r0}+{n}"
        assert_scales_exact(f.row_scales[rows], ref["row_scales"], what + " row scales")
        assert_codes(f.row_codes[rows], ref["row_codes"], what + " row codes", exact=True)
        assert_scales_exact(f.col_scales[cs_row:cs_row + 1], ref["col_scales"], what + " col scales")
        assert_codes(f.col_codes[rows], ref["col_codes"], what + " col codes", exact=True)
        if b is None:
            continue
        dyb = bf16_bits(inp["dy"][rows])
        refb = oracle.act_bwd(dyb, xb, sv, N, 3, act=actc)
        what = f"{wl.key} {act} bwd rows {r0}+{n}"
        assert np.array_equal(bf16_u16(b.dx[rows]), refb["dx"]), what + " dx"
        assert_dscale(b.dscale[rows], refb["dscale"], dscale_abs_bound(dyb, xb, sv, N, act == "swiglu"),
                      what + " dscale")
        assert_scales_exact(b.mx.row_scales[rows], refb["row_scales"], what + " row scales")
        assert_codes(b.mx.row_codes[rows], refb["row_codes"], what + " row codes", exact=True)
        assert_scales_exact(b.mx.col_scales[cs_row:cs_row + 1], refb["col_scales"], what + " col scales")
        assert_codes(b.mx.col_codes[rows], refb["col_codes"], what + " col codes", exact=True)
    # properties over the whole output: every block max code in [0x76, 0x7E]
    # (no NaN/Inf/zero blocks occur in these inputs)
    for mx, w in ((f, N),) + (((b.mx, W),) if b is not None else ()):
        rq = mx.row_codes.view(torch.uint8)
        blk = (rq & 0x7F).view(rq.shape[0], w // 32, 32).amax(dim=2)
        live = mx.row_scales > 0
        assert bool(((blk >= 0x76) & (blk <= 0x7E))[live].all())


@pytest.mark.parametrize("key", ["c1", "c2", "c3", "c4", "c5"])
def test_workload_sampled_parity(cuda_device, key):
    wl = WORKLOADS[key]
    inp = make_inputs(wl, device=cuda_device)
    for staged in wl.staged:
        f, b = _run(wl, inp, "swiglu", staged, cuda_device)
        _check(wl, inp, f, b if not staged else None, "swiglu", staged, wl.N)
        del f, b
    del inp
    if wl.srelu_N:
        inp = make_inputs(wl, device=cuda_device, srelu=True)
        f, b = _run(wl, inp, "srelu", False, cuda_device)
        _check(wl, inp, f, b, "srelu", False, wl.srelu_N)
        del f, b, inp
    torch.cuda.empty_cache()

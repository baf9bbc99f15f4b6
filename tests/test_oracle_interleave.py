"""Pins of the oracle's interleaved gate / up layout (TE PR #3238, Important
Files Changed, swiglu.py row: the GLU interleave reshaping moves into the
scaled_swiglu / scaled_dswiglu kernels; block order and size are a reading).

The interleaved functions rearrange columns around the halves-layout oracle,
so they are pinned by (a) the layout built element by element with loops
from its description, (b) the special case G = N, which is the halves layout
itself, and (c) block-permutation invariance of MXFP8: with G a multiple of
32 every 1x32 block of the stored dX is one whole block of dgate or of dup,
and every column keeps its own colwise blocks, so the interleaved MXFP8 is
the halves-layout MXFP8 with its blocks moved -- a fact of the block
definition, checked here against the independently pinned halves oracle."""
import numpy as np
import pytest

import oracle
from moe_gated_activation_b200.workloads import bf16_bits, random_case



def _stored_col(j, N, G, up):
    """Stored column of gate column j (up=False) or up column j (up=True),
    from the layout's description: block b = j // G holds gate columns
    [bG, bG + G) at [2bG, 2bG + G) and their up columns right after."""
    b, k = divmod(j, G)
    return 2 * b * G + (G if up else 0) + k


def _interleave_loops(halves, N, G):
    """[gate | up] -> interleaved, one element at a time."""
    M = halves.shape[0]
    out = np.zeros((M, 2 * N), halves.dtype)
    for j in range(N):
        out[:, _stored_col(j, N, G, False)] = halves[:, j]
        out[:, _stored_col(j, N, G, True)] = halves[:, N + j]
    return out


def _move_row_blocks(a, N, G, per):
    """Columns of a [M, 2N / per] per-block array (per = 32: scales; per = 1:
    elements) of the halves layout, moved to the interleaved order."""
    Wb = 2 * N // per
    out = np.zeros_like(a)
    for jb in range(Wb // 2):
        j = jb * per
        out[:, _stored_col(j, N, G, False) // per] = a[:, jb]
        out[:, _stored_col(j, N, G, True) // per] = a[:, Wb // 2 + jb]
    return out


def test_hand_built_row():
    N, G = 64, 32
    gate = np.arange(100, 164, dtype=np.uint16)
    up = np.arange(500, 564, dtype=np.uint16)
    row = np.concatenate([gate[0:32], up[0:32], gate[32:64], up[32:64]])[None, :]
    halves = oracle.glu_halves(row, N, G)
    assert np.array_equal(halves[0, :N], gate) and np.array_equal(halves[0, N:], up)
    assert np.array_equal(oracle.glu_interleave(halves, N, G), row)


@pytest.mark.parametrize("N,G", [(256, 32), (256, 64), (256, 128), (384, 128), (96, 32)])
def test_layout_matches_loops(N, G):
    rng = np.random.default_rng(N + G)
    halves = rng.integers(0, 65535, size=(5, 2 * N), dtype=np.uint16)
    ilv = _interleave_loops(halves, N, G)
    assert np.array_equal(oracle.glu_interleave(halves, N, G), ilv)
    assert np.array_equal(oracle.glu_halves(ilv, N, G), halves)


def test_g_equal_n_is_halves():
    N = 128
    halves = np.random.default_rng(3).integers(0, 65535, size=(4, 2 * N), dtype=np.uint16)
    assert np.array_equal(oracle.glu_halves(halves, N, N), halves)
    assert np.array_equal(oracle.glu_interleave(halves, N, N), halves)


def _case(M, N, seed):
    c = random_case(M, N, seed, std=2.0)
    return bf16_bits(c["x"]), c["s"].numpy(), bf16_bits(c["dy"])


@pytest.mark.parametrize("act", ["swiglu", "clamped"])
@pytest.mark.parametrize("G", [32, 64, 128])
def test_forward_is_the_halves_forward(act, G):
    M, N = 70, 256
    xh, s, _ = _case(M, N, G)
    xi = _interleave_loops(xh, N, G)
    got = oracle.interleaved_fwd(xi, s, N, 3, G, act=act)
    ref = oracle.clamped_fwd(xh, s, N, 3) if act == "clamped" else oracle.act_fwd(xh, s, N, 3)
    for k in ("row_codes", "row_scales", "col_codes", "col_scales"):
        assert np.array_equal(got[k], ref[k]), k


@pytest.mark.parametrize("act", ["swiglu", "clamped"])
@pytest.mark.parametrize("G", [32, 64, 128])
def test_backward_moves_blocks(act, G):
    M, N = 70, 256
    xh, s, dy = _case(M, N, 7 * G)
    xi = _interleave_loops(xh, N, G)
    got = oracle.interleaved_bwd(dy, xi, s, N, 3, G, act=act)
    ref = (oracle.clamped_bwd(dy, xh, s, N, 3) if act == "clamped"
           else oracle.act_bwd(dy, xh, s, N, 3))
    assert np.array_equal(got["dscale"], ref["dscale"])
    assert np.array_equal(got["dx"], _move_row_blocks(ref["dx"], N, G, 1))
    assert np.array_equal(got["row_codes"], _move_row_blocks(ref["row_codes"], N, G, 1))
    assert np.array_equal(got["col_codes"], _move_row_blocks(ref["col_codes"], N, G, 1))
    assert np.array_equal(got["col_scales"], _move_row_blocks(ref["col_scales"], N, G, 1))
    assert np.array_equal(got["row_scales"], _move_row_blocks(ref["row_scales"], N, G, 32))


def test_grouped_backward_moves_blocks():
    N, G = 128, 32
    m = np.array([40, 0, 33, 64, 7], np.int64)
    M = int(m.sum())
    xh, s, dy = _case(M, N, 11)
    xi = _interleave_loops(xh, N, G)
    _, ro, cb = oracle.splits_to_offsets(m, M)
    got = oracle.interleaved_bwd(dy, xi, s, N, 3, G, row_offs=ro, colblk_offs=cb)
    ref = oracle.grouped_act_bwd(dy, xh, s, N, 3, ro, cb)
    assert np.array_equal(got["dx"], _move_row_blocks(ref["dx"], N, G, 1))
    assert np.array_equal(got["row_codes"], _move_row_blocks(ref["row_codes"], N, G, 1))
    assert np.array_equal(got["col_codes"], _move_row_blocks(ref["col_codes"], N, G, 1))
    assert np.array_equal(got["col_scales"], _move_row_blocks(ref["col_scales"], N, G, 1))
    assert np.array_equal(got["row_scales"], _move_row_blocks(ref["row_scales"], N, G, 32))
    gotf = oracle.interleaved_fwd(xi, s, N, 3, G, row_offs=ro, colblk_offs=cb)
    reff = oracle.grouped_act_fwd(xh, s, N, 3, ro, cb)
    for k in ("row_codes", "row_scales", "col_codes", "col_scales"):
        assert np.array_equal(gotf[k], reff[k]), k

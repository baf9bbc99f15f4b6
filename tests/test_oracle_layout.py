"""Pins of the oracle's GEMM-ready scale layout (128 x 4 tiles of E8M0
scales, 512 bytes each, element (r, c) of a tile at (r % 32) * 16 +
(r / 32) * 4 + c).

The layout is checked against (a) positions worked out by hand from that
definition, (b) an independent formulation as a chain of tensor reshapes and
transposes, and (c) for the colwise scales of a grouped tensor, a per-expert
numpy transpose followed by (b)."""
import numpy as np
import pytest
import torch

import oracle


def _by_reshapes(S):
    """The tiled layout written as view / permute operations on a padded
    matrix: tiles [rt, 128, ct, 4] -> [rt, ct, 128, 4]; inside a tile rows
    r = 32 * r1 + r0 are reordered to (r0, r1, c)."""
    R, C = S.shape
    rt, ct = -(-R // 128), -(-C // 4)
    P = torch.zeros(rt * 128, ct * 4, dtype=torch.uint8)
    P[:R, :C] = torch.from_numpy(S)
    t = P.view(rt, 128, ct, 4).permute(0, 2, 1, 3)            # [rt, ct, 128, 4]
    t = t.reshape(rt * ct, 4, 32, 4).transpose(1, 2)          # [tile, r0, r1, c]
    return t.reshape(-1).numpy()


def test_hand_worked_positions():
    # a single 128 x 4 tile holding S[r, c] = (4 r + c) mod 251
    S = ((4 * np.arange(128)[:, None] + np.arange(4)[None, :]) % 251).astype(np.uint8)
    out = oracle.scales_gemm_layout(S)
    assert out.size == 512
    # (r, c) -> (r % 32) * 16 + (r // 32) * 4 + c, worked out by hand:
    cases = {(0, 0): 0, (0, 3): 3, (1, 0): 16, (31, 0): 496, (32, 0): 4, (33, 2): 22,
             (64, 1): 9, (96, 3): 15, (127, 3): 511, (100, 2): 4 * 16 + 3 * 4 + 2}
    for (r, c), off in cases.items():
        assert out[off] == S[r, c], (r, c, off)
    # the 16 bytes of tile row 0 are rows 0, 32, 64, 96, 4 columns each
    assert list(out[:16]) == [S[r, c] for r in (0, 32, 64, 96) for c in range(4)]


def test_tiles_follow_row_major_tile_order_and_padding_is_zero():
    R, C = 256, 6                       # 2 x 2 tiles, the second column of tiles half empty
    S = np.full((R, C), 7, np.uint8)
    out = oracle.scales_gemm_layout(S).reshape(4, 512)
    # tile (0, 1) holds columns 4, 5 (then two padding columns) of rows 0..127
    t01 = out[1].reshape(32, 4, 4)      # [r0, r1, c]
    assert (t01[:, :, :2] == 7).all() and (t01[:, :, 2:] == 0).all()
    assert (out[0] == 7).all() and (out[2] == 7).all()


@pytest.mark.parametrize("R,C", [(128, 4), (256, 12), (384, 224), (100, 5), (1, 1), (130, 7)])
def test_matches_the_reshape_formulation(R, C):
    g = np.random.default_rng(R * 31 + C)
    S = g.integers(0, 256, (R, C), dtype=np.uint8)
    assert np.array_equal(oracle.scales_gemm_layout(S), _by_reshapes(S))


def test_it_is_a_permutation_on_whole_tiles():
    R, C = 256, 8
    S = np.arange(R * C, dtype=np.int64)
    lo = (S % 256).astype(np.uint8).reshape(R, C)
    hi = (S // 256).astype(np.uint8).reshape(R, C)
    idx = (oracle.scales_gemm_layout(lo).astype(np.int64)
           + 256 * oracle.scales_gemm_layout(hi).astype(np.int64))
    assert np.array_equal(np.sort(idx), np.arange(R * C))


def test_colwise_scales_of_experts_are_transposed_per_expert():
    W = 256
    m = np.array([128, 0, 256, 128], np.int64)
    M = int(m.sum())
    st, ro, cb = oracle.splits_to_offsets(m, M)
    assert st == 0
    g = np.random.default_rng(5)
    cs = g.integers(0, 256, (int(cb[-1]), W), dtype=np.uint8)
    out = oracle.col_scales_gemm_layout(cs, W, ro, cb)
    parts = []
    for e in range(len(m)):
        blk = cs[cb[e]:cb[e + 1]]                     # [m_e / 32, W]
        if blk.size:
            parts.append(_by_reshapes(np.ascontiguousarray(blk.T)))
    assert np.array_equal(out, np.concatenate(parts))
    assert out.size == M * W // 32


def test_colwise_layout_rejects_unaligned_groups():
    m = np.array([96, 160], np.int64)
    _, ro, cb = oracle.splits_to_offsets(m, 256)
    with pytest.raises(ValueError):
        oracle.col_scales_gemm_layout(np.zeros((int(cb[-1]), 128), np.uint8), 128, ro, cb)


def test_row_scales_of_aligned_experts_equal_the_dense_layout():
    """With every group a multiple of 128 rows, laying out each expert's row
    scales separately and concatenating gives the dense layout."""
    W32 = 12
    m = np.array([256, 128, 0, 384], np.int64)
    g = np.random.default_rng(9)
    S = g.integers(0, 256, (int(m.sum()), W32), dtype=np.uint8)
    ro = np.concatenate([[0], np.cumsum(m)])
    parts = [oracle.scales_gemm_layout(S[ro[e]:ro[e + 1]]) for e in range(len(m)) if m[e]]
    assert np.array_equal(np.concatenate(parts), oracle.scales_gemm_layout(S))

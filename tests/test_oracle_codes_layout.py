"""Pins of the oracle's tiled operand layout of weight codes
(oracle.codes_gemm_layout): tiles of 128 rows x 128 bytes of k, row blocks
then k blocks in order, row r of a tile at byte 128 r with its 16-byte chunk
c at chunk position c ^ (r mod 8) -- the 128-byte-swizzled K-major layout the
tensor cores read an operand tile in.

Checked against (a) positions worked out by hand from that definition,
(b) an independent formulation that gathers each destination chunk from its
source (the definition scatters source chunks), and (c) permutation and
round-trip properties."""
import numpy as np
import pytest
import torch

import oracle


def _pattern(R, K):
    r = np.arange(R)[:, None]
    k = np.arange(K)[None, :]
    return ((7 * r + 3 * k) % 251).astype(np.uint8)


def test_hand_worked_positions():
    W = _pattern(256, 256)
    t = oracle.codes_gemm_layout(W)
    # (row, k) -> byte offset, worked out by hand:
    #   (1, 0): tile 0, row 1, chunk 0 at position 0 ^ 1 = 1      -> 128 + 16
    #   (9, 37): tile 0, row 9, chunk 2 at 2 ^ 1 = 3, byte 5       -> 1152 + 48 + 5
    #   (130, 200): tile 1 * 2 + 1 = 3, row 2, chunk 4 at 4 ^ 2 = 6, byte 8
    #                                                             -> 49152 + 256 + 96 + 8
    #   (127, 127): tile 0, row 127, chunk 7 at 7 ^ 7 = 0, byte 15 -> 16256 + 15
    #   (5, 130): tile 1, row 5, chunk 0 at 0 ^ 5 = 5, byte 2      -> 16384 + 640 + 80 + 2
    for (r, k), off in {(0, 0): 0, (1, 0): 144, (9, 37): 1205, (130, 200): 49512,
                        (127, 127): 16271, (5, 130): 17106}.items():
        assert t[off] == W[r, k], (r, k, off)


@pytest.mark.parametrize("R,K", [(128, 128), (256, 384), (384, 768)])
def test_matches_a_gather_formulation(R, K):
    W = np.random.default_rng(R + K).integers(0, 256, (R, K), dtype=np.uint8)
    src = torch.from_numpy(W).view(R // 128, 128, K // 128, 8, 16).permute(0, 2, 1, 3, 4)
    r = torch.arange(128).view(128, 1)
    p = torch.arange(8).view(1, 8)
    dst = src[:, :, r, p ^ (r % 8), :]        # destination chunk p takes source chunk p ^ (r % 8)
    assert np.array_equal(oracle.codes_gemm_layout(W), dst.reshape(-1).numpy())


def test_it_is_a_permutation_and_rows_stay_in_their_tile_row():
    R, K = 256, 384
    idx = np.arange(R * K).reshape(R, K)
    t = oracle.codes_gemm_layout(idx)
    assert np.array_equal(np.sort(t), np.arange(R * K))
    tiles = t.reshape(R // 128, K // 128, 128, 128)
    for rb in range(R // 128):
        for kb in range(K // 128):
            for r in (0, 5, 77, 127):
                row = tiles[rb, kb, r]
                want = idx[128 * rb + r, 128 * kb:128 * kb + 128]
                assert np.array_equal(np.sort(row), want)
                # undoing the swizzle of the row's chunks gives the row back
                chunks = row.reshape(8, 16)
                assert np.array_equal(chunks[np.arange(8) ^ (r % 8)].reshape(-1), want)


def test_rejects_shapes_that_are_not_whole_tiles():
    with pytest.raises(ValueError):
        oracle.codes_gemm_layout(np.zeros((100, 128), np.uint8))

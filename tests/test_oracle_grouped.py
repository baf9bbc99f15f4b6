"""Pins of the oracle's grouped path: splits -> offsets, and several expert
tensors stored contiguously and addressed by per-expert offsets.

Sources: TransformerEngine PR #3238 (Greptile summary: splits_to_offsets_multi
computes all offset arrays up front; sequence diagram: the grouped activation
consumes per-expert offsets and returns quantized grouped storage);
TransformerEngine PR #2600 "[PyTorch] GroupedTensor integration" (several
tensors of different shapes in one contiguous buffer, addressed by offsets);
TransformerEngine PR #3224 (Greptile summary: an MXFP8 scale-address bug for
uniform-group layouts -- hence the uniform-split case below).
"""
import numpy as np
import pytest

import naive_ref
import oracle
from moe_gated_activation_b200.workloads import bf16_bits, random_case

BOTH = oracle.ROWWISE | oracle.COLWISE


def test_splits_to_offsets_hand_cases():
    st, ro, co = oracle.splits_to_offsets(np.array([3, 0, 5], np.int64), 8)
    assert st == 0
    assert ro.tolist() == [0, 3, 3, 8]
    assert co.tolist() == [0, 1, 1, 2]       # ceil(3/32)=1, ceil(0/32)=0, ceil(5/32)=1
    st, ro, co = oracle.splits_to_offsets(np.array([64, 32, 0, 96], np.int64), 192)
    assert ro.tolist() == [0, 64, 96, 96, 192] and co.tolist() == [0, 2, 3, 3, 6]
    st, ro, co = oracle.splits_to_offsets(np.array([], np.int64), 0)
    assert st == 0 and ro.tolist() == [0] and co.tolist() == [0]


def test_splits_to_offsets_errors():
    assert oracle.splits_to_offsets(np.array([4, -1, 5], np.int64), 8)[0] == 1
    assert oracle.splits_to_offsets(np.array([4, 5], np.int64), 8)[0] == 2
    assert oracle.splits_to_offsets(np.array([4, 3], np.int64), 8)[0] == 2
    big = np.array([2 ** 62, 2 ** 62, 2 ** 62], np.int64)   # would overflow a plain sum
    assert oracle.splits_to_offsets(big, 8)[0] == 2


def _per_expert_dense(xb, s, N, splits, dirs, act=oracle.SWIGLU):
    outs = []
    r = 0
    for m in splits:
        outs.append(oracle.act_fwd(xb[r:r + m], s[r:r + m], N, dirs, act=act))
        r += m
    return outs


@pytest.mark.parametrize("splits", [[64, 0, 96, 32, 0, 64],       # aligned, with empties
                                    [32] * 8,                     # uniform (M/E each)
                                    [5, 40, 0, 33, 1, 49]])      # ragged
def test_grouped_forward_is_per_expert_tensors_in_one_buffer(splits):
    N = 64
    M = sum(splits)
    c = random_case(M, N, 31)
    xb, s = bf16_bits(c["x"]), c["s"].numpy()
    st, ro, co = oracle.splits_to_offsets(np.array(splits, np.int64), M)
    got = oracle.grouped_act_fwd(xb, s, N, BOTH, ro, co)
    per = _per_expert_dense(xb, s, N, splits, BOTH)
    # expected buffer: each expert's arrays placed at its offsets, no gaps
    exp_rq = np.concatenate([p["row_codes"] for p in per])
    exp_rs = np.concatenate([p["row_scales"] for p in per])
    exp_cq = np.concatenate([p["col_codes"] for p in per])
    exp_cs = np.concatenate([p["col_scales"] for p in per])
    assert np.array_equal(got["row_codes"], exp_rq)
    assert np.array_equal(got["row_scales"], exp_rs)
    assert np.array_equal(got["col_codes"], exp_cq)
    assert got["col_scales"].shape[0] == sum((m + 31) // 32 for m in splits)
    assert np.array_equal(got["col_scales"], exp_cs)


def test_grouped_equals_dense_when_splits_are_32_aligned():
    N = 96
    splits = [96, 32, 0, 128, 0, 64]
    M = sum(splits)
    c = random_case(M, N, 41)
    xb, s, dyb = bf16_bits(c["x"]), c["s"].numpy(), bf16_bits(c["dy"])
    st, ro, co = oracle.splits_to_offsets(np.array(splits, np.int64), M)
    g = oracle.grouped_act_fwd(xb, s, N, BOTH, ro, co)
    d = oracle.act_fwd(xb, s, N, BOTH)
    for k in g:
        assert np.array_equal(g[k], d[k]), k
    gb = oracle.grouped_act_bwd(dyb, xb, s, N, BOTH, ro, co)
    db = oracle.act_bwd(dyb, xb, s, N, BOTH)
    for k in gb:
        assert np.array_equal(gb[k], db[k]), k


def test_ragged_grouped_against_naive_per_expert_blocks():
    N = 32
    splits = [7, 0, 33, 2]
    M = sum(splits)
    c = random_case(M, N, 51)
    xb, s = bf16_bits(c["x"]), c["s"].numpy()
    st, ro, co = oracle.splits_to_offsets(np.array(splits, np.int64), M)
    got = oracle.grouped_act_fwd(xb, s, N, oracle.COLWISE, ro, co)
    y = naive_ref.fwd_values([list(map(int, r)) for r in xb], [float(v) for v in s], N)
    r = 0
    cs_rows = []
    cq_rows = []
    for m in splits:
        if m:
            q = naive_ref.mxfp8(y[r:r + m], oracle.COLWISE)
            cs_rows += q["col_scales"]
            cq_rows += q["col_codes"]
        r += m
    assert np.array_equal(got["col_scales"], np.array(cs_rows, np.uint8))
    assert np.array_equal(got["col_codes"], np.array(cq_rows, np.uint8))

"""GPU parity of the fused activation -> MXFP8 -> FC2 GEMM (tcgen05) against
the oracle (oracle.grouped_fc2).

TE PR #3238 (Greptile summary, sequence diagram): the grouped scaled
activation's quantized grouped tensor feeds the grouped linear after it.  The
kernel keeps that quantized activation on chip; the oracle builds it with the
pinned forward and multiplies exact values in binary64.

Tolerance (fp32 accumulation on the tensor cores, then one bf16 rounding):
|out - ref| <= 2^-8 |ref| + 2^-13 sum_k |a_k w_k|.  The first term covers the
bf16 rounding (half an ulp is 2^-9 relative) of a sum carrying its own fp32
error, the second an fp32 sum of up to 1024 products in any order (1024
roundings of 2^-24 relative each is 2^-14 of the sum of magnitudes).  A
wrong scale, a dropped K block, a transposed operand or a row of the wrong
expert is off by far more.  Where the weight is an exact identity the output
must equal the dequantized activation exactly (one product per output, exact
in fp32 and bf16).
"""
import numpy as np
import pytest
import torch

import oracle
import moe_gated_activation_b200 as mg
from moe_gated_activation_b200.workloads import (bf16_bits, fc2_weights, make_inputs,
                                                 random_case)

pytestmark = pytest.mark.gpu


def _bound(xb, s, N, row_offs, wc, ws, staged=False, rows=None):
    """sum_k |a_k w_k| per output element (binary64)."""
    a = oracle.act_fwd(xb, s, N, oracle.ROWWISE, staged=staged)
    av = np.abs(oracle.mxfp8_dequantize_rows(a["row_codes"], a["row_scales"]))
    out = np.zeros((av.shape[0], wc.shape[1]))
    ro = np.asarray(row_offs)
    for e in range(wc.shape[0]):
        r0, r1 = int(ro[e]), int(ro[e + 1])
        if r1 > r0:
            wv = np.abs(oracle.mxfp8_dequantize_rows(wc[e], ws[e]))
            out[r0:r1] = av[r0:r1] @ wv.T
    return out


def _check(got, ref, bound, what):
    g = got.float().cpu().numpy().astype(np.float64)
    assert g.shape == ref.shape, (what, g.shape, ref.shape)
    err = np.abs(g - ref)
    lim = 2.0 ** -8 * np.abs(ref) + 2.0 ** -13 * bound
    bad = err > lim
    if bad.any():
        i, h = np.argwhere(bad)[0]
        with np.errstate(divide="ignore", invalid="ignore"):
            ratio = np.where(ref != 0, g / ref, np.nan)
        rows_bad = np.unique(np.argwhere(bad)[:, 0])
        cols_bad = np.unique(np.argwhere(bad)[:, 1])
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} outputs outside the bound; first "
            f"({i}, {h}): got {g[i, h]!r} ref {ref[i, h]!r} bound {lim[i, h]!r}; "
            f"bad rows {rows_bad[:16].tolist()} ({rows_bad.size}), bad cols "
            f"{cols_bad[:16].tolist()} ({cols_bad.size}); median got/ref "
            f"{np.nanmedian(ratio)!r}")
    return float((err / np.maximum(lim, 1e-300)).max())


def _tiled(ws):
    """Row-major weight scales [E, H, N/32] -> the kernel's GEMM-ready tiled
    layout per expert (the oracle's pinned layout function)."""
    ws = np.asarray(ws)
    return torch.from_numpy(np.stack([oracle.scales_gemm_layout(w).reshape(w.shape)
                                      for w in ws]))


_PERM = {}


def _tiled_codes(wc):
    """Row-major weight codes [E, H, N] (torch, any device) -> the kernel's
    tiled operand layout per expert: the oracle's pinned layout function,
    applied as the permutation it gives an index matrix."""
    E, H, N = wc.shape
    if (H, N) not in _PERM:
        _PERM[(H, N)] = torch.from_numpy(
            oracle.codes_gemm_layout(np.arange(H * N, dtype=np.int64).reshape(H, N)))
    perm = _PERM[(H, N)].to(wc.device)
    return wc.reshape(E, H * N)[:, perm].reshape(E, H, N).contiguous()


def _run(case, N, splits, wc, ws, dev, staged=False):
    m = torch.tensor(splits, dtype=torch.int64)
    M = int(m.sum())
    ro, cb, st = mg.splits_to_offsets(m.to(dev), M)
    x, s = case["x"].to(dev), case["s"].to(dev)
    out, st2 = mg.grouped_scaled_swiglu_mxfp8_fc2(x, s, ro, _tiled_codes(wc).to(dev),
                                                  _tiled(ws).to(dev), staged_rounding=staged)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and int(st2.item()) == 0
    _, oro, _ = oracle.splits_to_offsets(m.numpy(), M)
    return out, oro


def _identity(E, N, scale_of=lambda e: 127):
    eye = np.where(np.eye(N, dtype=bool), 0x38, 0).astype(np.uint8)   # 1.0 on the diagonal
    wc = np.stack([eye] * E)
    ws = np.stack([np.full((N, N // 32), scale_of(e), np.uint8) for e in range(E)])
    return torch.from_numpy(wc), torch.from_numpy(ws)


def test_identity_weight_returns_the_dequantized_activation(cuda_device):
    N, M = 256, 256
    case = random_case(M, N, 31, std=2.0)
    wc, ws = _identity(1, N)
    out, oro = _run(case, N, [M], wc, ws, cuda_device)
    ref = oracle.grouped_fc2(bf16_bits(case["x"]), case["s"].numpy(), N, oro, wc.numpy(),
                             ws.numpy())
    assert np.array_equal(out.float().cpu().numpy().astype(np.float64), ref)


def test_identity_weight_with_gates_at_the_ends_of_the_sigmoid_table(cuda_device):
    """Gates where sigma saturates, at the largest tabulated magnitude (127.5)
    and past it (clamped to it: the same fp32 sigma, 1 or +0), and where it
    rounds to 1/2; every output equals the dequantized activation exactly."""
    N, M = 256, 256
    case = random_case(M, N, 33, std=2.0)
    x = case["x"]
    special = torch.tensor([127.5, 128.0, 129.0, 1000.0, 30000.0, 17.25, 17.5, 88.0, 103.5,
                            104.0, 2.0 ** -25, 2.0 ** -24, 1e-8, 0.0, 126.0, 127.0])
    special = torch.cat([special, -special]).to(torch.bfloat16)
    g = torch.Generator().manual_seed(34)
    pos = torch.randperm(M * N, generator=g)[: M * N // 8]
    gate = x[:, :N].reshape(-1).clone()
    gate[pos] = special[torch.randint(0, special.numel(), (pos.numel(),), generator=g)]
    x[:, :N] = gate.reshape(M, N)
    wc, ws = _identity(1, N)
    out, oro = _run(case, N, [M], wc, ws, cuda_device)
    ref = oracle.grouped_fc2(bf16_bits(case["x"]), case["s"].numpy(), N, oro, wc.numpy(),
                             ws.numpy())
    assert np.isfinite(ref).all()
    assert np.array_equal(out.float().cpu().numpy().astype(np.float64), ref)


def test_each_expert_uses_its_own_weight_and_rows(cuda_device):
    # ragged and empty experts; expert e's weight is 2^(e - 2) times the identity
    N = 384
    splits = [0, 200, 56, 0, 129, 1]
    M = sum(splits)
    case = random_case(M, N, 32)
    wc, ws = _identity(len(splits), N, lambda e: 125 + e)
    out, oro = _run(case, N, splits, wc, ws, cuda_device)
    ref = oracle.grouped_fc2(bf16_bits(case["x"]), case["s"].numpy(), N, oro, wc.numpy(),
                             ws.numpy())
    assert np.array_equal(out.float().cpu().numpy().astype(np.float64), ref)


@pytest.mark.parametrize("N,H,splits,staged", [
    (128, 128, [128], False),
    (256, 384, [128, 0, 256], False),
    (384, 256, [37, 300, 0, 91], False),          # ragged: partial 128-row blocks
    (768, 512, [256, 128, 0, 384], False),         # the Qwen3-MoE width
    (768, 256, [200, 56], True),                   # staged rounding
    (128, 128, [1], False),                        # a single row
    (256, 128, [0, 1, 0, 129], False),             # one-row and 129-row experts
    # fewer blocks than SMs: each block's output tiles split over several CTAs,
    # unevenly here (5 tiles in parts of 1, 2, 2 when 38 blocks meet 148 SMs)
    (256, 640, [1200, 0, 3536], False),
    # more blocks than SMs: whole blocks, then a split last wave
    (128, 256, [20403, 77], False),
    # a wide FC2 (32 output tiles) over three blocks: 148 / 3 = 49 parts
    # capped at one tile each
    (256, 4096, [300, 84], False),
    # many small experts (one partial block each, empty ones among them)
    (128, 256, [(7 * e) % 5 for e in range(300)], False),
])
def test_fc2_matches_the_oracle(cuda_device, N, H, splits, staged):
    M = sum(splits)
    E = len(splits)
    case = random_case(M, N, 40 + N + H, std=1.5)
    wc, ws = fc2_weights(E, H, N, 7 + N)
    out, oro = _run(case, N, splits, wc, ws, cuda_device, staged)
    xb, s = bf16_bits(case["x"]), case["s"].numpy()
    ref = oracle.grouped_fc2(xb, s, N, oro, wc.numpy(), ws.numpy(), staged=staged)
    bound = _bound(xb, s, N, oro, wc.numpy(), ws.numpy(), staged)
    _check(out, ref, bound, f"N={N} H={H} splits={splits}")


def test_fc2_reads_a_strided_input_and_writes_into_a_wider_output(cuda_device):
    """X as a column slice of a wider tensor (row stride 2N + 64) and `out` as
    the first H columns of a wider buffer: the same bits as the contiguous
    call, the extra output columns untouched, the input unchanged."""
    dev = cuda_device
    N, H, splits = 256, 384, [200, 0, 184]
    M, E = sum(splits), len(splits)
    case = random_case(M, N, 43, std=1.5)
    wc, ws = fc2_weights(E, H, N, 44)
    wc, ws = _tiled_codes(wc).to(dev), _tiled(ws).to(dev)
    ro, _, st = mg.splits_to_offsets(torch.tensor(splits, dtype=torch.int64, device=dev), M)
    x, s = case["x"].to(dev), case["s"].to(dev)
    ref, st0 = mg.grouped_scaled_swiglu_mxfp8_fc2(x, s, ro, wc, ws)
    wide = torch.zeros(M, 2 * N + 64, dtype=torch.bfloat16, device=dev)
    wide[:, 32:32 + 2 * N] = x
    xv = wide[:, 32:32 + 2 * N]
    before = wide.clone()
    big = torch.full((M, H + 64), 7.0, dtype=torch.bfloat16, device=dev)
    out, st1 = mg.grouped_scaled_swiglu_mxfp8_fc2(xv, s, ro, wc, ws, out=big[:, :H])
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and int(st0.item()) == 0 and int(st1.item()) == 0
    assert xv.stride(0) == 2 * N + 64 and out.stride(0) == H + 64
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    assert bool((big[:, H:] == 7.0).all())
    assert torch.equal(wide.view(torch.int16), before.view(torch.int16))


def test_fc2_writes_nothing_for_bad_offsets_or_a_set_noop_flag(cuda_device):
    N, H, M = 128, 128, 256
    case = random_case(M, N, 41)
    wc, ws = fc2_weights(2, H, N, 8)
    wc, ws = _tiled_codes(wc), _tiled(ws)
    dev = cuda_device
    x, s = case["x"].to(dev), case["s"].to(dev)
    bad = torch.tensor([0, 200, 100], dtype=torch.int64, device=dev)   # ends past M
    out = torch.full((M, H), 3.0, dtype=torch.bfloat16, device=dev)
    _, st = mg.grouped_scaled_swiglu_mxfp8_fc2(x, s, bad, wc.to(dev), ws.to(dev), out=out)
    torch.cuda.synchronize()
    assert int(st.item()) == 3
    assert bool((out == 3.0).all())
    good = torch.tensor([0, 128, 256], dtype=torch.int64, device=dev)
    flag = torch.ones(1, dtype=torch.int32, device=dev)
    mg.grouped_scaled_swiglu_mxfp8_fc2(x, s, good, wc.to(dev), ws.to(dev), out=out,
                                       noop_flag=flag)
    torch.cuda.synchronize()
    assert bool((out == 3.0).all())
    flag.zero_()
    mg.grouped_scaled_swiglu_mxfp8_fc2(x, s, good, wc.to(dev), ws.to(dev), out=out,
                                       noop_flag=flag)
    torch.cuda.synchronize()
    assert not bool((out == 3.0).all())


def test_fc2_at_the_qwen3_moe_workload_sampled_rows(cuda_device):
    """The c3 workload (65536 routed rows, 128 experts with empty ones, N =
    768) into an FC2 of width 2048 (the model's hidden size), launched as the
    benchmark launches it; sampled rows against the oracle row by row."""
    dev = cuda_device
    inp = make_inputs("c3", device=dev)
    m = inp["m_splits"]
    M, N, H = 65536, 768, 2048
    E = int(m.numel())
    wc, ws = fc2_weights(E, H, N, 11, device=dev)
    ro, cb, st = mg.splits_to_offsets(m.to(dev), M)
    out, st2 = mg.grouped_scaled_swiglu_mxfp8_fc2(inp["x"], inp["s"], ro, _tiled_codes(wc),
                                                  _tiled(ws.cpu()).to(dev))
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and int(st2.item()) == 0
    ro_h = ro.cpu().numpy()
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([rng.integers(0, M, 48), ro_h[1:-1][:16],
                                     np.maximum(ro_h[1:] - 1, 0)[:16]]))
    rows = rows[rows < M]
    xb = bf16_bits(inp["x"][torch.from_numpy(rows).to(dev)])
    sv = inp["s"][torch.from_numpy(rows).to(dev)].cpu().numpy()
    a = oracle.act_fwd(xb, sv, N, oracle.ROWWISE)
    av = oracle.mxfp8_dequantize_rows(a["row_codes"], a["row_scales"])
    experts = np.searchsorted(ro_h, rows, side="right") - 1
    wc_h, ws_h = wc.cpu().numpy(), ws.cpu().numpy()
    got = out[torch.from_numpy(rows).to(dev)]
    ref = np.zeros((rows.size, H))
    bound = np.zeros((rows.size, H))
    for k, e in enumerate(experts):
        wv = oracle.mxfp8_dequantize_rows(wc_h[e], ws_h[e])
        ref[k] = wv @ av[k]
        bound[k] = np.abs(wv) @ np.abs(av[k])
    _check(got, ref, bound, "c3 sampled rows")

"""The GEMM-ready scale layout read by a block-scaled tensor-core GEMM.

The consumer of the quantized activation is an MXFP8 GEMM (TE PR #3238: the
grouped GEMM after the activation).  Here a library MXFP8 GEMM
(torch._scaled_mm with E8M0 scales, cuBLASLt) multiplies the codes and
GEMM-layout scales this library wrote -- rowwise data as the K-major A
operand (K = N), and each group's colwise data transposed (K = the group's
rows) -- by a weight operand the oracle quantized.  The product must equal
the fp64 product of the oracle's dequantized values within fp32-accumulation
and bf16-output rounding: a layout the GEMM read differently would put
scales on the wrong blocks and miss by orders of magnitude.  No expected
value comes from the GPU path (the A operand's reference values are the
oracle's forward outputs, which the parity tests show equal ours bitwise)."""
import numpy as np
import pytest
import torch

import oracle
import moe_gated_activation_b200 as mg
from moe_gated_activation_b200.workloads import bf16_bits, random_case

pytestmark = pytest.mark.gpu

E4M3 = np.array([oracle.e4m3_decode(c) for c in range(256)], np.float64)


def _deq_rows(codes, scales):
    """Rowwise MXFP8 [R, K] (scales [R, K/32]) -> fp64 values."""
    return E4M3[codes] * np.exp2(np.repeat(scales.astype(np.float64) - 127.0, 32, axis=1))


def _weights(H, K, seed):
    """An [H, K] operand quantized rowwise (along K) by the oracle."""
    g = torch.Generator().manual_seed(seed)
    y = torch.randn(H, K, generator=g).numpy().astype(np.float32)
    q = oracle.mxfp8_quantize(y, oracle.ROWWISE)
    return q["row_codes"], q["row_scales"]


def _scaled_mm(a_codes, a_scales_flat, bt_codes, bt_scales, dev):
    """A [R, K] (K-major codes) x B^T ([H, K] K-major, scales [H, K/32])."""
    a = torch.from_numpy(np.ascontiguousarray(a_codes)).to(dev).view(torch.float8_e4m3fn) \
        if isinstance(a_codes, np.ndarray) else a_codes
    bt = torch.from_numpy(bt_codes).to(dev).view(torch.float8_e4m3fn)
    sb = torch.from_numpy(oracle.scales_gemm_layout(bt_scales)).to(dev)
    try:
        c = torch._scaled_mm(a, bt.t(), a_scales_flat.view(torch.float8_e8m0fnu),
                             sb.view(torch.float8_e8m0fnu), out_dtype=torch.bfloat16)
    except (RuntimeError, NotImplementedError) as e:   # no MXFP8 GEMM in this torch / cuBLAS
        pytest.skip(f"block-scaled torch._scaled_mm unavailable: {e}")
    return c.float().cpu().numpy().astype(np.float64)


def _check(got, a_deq, b_deq, what):
    ref = a_deq @ b_deq.T
    bound = np.abs(a_deq) @ np.abs(b_deq).T
    K = a_deq.shape[1]
    tol = 2.0 * K * 2.0 ** -24 * bound + 2.0 ** -8 * np.abs(ref) + 1e-30   # fp32 sums, bf16 out
    bad = np.abs(got - ref) > tol
    assert not bad.any(), f"{what}: {int(bad.sum())} outputs off, worst {np.abs(got - ref)[bad].max()}"


def test_rowwise_operand(cuda_device):
    M, N, H = 256, 512, 384
    c = random_case(M, N, 5, std=2.0)
    xb, s = bf16_bits(c["x"]), c["s"].numpy()
    got = mg.scaled_swiglu_mxfp8_fwd(c["x"].to(cuda_device), c["s"].to(cuda_device),
                                     colwise=False, gemm_scales=True)
    ref = oracle.act_fwd(xb, s, N, oracle.ROWWISE)
    bt_codes, bt_scales = _weights(H, N, 6)
    out = _scaled_mm(got.row_codes, got.row_scales.reshape(-1), bt_codes, bt_scales, cuda_device)
    _check(out, _deq_rows(ref["row_codes"], ref["row_scales"]),
           _deq_rows(bt_codes, bt_scales), "rowwise forward")


def test_backward_rowwise_operand(cuda_device):
    """The gradient's MXFP8 (width 2N) as the A operand of the dgrad GEMM."""
    M, N, H = 128, 256, 256
    c = random_case(M, N, 9, std=2.0)
    xb, s, dyb = bf16_bits(c["x"]), c["s"].numpy(), bf16_bits(c["dy"])
    d = cuda_device
    got = mg.scaled_swiglu_mxfp8_bwd(c["dy"].to(d), c["x"].to(d), c["s"].to(d), colwise=False,
                                     gemm_scales=True)
    ref = oracle.act_bwd(dyb, xb, s, N, oracle.ROWWISE)
    bt_codes, bt_scales = _weights(H, 2 * N, 10)
    out = _scaled_mm(got.mx.row_codes, got.mx.row_scales.reshape(-1), bt_codes, bt_scales, d)
    _check(out, _deq_rows(ref["row_codes"], ref["row_scales"]),
           _deq_rows(bt_codes, bt_scales), "rowwise backward")


def test_colwise_operand_per_group(cuda_device):
    """Each group's colwise codes, transposed, as the K-major A operand of a
    GEMM over the group's rows (K = m_e), with the group's GEMM-layout
    colwise scales."""
    N, H = 256, 128
    m = np.array([128, 256, 0, 128], np.int64)
    M = int(m.sum())
    c = random_case(M, N, 13, std=2.0)
    xb, s = bf16_bits(c["x"]), c["s"].numpy()
    d = cuda_device
    gro, gcb, _ = mg.splits_to_offsets(torch.from_numpy(m).to(d), M)
    _, ro, cb = oracle.splits_to_offsets(m, M)
    got, st = mg.grouped_scaled_swiglu_mxfp8_fwd(c["x"].to(d), c["s"].to(d), gro, gcb,
                                                 rowwise=False, col_scale_rows=int(cb[-1]),
                                                 gemm_scales=True)
    assert int(st.item()) == 0
    ref = oracle.grouped_act_fwd(xb, s, N, oracle.COLWISE, ro, cb)
    cs_flat = got.col_scales.reshape(-1)
    for e in range(len(m)):
        me = int(m[e])
        if me == 0:
            continue
        r0, r1 = int(ro[e]), int(ro[e + 1])
        a = got.col_codes[r0:r1].t().contiguous()                  # [N, m_e], K = m_e
        base = r0 // 32 * N
        sa = cs_flat[base:base + N * me // 32]
        bt_codes, bt_scales = _weights(H, me, 20 + e)
        out = _scaled_mm(a, sa, bt_codes, bt_scales, d)
        codes = ref["col_codes"][r0:r1].T                          # [N, m_e]
        sc = ref["col_scales"][int(cb[e]):int(cb[e + 1])].T       # [N, m_e / 32]
        _check(out, _deq_rows(codes, sc), _deq_rows(bt_codes, bt_scales), f"colwise group {e}")

"""Caller-owned output buffers (`out=`) and CUDA-graph replay into them
(TE PR #3238: an output= argument and a noop_flag so that graph-captured
quantization replays in place without pointer changes): results equal the
oracle's bitwise, the returned tensors are the caller's buffers, and a
captured graph replayed on new input contents writes the new results into
the same buffers."""
import numpy as np
import pytest
import torch

import oracle
import moe_gated_activation_b200 as mg
from moe_gated_activation_b200.workloads import bf16_bits, random_case
from parity import assert_dscale, bf16_u16, compare_mx, dscale_abs_bound

pytestmark = pytest.mark.gpu


def _mx_buffers(M, W, col_rows, dev, fp8_codes=True):
    code_t = torch.float8_e4m3fn if fp8_codes else torch.uint8
    return mg.MXFP8(torch.empty((M, W), dtype=torch.uint8, device=dev).view(code_t),
                    torch.empty((M, W), dtype=torch.uint8, device=dev),
                    torch.empty((M, W // 32), dtype=torch.uint8, device=dev),
                    torch.empty((col_rows, W), dtype=torch.uint8, device=dev))


def test_forward_and_backward_into_caller_buffers(cuda_device):
    M, N = 96, 384
    c = random_case(M, N, 31, std=2.0)
    xb, s, dyb = bf16_bits(c["x"]), c["s"].numpy(), bf16_bits(c["dy"])
    x, sg, dy = c["x"].to(cuda_device), c["s"].to(cuda_device), c["dy"].to(cuda_device)
    fo = _mx_buffers(M, N, (M + 31) // 32, cuda_device)
    got = mg.scaled_swiglu_mxfp8_fwd(x, sg, out=fo)
    bo = mg.Backward(_mx_buffers(M, 2 * N, (M + 31) // 32, cuda_device, fp8_codes=False),
                     torch.empty((M, 2 * N), dtype=torch.bfloat16, device=cuda_device),
                     torch.empty(M, dtype=torch.float32, device=cuda_device))
    gotb = mg.scaled_swiglu_mxfp8_bwd(dy, x, sg, out=bo)
    torch.cuda.synchronize()
    assert got.row_codes.data_ptr() == fo.row_codes.data_ptr()
    assert got.col_scales.data_ptr() == fo.col_scales.data_ptr()
    assert gotb.dx.data_ptr() == bo.dx.data_ptr()
    compare_mx(got, oracle.act_fwd(xb, s, N, 3), "fwd out=")
    ref = oracle.act_bwd(dyb, xb, s, N, 3)
    compare_mx(gotb.mx, ref, "bwd out=")
    assert np.array_equal(bf16_u16(gotb.dx), ref["dx"])
    assert_dscale(gotb.dscale, ref["dscale"], dscale_abs_bound(dyb, xb, s, N), "dscale")
    # a backward without dx: its out= holds no dx, and none is written
    nb = mg.scaled_swiglu_mxfp8_bwd(dy, x, sg, rowwise=False,
                                    out=mg.Backward(_mx_buffers(M, 2 * N, (M + 31) // 32,
                                                                cuda_device), None, None))
    torch.cuda.synchronize()
    assert nb.dx is None and nb.dscale is None
    compare_mx(nb.mx, oracle.act_bwd(dyb, xb, s, N, 2, want_dx=False, want_dscale=False),
               "bwd colwise only")


def test_graph_replay_into_the_same_buffers(cuda_device):
    N = 256
    m = np.array([64, 0, 96, 32], np.int64)
    M = int(m.sum())
    d = cuda_device
    mg.init()
    static = random_case(M, N, 1, std=2.0)
    x, sg, dy = (static[k].to(d) for k in ("x", "s", "dy"))
    md = torch.from_numpy(m).to(d)
    ro, cb, _ = mg.splits_to_offsets(md, M)
    S = M // 32 + len(m)
    fo = _mx_buffers(M, N, S, d)
    bo = mg.Backward(_mx_buffers(M, 2 * N, S, d), torch.empty((M, 2 * N), dtype=torch.bfloat16,
                                                              device=d),
                     torch.empty(M, dtype=torch.float32, device=d))
    st = torch.empty(1, dtype=torch.int32, device=d)
    ws = torch.empty(mg.bwd_workspace_bytes(M, N), dtype=torch.uint8, device=d)
    stream = torch.cuda.Stream(d)
    stream.wait_stream(torch.cuda.current_stream(d))
    with torch.cuda.stream(stream):     # one eager run on the capture stream first
        mg.grouped_scaled_swiglu_mxfp8_fwd(x, sg, ro, cb, status=st, out=fo)
        mg.grouped_scaled_swiglu_mxfp8_bwd(dy, x, sg, ro, cb, status=st, workspace=ws, out=bo)
    torch.cuda.current_stream(d).wait_stream(stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        mg.grouped_scaled_swiglu_mxfp8_fwd(x, sg, ro, cb, status=st, out=fo)
        mg.grouped_scaled_swiglu_mxfp8_bwd(dy, x, sg, ro, cb, status=st, workspace=ws, out=bo)
    ptrs = [t.data_ptr() for t in (*fo, *bo.mx, bo.dx, bo.dscale)]
    _, oro, ocb = oracle.splits_to_offsets(m, M)
    for seed in (2, 3):
        new = random_case(M, N, seed, std=2.0)
        x.copy_(new["x"].to(d))
        sg.copy_(new["s"].to(d))
        dy.copy_(new["dy"].to(d))
        g.replay()
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert [t.data_ptr() for t in (*fo, *bo.mx, bo.dx, bo.dscale)] == ptrs
        xb, s, dyb = bf16_bits(new["x"]), new["s"].numpy(), bf16_bits(new["dy"])
        view = mg.MXFP8(fo.row_codes, fo.col_codes, fo.row_scales, fo.col_scales[:int(ocb[-1])])
        compare_mx(view, oracle.grouped_act_fwd(xb, s, N, 3, oro, ocb), f"replay {seed} fwd")
        ref = oracle.grouped_act_bwd(dyb, xb, s, N, 3, oro, ocb)
        bview = mg.MXFP8(bo.mx.row_codes, bo.mx.col_codes, bo.mx.row_scales,
                         bo.mx.col_scales[:int(ocb[-1])])
        compare_mx(bview, ref, f"replay {seed} bwd")
        assert np.array_equal(bf16_u16(bo.dx), ref["dx"])
    del g


def test_out_buffer_errors(cuda_device):
    M, N = 32, 128
    c = random_case(M, N, 4)
    x, sg = c["x"].to(cuda_device), c["s"].to(cuda_device)
    bad_shape = _mx_buffers(M, N, 1, cuda_device)._replace(
        row_scales=torch.empty((M, N // 16), dtype=torch.uint8, device=cuda_device))
    with pytest.raises(ValueError):
        mg.scaled_swiglu_mxfp8_fwd(x, sg, out=bad_shape)
    bad_type = _mx_buffers(M, N, 1, cuda_device)._replace(
        col_scales=torch.empty((1, N), dtype=torch.float32, device=cuda_device))
    with pytest.raises(TypeError):
        mg.scaled_swiglu_mxfp8_fwd(x, sg, out=bad_type)
    missing = _mx_buffers(M, N, 1, cuda_device)._replace(col_codes=None)
    with pytest.raises(ValueError):
        mg.scaled_swiglu_mxfp8_fwd(x, sg, out=missing)

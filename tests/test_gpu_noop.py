"""The device no-op flag (moeact_mx_out.noop_flag): a set flag makes a call
write nothing -- codes, scales, dX, dscale, status -- and a clear flag
computes as usual, including when the flag is flipped between replays of one
captured CUDA graph."""
import numpy as np
import pytest
import torch

import oracle
import moe_gated_activation_b200 as mg
from moe_gated_activation_b200 import _capi
from moe_gated_activation_b200.workloads import bf16_bits, random_case
from parity import compare_mx

pytestmark = pytest.mark.gpu

SENT = 0xA5


def _outs(M, W, dev):
    u8 = dict(dtype=torch.uint8, device=dev)
    o = {"rq": torch.full((M, W), SENT, **u8), "rs": torch.full((M, W // 32), SENT, **u8),
         "cq": torch.full((M, W), SENT, **u8), "cs": torch.full(((M + 31) // 32 + 8, W), SENT, **u8),
         "dx": torch.full((M, W), -7.0, dtype=torch.bfloat16, device=dev),
         "dscale": torch.full((M,), -7.0, device=dev),
         "st": torch.full((1,), 99, dtype=torch.int32, device=dev)}
    return o


def _untouched(o):
    for k in ("rq", "rs", "cq", "cs"):
        assert bool((o[k] == SENT).all()), k
    assert bool((o["dx"] == -7.0).all()) and bool((o["dscale"] == -7.0).all())
    assert int(o["st"].item()) == 99


@pytest.mark.parametrize("grouped", [False, True])
def test_set_flag_writes_nothing(cuda_device, grouped):
    M, N = 96, 224
    c = random_case(M, N, 5, std=2.0)
    x, s, dy = (c[k].to(cuda_device) for k in ("x", "s", "dy"))
    flag = torch.ones(1, dtype=torch.int32, device=cuda_device)
    m = torch.tensor([40, 0, 56], dtype=torch.int64, device=cuda_device)
    ro, cb, _ = mg.splits_to_offsets(m, M)
    ws = torch.zeros(_capi.lib().scaled_act_mxfp8_bwd_workspace_size(M, N, 3), dtype=torch.uint8,
                     device=cuda_device)
    stream = torch.cuda.current_stream(cuda_device).cuda_stream
    for W, call in ((N, "fwd"), (2 * N, "bwd")):
        o = _outs(M, W, cuda_device)
        mx = _capi.MxOut(o["rq"].data_ptr(), o["rs"].data_ptr(), o["cq"].data_ptr(),
                         o["cs"].data_ptr(), _capi.SCALES_ROWMAJOR, flag.data_ptr())
        if call == "fwd":
            if grouped:
                _capi.call("grouped_scaled_swiglu_mxfp8_fwd", x.data_ptr(), 2 * N, s.data_ptr(), M,
                           N, 3, 0, 0, ro.data_ptr(), cb.data_ptr(), 3, o["st"].data_ptr(), mx,
                           stream)
            else:
                _capi.call("scaled_swiglu_mxfp8_fwd", x.data_ptr(), 2 * N, s.data_ptr(), M, N, 3, 0,
                           0, mx, stream)
        else:
            args = [dy.data_ptr(), N, x.data_ptr(), 2 * N, s.data_ptr(), M, N, 3, 0]
            if grouped:
                _capi.call("grouped_scaled_swiglu_mxfp8_bwd", *args, ro.data_ptr(), cb.data_ptr(),
                           3, o["st"].data_ptr(), o["dx"].data_ptr(), o["dscale"].data_ptr(), mx,
                           ws.data_ptr(), ws.numel(), stream)
            else:
                _capi.call("scaled_swiglu_mxfp8_bwd", *args, o["dx"].data_ptr(),
                           o["dscale"].data_ptr(), mx, ws.data_ptr(), ws.numel(), stream)
        torch.cuda.synchronize()
        _untouched(o)


def test_clear_flag_computes_and_clamped_honours_it(cuda_device):
    M, N = 64, 128
    c = random_case(M, N, 6, std=2.0)
    x, s = c["x"].to(cuda_device), c["s"].to(cuda_device)
    off = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    got = mg.scaled_swiglu_mxfp8_fwd(x, s, noop_flag=off)
    torch.cuda.synchronize()
    compare_mx(got, oracle.act_fwd(bf16_bits(c["x"]), c["s"].numpy(), N, 3), "flag clear", exact=True)
    on = torch.ones(1, dtype=torch.int32, device=cuda_device)
    b = mg.scaled_clamped_swiglu_mxfp8_bwd(c["dy"].to(cuda_device), x, s, noop_flag=on)
    torch.cuda.synchronize()
    assert b.dx.shape == (M, 2 * N)       # allocated, never written: no error either


def test_flag_flipped_between_graph_replays(cuda_device):
    M, N = 128, 256
    c1, c2 = random_case(M, N, 7, std=2.0), random_case(M, N, 8, std=2.0)
    x = c1["x"].to(cuda_device).clone()
    s = c1["s"].to(cuda_device).clone()
    flag = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    mg.init()
    side = torch.cuda.Stream(cuda_device)
    side.wait_stream(torch.cuda.current_stream(cuda_device))
    with torch.cuda.stream(side):
        mg.scaled_swiglu_mxfp8_fwd(x, s, noop_flag=flag)          # warm-up outside capture
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            out = mg.scaled_swiglu_mxfp8_fwd(x, s, noop_flag=flag)
    torch.cuda.current_stream(cuda_device).wait_stream(side)
    g.replay()
    torch.cuda.synchronize()
    ref1 = oracle.act_fwd(bf16_bits(c1["x"]), c1["s"].numpy(), N, 3)
    compare_mx(out, ref1, "replay 1", exact=True)
    x.copy_(c2["x"].to(cuda_device))
    s.copy_(c2["s"].to(cuda_device))
    flag.fill_(1)
    g.replay()
    torch.cuda.synchronize()
    compare_mx(out, ref1, "skipped replay keeps the old outputs", exact=True)
    flag.fill_(0)
    g.replay()
    torch.cuda.synchronize()
    compare_mx(out, oracle.act_fwd(bf16_bits(c2["x"]), c2["s"].numpy(), N, 3), "replay 3",
               exact=True)
    del g

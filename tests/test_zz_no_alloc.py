"""The allocation-free backward entry point (scaled_swiglu_mxfp8_bwd_noalloc).

Some callers of this library cannot allocate device memory when they call it
(a cudaMalloc may synchronise the device, or all device memory belongs to a
framework allocator that cannot hand out scratch), so this entry point keeps the
dscale partial sums in an array built into the library instead of a caller
workspace.  This test calls it twice in a row through the C ABI, on different
inputs, and checks every output against the workspace-taking entry point
(scaled_swiglu_mxfp8_bwd) under the same rules as the other parity tests.
It lives in its own file so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

from moe_gated_activation_b200 import _capi
from moe_gated_activation_b200.workloads import bf16_bits, random_case
from parity import assert_dscale, dscale_abs_bound

pytestmark = pytest.mark.gpu


def _outputs(M, N, dev):
    W = 2 * N
    u8 = dict(dtype=torch.uint8, device=dev)
    o = {"rq": torch.empty(M, W, **u8), "rs": torch.empty(M, W // 32, **u8),
         "cq": torch.empty(M, W, **u8), "cs": torch.empty((M + 31) // 32, W, **u8),
         "dx": torch.empty(M, W, dtype=torch.bfloat16, device=dev),
         "dscale": torch.empty(M, dtype=torch.float32, device=dev)}
    mx = _capi.MxOut(o["rq"].data_ptr(), o["rs"].data_ptr(), o["cq"].data_ptr(),
                     o["cs"].data_ptr())
    return o, mx


def _run(name, case, dev, workspace=None):
    x = case["x"].to(dev)
    s = case["s"].to(dev)
    dy = case["dy"].to(dev)
    M, N = dy.shape
    o, mx = _outputs(M, N, dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    args = [dy.data_ptr(), N, x.data_ptr(), 2 * N, s.data_ptr(), M, N, 3]
    if workspace is not None:
        args.append(0)   # glu_interleave: [gate | up] halves (the no-alloc call has no such argument)
    args += [o["dx"].data_ptr(), o["dscale"].data_ptr(), mx]
    if workspace is not None:
        args += [workspace.data_ptr(), workspace.numel()]
    _capi.call(name, *args, stream)
    torch.cuda.synchronize()
    return o


def test_noalloc_backward_matches_the_workspace_entry_point(cuda_device):
    lib = _capi.lib()
    for M, N, seed in ((96, 224, 3), (257, 320, 4)):
        case = random_case(M, N, seed, std=2.0)
        ws = torch.zeros(lib.scaled_act_mxfp8_bwd_workspace_size(M, N, 1), dtype=torch.uint8,
                         device=cuda_device)
        ref = _run("scaled_swiglu_mxfp8_bwd", case, cuda_device, ws)
        got = _run("scaled_swiglu_mxfp8_bwd_noalloc", case, cuda_device)
        for k in ("rq", "rs", "cq", "cs"):
            assert torch.equal(got[k], ref[k]), k
        assert torch.equal(got["dx"].view(torch.int16), ref["dx"].view(torch.int16))
        bound = dscale_abs_bound(bf16_bits(case["dy"]), bf16_bits(case["x"]),
                                 case["s"].numpy(), N)
        assert_dscale(got["dscale"], ref["dscale"].cpu().numpy(), bound, "noalloc dscale")


def test_noalloc_backward_rejects_sizes_beyond_its_scratch(cuda_device):
    lib = _capi.lib()
    A16 = 1 << 20   # never dereferenced: the call must fail before launching
    M, N = 1 << 17, 8192          # needs 128 * 131072 * 4 bytes = 64 MiB > 16 MiB
    st = lib.scaled_swiglu_mxfp8_bwd_noalloc(A16, N, A16, 2 * N, A16, M, N, 0, None, A16,
                                             _capi.MxOut(None, None, None, None), None)
    assert st == _capi.ERANGE
    assert b"built-in scratch" in lib.moeact_last_error()

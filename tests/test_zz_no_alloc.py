"""The allocation-free backward entry point (scaled_swiglu_mxfp8_bwd_noalloc).

Some callers of this library cannot allocate device memory when they call it
(a cudaMalloc may synchronise the device, or all device memory belongs to a
framework allocator that cannot hand out scratch), so this entry point keeps the
dscale partial sums in an array built into the library instead of a caller
workspace.  These tests call it through the C ABI, two calls in a row on
different inputs, and check every output against the workspace-taking entry
point (scaled_swiglu_mxfp8_bwd: the same kernels and the same fixed-order
dscale sum, so everything must agree bit for bit) and against the oracle
(under the parity rules of the other GPU tests).  The file is named so that
pytest collects it last.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_gated_activation_b200 import _capi
from moe_gated_activation_b200.workloads import bf16_bits, random_case
from parity import assert_dscale, dscale_abs_bound

pytestmark = pytest.mark.gpu


def _outputs(M, N, dirs, dev, want_dscale=True):
    W = 2 * N
    u8 = dict(dtype=torch.uint8, device=dev)
    o = {"rq": torch.empty(M, W, **u8) if dirs & 1 else None,
         "rs": torch.empty(M, W // 32, **u8) if dirs & 1 else None,
         "cq": torch.empty(M, W, **u8) if dirs & 2 else None,
         "cs": torch.empty((M + 31) // 32, W, **u8) if dirs & 2 else None,
         "dx": torch.empty(M, W, dtype=torch.bfloat16, device=dev),
         "dscale": torch.empty(M, dtype=torch.float32, device=dev) if want_dscale else None}
    p = lambda t: None if t is None else t.data_ptr()
    mx = _capi.MxOut(p(o["rq"]), p(o["rs"]), p(o["cq"]), p(o["cs"]))
    return o, mx


def _run(name, case, dev, dirs=3, workspace=None, want_dscale=True):
    x = case["x"].to(dev)
    s = case["s"].to(dev)
    dy = case["dy"].to(dev)
    M, N = dy.shape
    o, mx = _outputs(M, N, dirs, dev, want_dscale)
    stream = torch.cuda.current_stream(dev).cuda_stream
    args = [dy.data_ptr(), N, x.data_ptr(), 2 * N, s.data_ptr(), M, N, dirs]
    if workspace is not None:
        args.append(0)   # glu_interleave: [gate | up] halves (the no-alloc call has no such argument)
    args += [o["dx"].data_ptr(), None if o["dscale"] is None else o["dscale"].data_ptr(), mx]
    if workspace is not None:
        args += [workspace.data_ptr(), workspace.numel()]
    _capi.call(name, *args, stream)
    torch.cuda.synchronize()
    return o


def _check_against_oracle(got, case, N, dirs, what):
    ref = oracle.act_bwd(bf16_bits(case["dy"]), bf16_bits(case["x"]), case["s"].numpy(), N, dirs,
                         want_dscale=got["dscale"] is not None)
    assert np.array_equal(got["dx"].view(torch.int16).cpu().numpy().view(np.uint16), ref["dx"]), \
        what + " dx"
    for k, rk in (("rq", "row_codes"), ("rs", "row_scales"), ("cq", "col_codes"),
                  ("cs", "col_scales")):
        if got[k] is None:
            assert ref[rk] is None, what + " " + k
        else:
            assert np.array_equal(got[k].cpu().numpy(), ref[rk]), what + " " + k
    if got["dscale"] is not None:
        bound = dscale_abs_bound(bf16_bits(case["dy"]), bf16_bits(case["x"]),
                                 case["s"].numpy(), N)
        assert_dscale(got["dscale"], ref["dscale"], bound, what + " dscale")


def test_noalloc_backward_matches_the_workspace_entry_point_and_the_oracle(cuda_device):
    lib = _capi.lib()
    # two calls in a row: the second one starts on the first one's scratch
    for M, N, seed in ((96, 224, 3), (257, 320, 4)):
        case = random_case(M, N, seed, std=2.0)
        ws = torch.zeros(lib.scaled_act_mxfp8_bwd_workspace_size(M, N, 1), dtype=torch.uint8,
                         device=cuda_device)
        ref = _run("scaled_swiglu_mxfp8_bwd", case, cuda_device, workspace=ws)
        got = _run("scaled_swiglu_mxfp8_bwd_noalloc", case, cuda_device)
        for k in ("rq", "rs", "cq", "cs"):
            assert torch.equal(got[k], ref[k]), k
        assert torch.equal(got["dx"].view(torch.int16), ref["dx"].view(torch.int16))
        # the same partial sums, summed in the same fixed order
        assert torch.equal(got["dscale"].view(torch.int32), ref["dscale"].view(torch.int32))
        _check_against_oracle(got, case, N, 3, f"noalloc M={M} N={N}")


def test_noalloc_backward_without_dscale_and_one_direction(cuda_device):
    # without dscale the built-in scratch is not used; rowwise and colwise alone
    case = random_case(160, 256, 5)
    for dirs, want_dscale in ((3, False), (1, True), (2, True), (1, False)):
        got = _run("scaled_swiglu_mxfp8_bwd_noalloc", case, cuda_device, dirs=dirs,
                   want_dscale=want_dscale)
        _check_against_oracle(got, case, 256, dirs, f"noalloc dirs={dirs} dscale={want_dscale}")


def test_noalloc_backward_rejects_sizes_beyond_its_scratch(cuda_device):
    # ceil(N/128) * M = 64 * 65568 > 4194304: needs more than the 16 MiB of
    # built-in scratch.  Every buffer is real and of the full size, so even a
    # call that got past the check would stay inside memory it owns.
    lib = _capi.lib()
    M, N = 65568, 8192
    dy = torch.zeros(M, N, dtype=torch.bfloat16, device=cuda_device)
    x = torch.zeros(M, 2 * N, dtype=torch.bfloat16, device=cuda_device)
    s = torch.zeros(M, dtype=torch.float32, device=cuda_device)
    dscale = torch.full((M,), 7.0, dtype=torch.float32, device=cuda_device)
    st = lib.scaled_swiglu_mxfp8_bwd_noalloc(dy.data_ptr(), N, x.data_ptr(), 2 * N, s.data_ptr(),
                                             M, N, 0, None, dscale.data_ptr(),
                                             _capi.MxOut(None, None, None, None), None)
    assert st == _capi.ERANGE
    assert b"built-in scratch" in lib.moeact_last_error()
    torch.cuda.synchronize()
    assert bool((dscale == 7.0).all()), "a rejected call wrote its output"
    # one row fewer per tile fits: 64 * 65536 = 4194304
    st = lib.scaled_swiglu_mxfp8_bwd_noalloc(dy.data_ptr(), N, x.data_ptr(), 2 * N, s.data_ptr(),
                                             65536, N, 0, None, dscale.data_ptr(),
                                             _capi.MxOut(None, None, None, None), None)
    assert st == _capi.OK
    torch.cuda.synchronize()
    assert bool((dscale[:65536] == 0.0).all()) and bool((dscale[65536:] == 7.0).all())
    # a bad shape gets the shape error, not the scratch error
    st = lib.scaled_swiglu_mxfp8_bwd_noalloc(dy.data_ptr(), N, x.data_ptr(), 2 * N, s.data_ptr(),
                                             M, N + 16, 0, None, dscale.data_ptr(),
                                             _capi.MxOut(None, None, None, None), None)
    assert st == _capi.EINVAL

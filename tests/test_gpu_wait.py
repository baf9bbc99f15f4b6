"""Failure detection of the fused kernels' bounded waits, without a GPU fault.

Every wait of the fused kernels on their TMA copies is bounded by the GPU's
global timer; a wait that gives up sets a bit in the device error word and
the kernel returns.  moeact_wait_selftest runs that same wait routine on an
mbarrier that nothing ever arrives on (a phase that never completes), with a
short limit, so the timeout path runs for real: the wait must give up after
about its limit, the bit must reach the host through moeact_device_error,
reading must clear it, and the GPU must stay usable (a fused call afterwards
still matches the oracle).  The positive case (the barrier completes) must
not time out.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import moe_gated_activation_b200 as mg
from moe_gated_activation_b200 import _capi
from moe_gated_activation_b200.workloads import bf16_bits, random_case

pytestmark = pytest.mark.gpu


def _error_word():
    v = ctypes.c_uint32(0)
    _capi.call("moeact_device_error", ctypes.byref(v))
    return v.value


def _selftest(arrive, limit_us, dev):
    res = torch.zeros(2, dtype=torch.int64, device=dev)
    _capi.call("moeact_wait_selftest", arrive, limit_us, res.data_ptr(),
               torch.cuda.current_stream(dev).cuda_stream)
    torch.cuda.synchronize()
    done, ns = (int(v) for v in res.cpu())
    return done, ns


def test_wait_completes_when_the_barrier_does(cuda_device):
    mg.init()
    assert _error_word() == 0
    done, ns = _selftest(1, 50_000, cuda_device)
    assert done == 1
    assert ns < 50_000_000
    assert _error_word() == 0


def test_wait_gives_up_after_its_limit_and_reports_it(cuda_device):
    mg.init()
    assert _error_word() == 0
    limit_us = 20_000                       # 20 ms
    done, ns = _selftest(0, limit_us, cuda_device)
    assert done == 0, "a wait on a barrier nothing arrives on completed"
    assert ns >= limit_us * 1000, f"gave up after {ns} ns, before its {limit_us} us limit"
    assert ns < 20 * limit_us * 1000, f"gave up only after {ns} ns"
    assert _error_word() == _capi.DEVERR_WAIT_SELFTEST
    assert _error_word() == 0, "reading the error word must clear it"
    # the context is still usable: a fused forward after the timeout is exact
    c = random_case(64, 128, 11)
    got = mg.scaled_swiglu_mxfp8_fwd(c["x"].to(cuda_device), c["s"].to(cuda_device))
    ref = oracle.act_fwd(bf16_bits(c["x"]), c["s"].numpy(), 128, 3)
    torch.cuda.synchronize()
    assert np.array_equal(got.row_codes.view(torch.uint8).cpu().numpy(), ref["row_codes"])
    assert np.array_equal(got.col_scales.cpu().numpy(), ref["col_scales"])
    assert _error_word() == 0


def test_wait_selftest_argument_errors(cuda_device):
    lib = _capi.lib()
    res = torch.zeros(4, dtype=torch.int64, device=cuda_device)
    assert lib.moeact_wait_selftest(0, 0, res.data_ptr(), None) == _capi.ERANGE
    assert lib.moeact_wait_selftest(0, 2_000_001, res.data_ptr(), None) == _capi.ERANGE
    assert lib.moeact_wait_selftest(2, 10, res.data_ptr(), None) == _capi.EINVAL
    assert lib.moeact_wait_selftest(0, 10, None, None) == _capi.EINVAL
    assert lib.moeact_wait_selftest(0, 10, res.data_ptr() + 4, None) == _capi.EALIGN
    torch.cuda.synchronize()
    assert int(res.abs().sum()) == 0

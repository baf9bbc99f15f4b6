"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/moeact.h declares, and rejects invalid arguments on the
host before touching CUDA (pytorch/ao PR #4743, Numerics and tests: every
launcher error path is exercised).

These calls are meant to fail on the host.  Their pointers point into this
module's own host buffer, and they only ever run in a process that sees no
GPU: where one is visible, the module runs itself again in a child process
with CUDA_VISIBLE_DEVICES empty, so that a regressed host check can never
launch a kernel on them."""
import ctypes
import os
import re
import subprocess
import sys

import numpy as np
import pytest

from moe_gated_activation_b200 import _capi
from moe_gated_activation_b200 import build as mbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
_CHILD = os.environ.get("MOEACT_HOST_CHECKS_CHILD") == "1"


def _gpu_visible():
    import torch
    return torch.cuda.is_available()


GPU_VISIBLE = (not _CHILD) and _gpu_visible()


@pytest.fixture(autouse=True)
def _only_without_a_gpu(request):
    if GPU_VISIBLE and request.node.originalname != "test_host_checks_run_without_a_gpu":
        pytest.skip("runs in a child process with no GPU visible "
                    "(test_host_checks_run_without_a_gpu)")


def test_host_checks_run_without_a_gpu():
    """With a GPU visible, this module's checks run again in a child process
    that sees none (and must pass there)."""
    if not GPU_VISIBLE:
        return
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", MOEACT_HOST_CHECKS_CHILD="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider",
                        os.path.abspath(__file__)], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]


@pytest.fixture(scope="module")
def lib():
    mbuild.build()
    return _capi.lib()


def header_functions():
    src = open(os.path.join(ROOT, "include", "moeact.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z_][a-z0-9_]*)\s*\(",
                       src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_expected_entry_points():
    names = header_functions()
    for n in ["splits_to_offsets", "scaled_swiglu_mxfp8_fwd", "scaled_swiglu_mxfp8_bwd",
              "grouped_scaled_swiglu_mxfp8_fwd", "grouped_scaled_swiglu_mxfp8_bwd",
              "scaled_srelu_mxfp8_fwd", "scaled_srelu_mxfp8_bwd", "moeact_init",
              "moeact_status_string", "moeact_last_error", "scaled_act_mxfp8_bwd_workspace_size"]:
        assert n in names, n


def test_library_exports_every_declared_function(lib):
    for n in header_functions():
        assert hasattr(lib, n), n
        assert n in _capi._SIGS, f"{n} has no ctypes declaration"


def test_status_strings(lib):
    for st in range(7):
        assert lib.moeact_status_string(st)
    assert lib.moeact_status_string(99) == b"unknown status"


# This module's own host memory (1 MiB); A16 is a 16-byte-aligned address in
# it, and A16 + k (k < 64) stays inside it.  No call here gets as far as using
# a pointer.
_BUF = np.zeros(1 << 20, dtype=np.uint8)
A16 = (_BUF.ctypes.data + 15) & ~15
MX_ROW = _capi.MxOut(A16, A16, None, None)
MX_BOTH = _capi.MxOut(A16, A16, A16, A16)


def fwd(lib, x=A16, ldx=512, s=A16, M=64, N=256, dirs=1, staged=0, mx=MX_ROW, ilv=0):
    return lib.scaled_swiglu_mxfp8_fwd(x, ldx, s, M, N, dirs, staged, ilv, mx, None)


@pytest.mark.parametrize("kw,status", [
    (dict(x=None), _capi.EINVAL),
    (dict(s=None), _capi.EINVAL),
    (dict(M=-1), _capi.EINVAL),
    (dict(N=0), _capi.EINVAL),
    (dict(N=48), _capi.EINVAL),                 # not a multiple of 32
    (dict(ldx=256), _capi.EINVAL),              # narrower than 2N
    (dict(ldx=516), _capi.EALIGN),              # not a multiple of 8 elements
    (dict(x=A16 + 8), _capi.EALIGN),
    (dict(s=A16 + 2), _capi.EALIGN),
    (dict(dirs=0), _capi.EINVAL),
    (dict(dirs=4), _capi.EINVAL),
    (dict(staged=2), _capi.EINVAL),
    (dict(dirs=3), _capi.EINVAL),               # colwise pointers missing
    (dict(mx=_capi.MxOut(A16, None, None, None)), _capi.EINVAL),
    (dict(mx=_capi.MxOut(A16 + 4, A16, None, None)), _capi.EALIGN),
    (dict(mx=MX_BOTH), _capi.EINVAL),           # colwise pointers given, not requested
    (dict(M=1 << 37), _capi.ERANGE),
    (dict(N=1 << 25, ldx=1 << 26), _capi.ERANGE),
])
def test_forward_argument_errors(lib, kw, status):
    assert fwd(lib, **kw) == status
    assert lib.moeact_last_error()


def test_empty_input_is_ok_without_launch(lib):
    assert fwd(lib, M=0) == _capi.OK
    assert lib.scaled_srelu_mxfp8_fwd(A16, 256, A16, 0, 256, 1, MX_ROW, None) == _capi.OK


def bwd(lib, dy=A16, lddy=256, x=A16, ldx=512, s=A16, M=64, N=256, dirs=1, dx=A16, dscale=A16,
        mx=MX_ROW, ws=A16, wsb=1 << 30, ilv=0):
    return lib.scaled_swiglu_mxfp8_bwd(dy, lddy, x, ldx, s, M, N, dirs, ilv, dx, dscale, mx, ws,
                                       wsb, None)


@pytest.mark.parametrize("kw,status", [
    (dict(dy=None), _capi.EINVAL),
    (dict(lddy=128), _capi.EINVAL),
    (dict(lddy=260), _capi.EALIGN),
    (dict(dy=A16 + 2), _capi.EALIGN),
    (dict(dx=A16 + 4), _capi.EALIGN),
    (dict(dscale=A16 + 1), _capi.EALIGN),
    (dict(ws=None), _capi.EWORKSPACE),
    (dict(wsb=16), _capi.EWORKSPACE),
    (dict(ws=A16 + 8), _capi.EALIGN),
    (dict(dirs=0, dx=None, dscale=None), _capi.EINVAL),
    (dict(dirs=5), _capi.EINVAL),
])
def test_backward_argument_errors(lib, kw, status):
    assert bwd(lib, **kw) == status


def test_backward_workspace_only_needed_for_dscale(lib):
    assert bwd(lib, M=0, dscale=None, ws=None) == _capi.OK
    n = lib.scaled_act_mxfp8_bwd_workspace_size(4096, 2048, 1)
    assert n >= -(-2048 // 128) * 4096 * 4     # ceil(N/128) x M fp32 partial sums
    assert n % 16 == 0
    assert lib.scaled_act_mxfp8_bwd_workspace_size(-1, 2048, 1) == 0


def test_grouped_argument_errors(lib):
    f = lib.grouped_scaled_swiglu_mxfp8_fwd
    args = lambda ro=A16, cb=A16, E=4, st=A16: (A16, 512, A16, 64, 256, 1, 0, 0, ro, cb, E, st,
                                                 MX_ROW, None)
    assert f(*args(ro=None)) == _capi.EINVAL
    assert f(*args(st=None)) == _capi.EINVAL
    assert f(*args(E=0)) == _capi.EINVAL
    assert f(*args(E=_capi.MAX_GROUPS + 1)) == _capi.EINVAL
    assert f(*args(ro=A16 + 4)) == _capi.EALIGN


def test_splits_to_offsets_argument_errors(lib):
    f = lib.splits_to_offsets
    assert f(A16, 4, 64, None, A16, A16, None) == _capi.EINVAL
    assert f(A16, -1, 64, A16, A16, A16, None) == _capi.EINVAL
    assert f(A16, _capi.MAX_GROUPS + 1, 64, A16, A16, A16, None) == _capi.EINVAL
    assert f(A16, 4, -1, A16, A16, A16, None) == _capi.EINVAL
    assert f(A16 + 4, 4, 64, A16, A16, A16, None) == _capi.EALIGN
    assert f(A16, 4, 1 << 40, A16, A16, A16, None) == _capi.ERANGE


def test_gemm_scale_layout_argument_errors(lib):
    gemm = lambda *p: _capi.MxOut(*p, _capi.SCALES_GEMM)
    bad_layout = _capi.MxOut(A16, A16, None, None, 2)
    assert fwd(lib, mx=bad_layout) == _capi.EINVAL
    assert fwd(lib, M=256, N=96, ldx=192, mx=gemm(A16, A16, None, None)) == _capi.EINVAL
    assert b"multiples of 128" in lib.moeact_last_error()
    assert fwd(lib, M=100, N=256, mx=gemm(A16, A16, None, None)) == _capi.EINVAL
    assert bwd(lib, M=96, N=128, ldx=256, lddy=128, mx=gemm(A16, A16, None, None)) == _capi.EINVAL
    assert fwd(lib, M=0, N=256, mx=gemm(A16, A16, None, None)) == _capi.OK


def test_noop_flag_alignment(lib):
    mx = _capi.MxOut(A16, A16, None, None, _capi.SCALES_ROWMAJOR, A16 + 2)
    assert fwd(lib, mx=mx) == _capi.EALIGN


@pytest.mark.parametrize("ilv,N,status", [
    (16, 256, _capi.EINVAL),      # not a multiple of 32
    (-32, 256, _capi.EINVAL),
    (96, 384, _capi.EINVAL),      # divides N, but neither 32, 64 nor a multiple of 128
    (256, 384, _capi.EINVAL),     # does not divide N
    (64, 96, _capi.EINVAL),       # does not divide N
    (32, 256, _capi.OK),          # M = 0: checked, nothing launched
    (64, 192, _capi.OK),
    (128, 384, _capi.OK),
    (96, 96, _capi.OK),           # G = N is the halves layout
])
def test_glu_interleave_arguments(lib, ilv, N, status):
    """glu_interleave: 32, 64 or a multiple of 128 dividing N, or 0 / N."""
    assert fwd(lib, M=0, N=N, ldx=2 * N, ilv=ilv) == status
    assert bwd(lib, M=0, N=N, ldx=2 * N, lddy=N, ilv=ilv) == status
    clamped = lib.scaled_clamped_swiglu_mxfp8_fwd(A16, 2 * N, A16, 0, N, 1, 1.702, 7.0, ilv,
                                                  MX_ROW, None)
    assert clamped == status



def fc2(lib, x=A16, ldx=512, s=A16, M=64, N=256, staged=0, ro=A16, E=4, st=A16, wc=A16,
        ws=A16, H=256, out=A16, ldo=256, noop=None):
    return lib.grouped_scaled_swiglu_mxfp8_fc2(x, ldx, s, M, N, staged, ro, E, st, wc, ws, H, out,
                                               ldo, noop, None)


@pytest.mark.parametrize("kw,status", [
    (dict(x=None), _capi.EINVAL),
    (dict(N=96, ldx=192), _capi.EINVAL),          # N not a multiple of 128
    (dict(N=896, ldx=1792), _capi.EUNSUPPORTED),  # the 128-row block must fit on chip
    (dict(staged=2), _capi.EINVAL),
    (dict(ro=None), _capi.EINVAL),
    (dict(st=None), _capi.EINVAL),
    (dict(E=0), _capi.EINVAL),
    (dict(E=_capi.MAX_GROUPS + 1), _capi.EINVAL),
    (dict(ro=A16 + 4), _capi.EALIGN),
    (dict(st=A16 + 2), _capi.EALIGN),
    (dict(wc=None), _capi.EINVAL),
    (dict(ws=None), _capi.EINVAL),
    (dict(out=None), _capi.EINVAL),
    (dict(wc=A16 + 8), _capi.EALIGN),
    (dict(out=A16 + 8), _capi.EALIGN),
    (dict(H=0), _capi.EINVAL),
    (dict(H=192, ldo=192), _capi.EINVAL),         # H not a multiple of 128
    (dict(ldo=128), _capi.EINVAL),                # narrower than H
    (dict(ldo=260), _capi.EALIGN),                # not a multiple of 8 elements
    (dict(noop=A16 + 2), _capi.EALIGN),
    (dict(ldx=256), _capi.EINVAL),                # narrower than 2N
    (dict(H=1 << 21, E=1024, ldo=1 << 21), _capi.ERANGE),   # E * H above 2^31 - 1
])
def test_fc2_argument_errors(lib, kw, status):
    assert fc2(lib, **kw) == status
    assert lib.moeact_last_error()


def test_fc2_empty_input_is_ok_without_launch(lib):
    assert fc2(lib, M=0) == _capi.OK

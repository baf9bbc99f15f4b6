import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a B200 (sm_100a) GPU; runs the CUDA path through the C-ABI")


def golden_path(name):
    return os.path.join(HERE, "golden", name)


def read_golden(name):
    """Rows of a whitespace-separated golden fixture, comments stripped."""
    rows = []
    with open(golden_path(name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split(None, 2))
    return rows


@pytest.fixture(scope="session")
def cuda_device():
    """The B200 the GPU tests run on.  Fails (never skips) without one, so a
    GPU run cannot pass silently on the wrong hardware."""
    import torch
    assert torch.cuda.is_available(), "GPU test needs CUDA"
    cap = torch.cuda.get_device_capability(0)
    assert cap == (10, 0), f"GPU tests target sm_100a (B200); found capability {cap}"
    return torch.device("cuda", 0)


@pytest.fixture(scope="session", autouse=True)
def device_error_word_stays_clear():
    """After the whole session: if the library ran kernels on a GPU, none of
    them may have given up a bounded wait (moeact_device_error reads 0).  The
    wait self-test sets and reads its own bit, so it leaves the word clear."""
    yield
    import ctypes
    import torch
    if not (torch.cuda.is_available() and torch.cuda.is_initialized()):
        return
    from moe_gated_activation_b200 import _capi
    if _capi._lib is None:
        return
    v = ctypes.c_uint32(0)
    _capi.call("moeact_device_error", ctypes.byref(v))
    assert v.value == 0, f"device error word {v.value:#x}: a kernel gave up a bounded wait"

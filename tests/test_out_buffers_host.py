"""Host-side checks of caller-owned output buffers (`out=`) in the Python
binding, on CPU tensors (the checks are independent of the device)."""
import pytest
import torch

from moe_gated_activation_b200 import ops

DEV = torch.device("cpu")


def _out(M, W, col_rows, code_dtype=torch.float8_e4m3fn):
    u8 = dict(dtype=torch.uint8, device=DEV)
    return ops.MXFP8(torch.empty((M, W), **u8).view(code_dtype), torch.empty((M, W), **u8),
                     torch.empty((M, W // 32), **u8), torch.empty((col_rows, W), **u8))


def test_buffers_are_taken_as_uint8_views():
    o = _out(64, 128, 3)
    rq, rs, cq, cs = ops._take_mx(o, 64, 128, ops.ROWWISE | ops.COLWISE, DEV, 2)
    assert rq.dtype == torch.uint8 and rq.data_ptr() == o.row_codes.data_ptr()
    assert cs.shape == (3, 128)      # more col-scale rows than needed is fine


def test_disabled_direction_is_ignored():
    o = _out(64, 128, 2)._replace(col_codes=None, col_scales=None)
    rq, rs, cq, cs = ops._take_mx(o, 64, 128, ops.ROWWISE, DEV, 2)
    assert cq.numel() == 0 and cs.numel() == 0


@pytest.mark.parametrize("field,value,exc", [
    ("row_codes", None, ValueError),
    ("row_scales", torch.empty((64, 8), dtype=torch.uint8), ValueError),      # wrong shape
    ("col_scales", torch.empty((1, 128), dtype=torch.uint8), ValueError),     # too few rows
    ("col_codes", torch.empty((64, 128), dtype=torch.int16), TypeError),
    ("row_codes", torch.empty((128, 64), dtype=torch.uint8).t(), ValueError),  # not contiguous
])
def test_bad_buffers(field, value, exc):
    o = _out(64, 128, 2)._replace(**{field: value})
    with pytest.raises(exc):
        ops._take_mx(o, 64, 128, ops.ROWWISE | ops.COLWISE, DEV, 2)

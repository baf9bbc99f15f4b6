"""Large extents: very wide rows and very many rows (64-bit row offsets, the
largest grids), checked against the oracle (whole output for the wide case,
sampled 32-row slabs plus whole-output properties for the tall one)."""
import numpy as np
import pytest
import torch

import oracle
import moe_gated_activation_b200 as mg
from moe_gated_activation_b200.workloads import bf16_bits, random_case
from parity import assert_dscale, bf16_u16, compare_mx, dscale_abs_bound, u8

pytestmark = pytest.mark.gpu


def test_wide_rows(cuda_device):
    M, N = 40, 65536 + 96          # 513 column tiles, the last one ragged; a partial slab
    c = random_case(M, N, 12, std=2.0)
    xb, s, dyb = bf16_bits(c["x"]), c["s"].numpy(), bf16_bits(c["dy"])
    x, sg, dy = c["x"].to(cuda_device), c["s"].to(cuda_device), c["dy"].to(cuda_device)
    got = mg.scaled_swiglu_mxfp8_fwd(x, sg)
    gotb = mg.scaled_swiglu_mxfp8_bwd(dy, x, sg)
    torch.cuda.synchronize()
    compare_mx(got, oracle.act_fwd(xb, s, N, 3), "wide fwd", exact=True)
    refb = oracle.act_bwd(dyb, xb, s, N, 3)
    compare_mx(gotb.mx, refb, "wide bwd", exact=True)
    assert np.array_equal(bf16_u16(gotb.dx), refb["dx"])
    assert_dscale(gotb.dscale, refb["dscale"], dscale_abs_bound(dyb, xb, s, N), "wide dscale")


def test_many_rows(cuda_device):
    M, N = (1 << 22) + 17, 32      # 131,073 slabs, the last one partial
    g = torch.Generator(device=cuda_device).manual_seed(13)
    x = (torch.randn(M, 2 * N, generator=g, device=cuda_device) * 2).to(torch.bfloat16)
    s = torch.rand(M, generator=g, device=cuda_device)
    dy = torch.randn(M, N, generator=g, device=cuda_device).to(torch.bfloat16)
    got = mg.scaled_swiglu_mxfp8_fwd(x, s)
    gotb = mg.scaled_swiglu_mxfp8_bwd(dy, x, s)
    torch.cuda.synchronize()
    S = (M + 31) // 32
    for slab in (0, 1, S // 2, S - 2, S - 1):
        r0, n = 32 * slab, min(32, M - 32 * slab)
        rows = slice(r0, r0 + n)
        xb = bf16_bits(x[rows].cpu())
        sv = s[rows].cpu().numpy()
        dyb = bf16_bits(dy[rows].cpu())
        ref = oracle.act_fwd(xb, sv, N, 3)
        for k in ("row_codes", "row_scales", "col_codes"):
            assert np.array_equal(u8(getattr(got, k)[rows]), ref[k]), (slab, k)
        assert np.array_equal(u8(got.col_scales[slab:slab + 1]), ref["col_scales"]), slab
        refb = oracle.act_bwd(dyb, xb, sv, N, 3)
        assert np.array_equal(bf16_u16(gotb.dx[rows]), refb["dx"]), slab
        for k in ("row_codes", "row_scales", "col_codes"):
            assert np.array_equal(u8(getattr(gotb.mx, k)[rows]), refb[k]), (slab, k)
        assert np.array_equal(u8(gotb.mx.col_scales[slab:slab + 1]), refb["col_scales"]), slab
        assert_dscale(gotb.dscale[rows], refb["dscale"], dscale_abs_bound(dyb, xb, sv, N),
                      f"dscale slab {slab}")
    # whole output: every live rowwise block's largest code is in [0x76, 0x7E]
    rq = got.row_codes.view(torch.uint8)
    blk = (rq & 0x7F).view(M, N // 32, 32).amax(dim=2)
    live = got.row_scales > 0
    assert bool(((blk >= 0x76) & (blk <= 0x7E))[live].all())

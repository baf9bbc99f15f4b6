"""The seeded synthetic workloads have the shapes and routing statistics the
pages describe (pytorch/ao PR #4743 Performance table; VeOmni PR #1340 Qwen3-MoE
configuration) and are reproducible."""
import torch

from moe_gated_activation_b200 import workloads as W


def test_qwen3_moe_splits():
    q = W.qwen3_moe_splits(seed=2)
    assert q.numel() == 128 and int(q.sum()) == 65536
    assert bool(((q % 128) == 0).all())
    assert int((q == 0).sum()) >= 8          # the dead experts plus undrawn ones
    assert torch.equal(q, W.qwen3_moe_splits(seed=2))


def test_qwen3_moe_row_scales_are_renormalised_top8_probs():
    s = W.qwen3_moe_row_scales(seed=2)
    assert s.shape == (65536,) and s.dtype == torch.float32
    per_tok = s.view(8192, 8)
    assert torch.allclose(per_tok.sum(1), torch.ones(8192), atol=1e-5)
    assert bool((per_tok[:, :-1] >= per_tok[:, 1:]).all())   # top-k order


def test_zipf_splits():
    z = W.zipf_splits(experts=32)
    assert int(z.sum()) == 131072 and bool(((z % 128) == 0).all())
    assert z[:3].tolist() == [37248, 17408, 11136] and int(z[-1]) == 768


def test_make_inputs_small_and_reproducible():
    a = W.make_inputs("c1")
    b = W.make_inputs("c1")
    assert a["x"].shape == (128, 256) and a["x"].dtype == torch.bfloat16
    assert a["s"].shape == (128,) and a["dy"] is None
    assert torch.equal(a["x"], b["x"]) and torch.equal(a["s"], b["s"])
    assert 0.0 <= float(a["s"].min()) and float(a["s"].max()) < 1.0


def test_outlier_recipe_statistics():
    wl = W.Workload("t", "t", M=2048, N=512, seed=3, x_std=2 ** 0.5,
                    outlier_p=1e-3, outlier_mul=100.0)
    x = W.make_inputs(wl, with_dy=False)["x"].float()
    frac = float((x.abs() > 30).float().mean())
    assert 3e-4 < frac < 2e-3
    core = x[x.abs() < 30]
    assert abs(float(core.std()) - 2 ** 0.5) < 0.05

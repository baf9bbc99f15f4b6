"""Seeded synthetic inputs for the scaled gated activation + MXFP8 path.

This module only draws inputs: it holds none of the method's arithmetic and is
the one piece shared by the CUDA path's tests/benchmark and the CPU oracle's
tests.  Every workload is generated with a ``torch.Generator`` seeded with the
workload's index, on the device it is requested for (CPU draws and CUDA draws
of the same seed differ; a test that compares two implementations always feeds
both the same tensors).

Shapes and distributions follow the workloads of the pages:
  * the MXFP8 microbenchmark table of pytorch/ao PR #4743 (section
    "Performance": (M, K) output shapes, gated input [M, 2K] bf16);
  * the Qwen3-MoE configuration of VeOmni PR #1340 (section "Test": hidden
    2048, expert intermediate 768, 128 experts, top-k 8) for the grouped
    routing statistics;
  * per-row routing-probability scales of TransformerEngine PR #3238
    (Greptile summary: per-row-scaled activation).
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    key: str
    title: str
    M: int                 # routed rows
    N: int                 # activation width (the pages' K); gated input is [M, 2N]
    seed: int
    groups: int = 1        # experts (1 = single group)
    x_std: float = 1.0
    outlier_p: float = 0.0
    outlier_mul: float = 1.0
    fwd_only: bool = False
    staged: tuple = (False,)
    srelu_N: int = 0       # width of the separate SReLU input, 0 = none

    @property
    def grouped(self) -> bool:
        return self.groups > 1


WORKLOADS = {
    "c1": Workload("c1", "single group, forward only, SwiGLU, X bf16 [128, 256]",
                   M=128, N=128, seed=0, fwd_only=True),
    "c2": Workload("c2", "single group, SwiGLU fwd+bwd, X bf16 [4096, 4096], dY [4096, 2048]",
                   M=4096, N=2048, seed=1),
    "c3": Workload("c3", "grouped MoE (Qwen3-MoE-like): 8192 tokens x top-8 = 65536 rows, "
                   "128 experts, X bf16 [65536, 1536]", M=65536, N=768, seed=2, groups=128),
    "c4": Workload("c4", "single group, X bf16 [16384, 14336] ~N(0,2) with 0.1% x100 outliers, "
                   "SwiGLU (staged and not) and SReLU on [16384, 7168]",
                   M=16384, N=7168, seed=3, x_std=math.sqrt(2.0), outlier_p=1e-3,
                   outlier_mul=100.0, staged=(False, True), srelu_N=7168),
    "c5": Workload("c5", "large grouped: X bf16 [131072, 16384], 32 experts Zipf(1.1)",
                   M=131072, N=8192, seed=4, groups=32),
}


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _bf16_normal(shape, g, device, std=1.0, outlier_p=0.0, outlier_mul=1.0,
                 chunk_rows=8192):
    """bf16 tensor of N(0, std^2) draws; each entry independently, with
    probability outlier_p, multiplied by outlier_mul before the bf16 rounding.
    Drawn in row chunks to bound the fp32 temporary."""
    M = shape[0]
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    for r0 in range(0, M, chunk_rows):
        r1 = min(M, r0 + chunk_rows)
        t = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=g, device=device)
        if std != 1.0:
            t.mul_(std)
        if outlier_p > 0.0:
            mask = torch.rand(t.shape, generator=g, device=device) < outlier_p
            t = torch.where(mask, t * outlier_mul, t)
        out[r0:r1] = t.to(torch.bfloat16)
    return out


def qwen3_moe_splits(tokens=8192, topk=8, experts=128, unit=128, dead=8, seed=2):
    """m_splits for the Qwen3-MoE-like workload: unit * Multinomial(tokens*topk/unit, p),
    p proportional to softmax of seeded N(0,1) logits with `dead` seeded experts at p = 0.
    Every split is a multiple of `unit` and some experts are empty."""
    g = _gen("cpu", seed + 1000)
    logits = torch.randn(experts, generator=g, dtype=torch.float64)
    p = torch.softmax(logits, 0)
    dead_idx = torch.randperm(experts, generator=g)[:dead]
    p[dead_idx] = 0.0
    p = p / p.sum()
    n_units = tokens * topk // unit
    draws = torch.multinomial(p, n_units, replacement=True, generator=g)
    counts = torch.bincount(draws, minlength=experts).to(torch.int64)
    return counts * unit


def qwen3_moe_row_scales(tokens=8192, topk=8, experts=128, seed=2):
    """Per-row scales: top-k renormalised softmax routing probabilities of seeded
    [tokens, experts] N(0,1) router logits, flattened token-major (fp32 [tokens*topk])."""
    g = _gen("cpu", seed + 2000)
    logits = torch.randn(tokens, experts, generator=g)
    probs = torch.softmax(logits, dim=-1)
    top, _ = torch.topk(probs, topk, dim=-1)
    top = top / top.sum(dim=-1, keepdim=True)
    return top.reshape(-1).to(torch.float32).contiguous()


def zipf_splits(experts=32, alpha=1.1, units=1024, unit=128):
    """Largest-remainder apportionment of `units` blocks of `unit` rows over
    experts with weights 1/(e+1)^alpha (ties to the lower expert index)."""
    w = [1.0 / (e + 1) ** alpha for e in range(experts)]
    tot = sum(w)
    quota = [units * x / tot for x in w]
    base = [int(math.floor(q)) for q in quota]
    rest = units - sum(base)
    order = sorted(range(experts), key=lambda e: (-(quota[e] - base[e]), e))
    for e in order[:rest]:
        base[e] += 1
    return torch.tensor([b * unit for b in base], dtype=torch.int64)


def make_inputs(wl: Workload | str, device="cpu", with_dy=True, srelu=False):
    """Inputs of a workload on `device`: dict with x (bf16 [M, 2N], or [M, N] for
    SReLU), s (fp32 [M]), dy (bf16 [M, N]) and m_splits (int64 [E], CPU)."""
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    device = torch.device(device)
    g = _gen(device, wl.seed + (500 if srelu else 0))
    width = wl.srelu_N if srelu else 2 * wl.N
    n_out = wl.srelu_N if srelu else wl.N
    x = _bf16_normal((wl.M, width), g, device, wl.x_std, wl.outlier_p, wl.outlier_mul)
    if wl.key == "c3":
        s = qwen3_moe_row_scales(seed=wl.seed).to(device)
        m_splits = qwen3_moe_splits(seed=wl.seed)
    else:
        s = torch.rand(wl.M, generator=g, device=device, dtype=torch.float32)
        m_splits = (zipf_splits(experts=wl.groups) if wl.key == "c5"
                    else torch.tensor([wl.M], dtype=torch.int64))
    dy = None
    if with_dy and not wl.fwd_only:
        dy = _bf16_normal((wl.M, n_out), g, device)
    return {"x": x, "s": s, "dy": dy, "m_splits": m_splits}


def random_case(M, N, seed, *, width=None, std=1.0, device="cpu", with_dy=True,
                s_low=0.0, s_high=1.0):
    """A small seeded case for tests: x bf16 [M, width or 2N] ~N(0, std^2),
    s fp32 [M] ~U(s_low, s_high), dy bf16 [M, N] ~N(0,1)."""
    g = _gen(device, seed)
    width = 2 * N if width is None else width
    x = (torch.randn(M, width, generator=g, device=device) * std).to(torch.bfloat16)
    s = torch.rand(M, generator=g, device=device) * (s_high - s_low) + s_low
    dy = (torch.randn(M, N, generator=g, device=device).to(torch.bfloat16)
          if with_dy else None)
    return {"x": x, "s": s.to(torch.float32), "dy": dy}


def bf16_bits(t: torch.Tensor):
    """uint16 numpy view of a bf16 tensor's bit patterns (copied to CPU)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")


def bits_to_bf16(a) -> torch.Tensor:
    """bf16 tensor from a uint16 numpy array of bit patterns."""
    return torch.from_numpy(a.astype("uint16").view("int16")).view(torch.bfloat16)


def fc2_weights(E, H, N, seed, device="cpu", scale_lo=118, scale_hi=124):
    """A seeded MXFP8 FC2 weight for the fused activation -> FC2 path: E4M3
    codes uint8 [E, H, N] drawn uniformly over the finite codes (0x7F and
    0xFF, the NaNs, excluded) and E8M0 scales uint8 [E, H, N/32] uniform in
    [scale_lo, scale_hi].  Both are i.i.d. uniform, so the same bytes serve
    as the tiled operand and scale layouts the fused kernel reads (a
    permutation of i.i.d. bytes has their law).  (The FC2 width of the
    Qwen3-MoE configuration is its hidden size, 2048.)"""
    g = _gen(device, seed)
    c = torch.randint(0, 254, (E, H, N), generator=g, device=device, dtype=torch.int32)
    c = c + (c >= 0x7F).to(torch.int32)          # 0..126 -> 0x00..0x7E, 127..253 -> 0x80..0xFE
    sc = torch.randint(scale_lo, scale_hi + 1, (E, H, N // 32), generator=g, device=device,
                       dtype=torch.int32)
    return c.to(torch.uint8).contiguous(), sc.to(torch.uint8).contiguous()

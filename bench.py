"""Benchmark of the fused scaled gated activation + MXFP8 path on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
splits_to_offsets (per-expert offsets) -> grouped forward (scaled SwiGLU, MXFP8
with the requested scale directions) -> grouped backward (dgate/dup bf16, dscale,
MXFP8 of the gradient).  A single-group workload runs the same calls with one
group.  The metric is algorithmic bytes / device time (GB/s), the byte model of
the pytorch/ao PR #4743 performance table extended with the per-row scale and
the backward's bf16 dX and dscale.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c2]
                    [--dirs both|row|col] [--impl ours|reference]

N > 1 runs under torchrun: every rank runs its own replica of the workload on
its GPU (rows are independent; there is no exchange step), and the device time
is the max over ranks.  L2 is flushed (written then read, 256 MiB) before every
timed step, outside the timed events.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "fused act+MXFP8 quant GB/s (fwd & bwd) and % of B200 HBM roofline"
DIRS = {"both": 3, "row": 1, "col": 2}
FALLBACK_HBM_GBS = 6650.0


# ------------------------------------------------------------------ byte model
def byte_model(M, N, E, dirs, srelu=False, S=None):
    """Algorithmic bytes of one forward and one backward (dx and dscale on)."""
    S = (M + 31) // 32 if S is None else S
    xin = 2 * M * (N if srelu else 2 * N)
    W = N if srelu else 2 * N

    def mx(width):
        b = 0
        if dirs & 1:
            b += M * width + M * width // 32
        if dirs & 2:
            b += M * width + S * width
        return b

    splits = 8 * E + 2 * 8 * (E + 1) + 4
    fwd = xin + 4 * M + mx(N)
    bwd = 2 * M * N + xin + 4 * M + 2 * M * W + 4 * M + mx(W)
    return {"splits": splits, "fwd": fwd, "bwd": bwd}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device):
        self.samples = []
        self.active = False
        self.stop = threading.Event()
        self.err = None
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device)
            bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001
            self.err = repr(e)
            self.h = None

    def _run(self):
        nv = self.nv
        while not self.stop.is_set():
            try:
                if self.active:
                    sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    self.samples.append((sm, rs))
            except Exception as e:  # noqa: BLE001
                self.err = repr(e)
            time.sleep(0.002)

    def __enter__(self):
        if self.h is not None:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self.stop.set()
        if self.h is not None:
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0, "error": self.err}
        mhz = [s for s, _ in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= r
        reasons = [n for b, n in self.REASONS.items() if bits & b]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(mhz), "sm_mhz_min": min(mhz)}


# ------------------------------------------------------------------ helpers
def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:  # noqa: BLE001
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "moe_gated_activation_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload, kernel, dirs_name):
    """Per-launch DRAM bytes from profiles/ncu_traffic.txt, if it was taken on
    the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(p):
        return None
    cur = kernel_source_hash()
    with open(p) as f:
        for line in f:
            line = line.split("#", 1)[0].split()
            if len(line) >= 5 and line[0] == workload and line[1] == kernel and \
                    line[2] == dirs_name and line[3] == cur:
                return int(float(line[4]))
    return None


def act_api(mg, act, glu_interleave=0, staged=False):
    """(grouped forward, grouped backward, forward and backward extra keyword
    arguments) of an activation; ClampedSwiGLU at the default slope and limit;
    gate and up interleaved in blocks of `glu_interleave` columns when it is
    non-zero; SwiGLU's forward with staged rounding when `staged`."""
    if act == "srelu":
        if glu_interleave or staged:
            raise SystemExit("SReLU takes neither --glu-interleave nor --staged")
        return mg.grouped_scaled_srelu_mxfp8_fwd, mg.grouped_scaled_srelu_mxfp8_bwd, {}, {}
    extra = {"glu_interleave": glu_interleave} if glu_interleave else {}
    if act == "clamped":
        if staged:
            raise SystemExit("ClampedSwiGLU has no staged rounding")
        mg.init_clamped()
        extra.update(alpha=mg.ops.CLAMPED_ALPHA, limit=mg.ops.CLAMPED_LIMIT)
        return (mg.grouped_scaled_clamped_swiglu_mxfp8_fwd,
                mg.grouped_scaled_clamped_swiglu_mxfp8_bwd, extra, dict(extra))
    fwd_extra = dict(extra, staged_rounding=True) if staged else dict(extra)
    return (mg.grouped_scaled_swiglu_mxfp8_fwd, mg.grouped_scaled_swiglu_mxfp8_bwd, fwd_extra,
            extra)


def max_over_ranks(value, world, device):
    """The largest `value` over all ranks (every rank gets it); with one rank,
    `value` itself.  `device` is where the collective's tensor lives (cuda
    for NCCL, cpu for gloo)."""
    if world <= 1:
        return float(value)
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world, steps, step_bytes, total_ms):
    """Whole-job throughput of `world` replicas: every rank processed
    `steps` steps of `step_bytes` each; the job took the slowest rank's
    `total_ms`."""
    return world * steps * step_bytes / (total_ms * 1e-3) / 1e9


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}: launch N>1 with torchrun")
    return world, rank, local


# ------------------------------------------------------------------ our arm
def run_ours(args):
    import moe_gated_activation_b200 as mg
    from moe_gated_activation_b200.workloads import WORKLOADS, make_inputs

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    mg.init()
    wl = WORKLOADS[args.workload]
    dirs = DIRS[args.dirs]
    srelu = args.act == "srelu"
    if srelu and not wl.srelu_N:
        raise SystemExit(f"workload {wl.key} has no SReLU input")
    inp = make_inputs(wl, device=dev, srelu=srelu)
    x, s, dy = inp["x"], inp["s"], inp["dy"]
    assert dy is not None, "the benchmark workload needs a backward (dY)"
    m_host = inp["m_splits"]
    m_dev = m_host.to(dev)
    E = int(m_host.numel())
    S = int(((m_host + 31) // 32).sum())
    M, N = wl.M, (wl.srelu_N if srelu else wl.N)
    rw, cw = bool(dirs & 1), bool(dirs & 2)
    bm = byte_model(M, N, E, dirs, srelu=srelu, S=S)
    step_bytes = bm["splits"] + bm["fwd"] + bm["bwd"]

    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    ws = torch.zeros(mg.bwd_workspace_bytes(M, N, E), dtype=torch.uint8, device=dev)

    def do_flush(i):
        flush.fill_(float(i & 7))
        flush.amax()

    def splits():
        return mg.splits_to_offsets(m_dev, M)

    gemm = args.scales == "gemm"
    fwd_api, bwd_api, fwd_extra, bwd_extra = act_api(mg, args.act, args.glu_interleave,
                                                     args.staged)

    def fwd(ro, cb, st):
        return fwd_api(x, s, ro, cb, rowwise=rw, colwise=cw, col_scale_rows=S, status=st,
                       gemm_scales=gemm, **fwd_extra)

    def bwd(ro, cb, st):
        return bwd_api(dy, x, s, ro, cb, rowwise=rw, colwise=cw, col_scale_rows=S, workspace=ws,
                       status=st, gemm_scales=gemm, **bwd_extra)

    # eager warm-up
    for i in range(3):
        ro, cb, st = splits()
        fwd(ro, cb, st)
        bwd(ro, cb, st)
    torch.cuda.synchronize()

    if args.eager:
        def run_step(ev):
            ev[0].record(stream)
            ro, cb, st = splits()
            ev[1].record(stream)
            fwd(ro, cb, st)
            ev[2].record(stream)
            bwd(ro, cb, st)
            ev[3].record(stream)
    else:
        # The step captured as a CUDA graph and replayed once per step.  The
        # timed graph has event-record nodes only at its ends (an event node
        # between two kernels costs a few microseconds); a second graph with
        # event nodes between the calls gives the per-kernel times.
        def capture(evs):
            g = torch.cuda.CUDAGraph()
            side = torch.cuda.Stream(dev)
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                with torch.cuda.graph(g, stream=side):
                    evs[0].record(side)
                    ro, cb, st = splits()
                    if len(evs) == 4:
                        evs[1].record(side)
                    fwd(ro, cb, st)
                    if len(evs) == 4:
                        evs[2].record(side)
                    bwd(ro, cb, st)
                    evs[-1].record(side)
            stream.wait_stream(side)
            torch.cuda.synchronize()
            return g

        sev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
        gev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)]
        graph = capture(sev)
        graph_parts = capture(gev)

    def timed_steps(n, record, parts=False):
        """n steps, each after an L2 flush; returns per-step [splits, fwd, bwd, total] ms
        (parts=False: the step graph, total only)."""
        out = []
        for i in range(n):
            do_flush(i)
            if args.eager:
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
                run_step(ev)
                if record:
                    out.append(ev)
            elif parts:
                graph_parts.replay()
                torch.cuda.synchronize()
                if record:
                    out.append([gev[0].elapsed_time(gev[1]), gev[1].elapsed_time(gev[2]),
                                gev[2].elapsed_time(gev[3]), gev[0].elapsed_time(gev[3])])
            else:
                graph.replay()
                torch.cuda.synchronize()
                if record:
                    out.append([None, None, None, sev[0].elapsed_time(sev[1])])
        if args.eager:
            torch.cuda.synchronize()
            out = [[e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]), e[2].elapsed_time(e[3]),
                    e[0].elapsed_time(e[3])] for e in out]
        return out

    timed_steps(args.warmup, False)
    if not args.eager:
        timed_steps(args.warmup, False, parts=True)
    torch.cuda.synchronize()
    sampler = ClockSampler(dev)
    with sampler:
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        sampler.active = True
        wall0 = time.perf_counter()
        times = timed_steps(args.steps, True)
        torch.cuda.synchronize()
        wall = time.perf_counter() - wall0
        # per-kernel times: the same steps again, with event nodes between the calls
        parts = times if args.eager else timed_steps(args.steps, True, parts=True)
        torch.cuda.synchronize()
        sampler.active = False
        if world > 1:
            torch.distributed.barrier()
    if not args.eager:
        del graph, graph_parts
    splits_ms = [t[0] for t in parts]
    fwd_ms = [t[1] for t in parts]
    bwd_ms = [t[2] for t in parts]
    total_ms = max_over_ranks(sum(t[3] for t in times), world, dev)

    # end to end through the public API with host buffers (pinned), H2D of the
    # step's inputs and D2H of every output inside the timed region
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(mg, wl, inp, dev, stream, dirs, S, args, world)

    peak, peak_kind = measured_peak()
    mean = lambda v: sum(v) / len(v)
    median = lambda v: sorted(v)[len(v) // 2]
    fwd_us, bwd_us = 1e3 * mean(fwd_ms), 1e3 * mean(bwd_ms)
    dom = "bwd" if bwd_us >= fwd_us else "fwd"
    dom_us = bwd_us if dom == "bwd" else fwd_us
    achieved = bm[dom] / (dom_us * 1e-6) / 1e9
    kname = "act_bwd_kernel" if dom == "bwd" else "act_fwd_kernel"
    # the profiled launches are the default variant (SwiGLU, halves layout,
    # row-major scales, no staged rounding); other variants report none
    default_variant = (args.act == "swiglu" and not args.staged and not args.glu_interleave
                       and args.scales == "rowmajor")
    traffic = ncu_traffic(args.workload, kname, args.dirs) if default_variant else None
    value = whole_job_gbs(world, args.steps, step_bytes, total_ms)
    out = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded torch generators; shapes and statistics of the pages' workloads)",
        "config": {"workload": f"{wl.key}: {wl.title}", "M": M, "N": N, "groups": E,
                   "dirs": args.dirs, "scales": args.scales, "activation": args.act,
                   "staged_rounding": bool(args.staged), "glu_interleave": args.glu_interleave,
                   "step": "splits_to_offsets + grouped fwd + grouped bwd (dx, dscale)",
                   "launch": "eager" if args.eager else "one CUDA graph per step (events at its ends only)",
                   "kernel_times": "eager events" if args.eager else "a second timed pass of the same steps, with event nodes between the calls",
                   "l2": "flushed before every step (256 MiB written then read), outside the timed events",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "kernel": kname, "achieved": round(achieved, 1),
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "algorithmic_bytes": bm[dom]},
        "kernels": {
            "fwd": {"us": round(fwd_us, 2), "us_median": round(1e3 * median(fwd_ms), 2),
                    "us_min": round(1e3 * min(fwd_ms), 2), "bytes": bm["fwd"],
                    "gbs": round(bm["fwd"] / (fwd_us * 1e-6) / 1e9, 1),
                    "frac": round(bm["fwd"] / (fwd_us * 1e-6) / 1e9 / peak, 4)},
            "bwd": {"us": round(bwd_us, 2), "us_median": round(1e3 * median(bwd_ms), 2),
                    "us_min": round(1e3 * min(bwd_ms), 2), "bytes": bm["bwd"],
                    "gbs": round(bm["bwd"] / (bwd_us * 1e-6) / 1e9, 1),
                    "frac": round(bm["bwd"] / (bwd_us * 1e-6) / 1e9 / peak, 4)},
            "splits_to_offsets": {"us": round(1e3 * mean(splits_ms), 2)},
        },
        "wall_s_timed_region": round(wall, 4),
        "gpu_launches": 4 * args.steps,   # splits, fwd, bwd, dscale reduction per step
        "clocks": sampler.summary(),
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(wl, dirs, budget_s=args.cpu_seconds, act=args.act,
                                           staged=args.staged)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(out))


def run_e2e(mg, wl, inp, dev, stream, dirs, S, args, world):
    """The step through the public API with host buffers: every step copies its
    inputs (X, s, dY, m_splits) from pinned host memory to the device, runs
    splits_to_offsets, the forward and the backward, and copies every output
    back to pinned host memory.  Three streams pipeline consecutive steps
    (host->device copies of step i+1 and device->host copies of step i-1 run
    while step i computes; the two copy directions use separate engines), with
    double-buffered device inputs and host outputs.  Timed from the first copy
    in to the last copy out."""
    srelu = args.act == "srelu"
    M, N = wl.M, (wl.srelu_N if srelu else wl.N)
    rw, cw = bool(dirs & 1), bool(dirs & 2)
    gemm = args.scales == "gemm"
    fwd_api, bwd_api, fwd_extra, bwd_extra = act_api(mg, args.act, args.glu_interleave,
                                                     args.staged)
    hin = [inp["x"].cpu().pin_memory(), inp["s"].cpu().pin_memory(),
           inp["dy"].cpu().pin_memory(), inp["m_splits"].clone().pin_memory()]
    h2d = sum(t.numel() * t.element_size() for t in hin)
    dbuf = [[torch.empty_like(t, device=dev) for t in hin] for _ in range(2)]
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    hout = [None, None]

    def step(i, in_free, out_free):
        """Enqueue step i; returns (inputs consumed, outputs copied) events."""
        b = i & 1
        xd, sd, dyd, md = dbuf[b]
        with torch.cuda.stream(s_in):
            if in_free[b] is not None:
                s_in.wait_event(in_free[b])
            for d, h in zip(dbuf[b], hin):
                d.copy_(h, non_blocking=True)
            loaded = torch.cuda.Event()
            loaded.record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(loaded)
            ro, cb, st = mg.splits_to_offsets(md, M)
            f, _ = fwd_api(xd, sd, ro, cb, rowwise=rw, colwise=cw, col_scale_rows=S, status=st,
                           gemm_scales=gemm, **fwd_extra)
            bw, _ = bwd_api(dyd, xd, sd, ro, cb, rowwise=rw, colwise=cw, col_scale_rows=S,
                            status=st, gemm_scales=gemm, **bwd_extra)
            outs = [t for t in (*f, *bw.mx, bw.dx, bw.dscale, st) if t is not None and t.numel()]
            done = torch.cuda.Event()
            done.record(s_comp)
        if hout[b] is None:
            hout[b] = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
        with torch.cuda.stream(s_out):
            s_out.wait_event(done)
            if out_free[b] is not None:
                s_out.wait_event(out_free[b])
            for h, t in zip(hout[b], outs):
                t.record_stream(s_out)
                h.copy_(t, non_blocking=True)
            copied = torch.cuda.Event()
            copied.record(s_out)
        return done, copied, outs

    in_free, out_free = [None, None], [None, None]
    keep = []                                  # outputs of the last steps stay referenced
    for i in range(4):                         # warm-up: host outputs, allocator pool
        in_free[i & 1], out_free[i & 1], outs = step(i, in_free, out_free)
        keep = (keep + [outs])[-2:]
    torch.cuda.synchronize()
    d2h = sum(t.numel() * t.element_size() for t in outs)
    steps = max(2, min(args.steps, 20))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0.record(s_in)
    for i in range(steps):
        in_free[i & 1], out_free[i & 1], outs = step(i, in_free, out_free)
        keep = (keep + [outs])[-2:]
    e1.record(s_out)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    E = int(inp["m_splits"].numel())
    bm = byte_model(M, N, E, dirs, srelu=srelu, S=S)
    step_bytes = bm["splits"] + bm["fwd"] + bm["bwd"]
    return {"value": round(whole_job_gbs(world, steps, step_bytes, ms), 2), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(ms / steps, 4),
            "pipeline": "copy-in / compute / copy-out streams, double-buffered"}


# ------------------------------------------------------------------ oracle timing
def _oracle_sample(wl, dirs, rows, act="swiglu"):
    """Inputs of the first `rows` rows of the workload, as numpy bit arrays."""
    from moe_gated_activation_b200.workloads import bf16_bits, make_inputs
    srelu = act == "srelu"
    N = wl.srelu_N if srelu else wl.N
    inp = make_inputs(wl, device="cpu", srelu=srelu) if wl.M * N <= (1 << 26) else None
    if inp is None:
        # large workloads: draw the same law for a sample of rows only
        from moe_gated_activation_b200.workloads import random_case
        c = random_case(rows, N, wl.seed, std=wl.x_std, width=N if srelu else 2 * N)
        return bf16_bits(c["x"]), c["s"].numpy(), bf16_bits(c["dy"])
    return (bf16_bits(inp["x"][:rows]), inp["s"][:rows].numpy().copy(),
            bf16_bits(inp["dy"][:rows]))


def _oracle_step(oracle, xb, s, dyb, N, dirs, act="swiglu", staged=False):
    if act == "clamped":
        oracle.clamped_fwd(xb, s, N, dirs)
        oracle.clamped_bwd(dyb, xb, s, N, dirs)
        return
    a = oracle.SRELU if act == "srelu" else oracle.SWIGLU
    oracle.act_fwd(xb, s, N, dirs, act=a, staged=staged)
    oracle.act_bwd(dyb, xb, s, N, dirs, act=a)


def _calibrate_rows(oracle, wl, dirs, budget_s, act="swiglu", staged=False):
    xb, s, dyb = _oracle_sample(wl, dirs, 32, act)
    N = wl.srelu_N if act == "srelu" else wl.N
    t0 = time.perf_counter()
    _oracle_step(oracle, xb, s, dyb, N, dirs, act, staged)
    per32 = max(time.perf_counter() - t0, 1e-4)
    rows = int(budget_s / per32) * 32
    return max(32, min(wl.M, rows))


def cpu_baseline(wl, dirs, budget_s=10.0, act="swiglu", staged=False):
    import oracle
    oracle.sigmoid_table()
    srelu = act == "srelu"
    N = wl.srelu_N if srelu else wl.N
    rows = _calibrate_rows(oracle, wl, dirs, budget_s, act, staged)
    xb, s, dyb = _oracle_sample(wl, dirs, rows, act)
    # whole passes over the sample until the budget is spent (a workload
    # smaller than the budget is passed over several times)
    passes = 0
    t0 = time.perf_counter()
    while True:
        _oracle_step(oracle, xb, s, dyb, N, dirs, act, staged)
        passes += 1
        dt = time.perf_counter() - t0
        if dt >= 0.9 * budget_s:
            break
    bm = byte_model(rows, N, 1, dirs, srelu=srelu)
    return {"value": round(passes * (bm["fwd"] + bm["bwd"]) / dt / 1e9, 4), "unit": "GB/s",
            "cores": 1, "kind": "oracle",
            "sample": f"rows [0, {rows}) of {wl.M} ({wl.key}) x {passes} pass(es), {act}"
                      f"{' staged' if staged else ''} forward + backward, dirs={dirs}, "
                      f"{dt:.1f} s single-threaded"}


def run_reference(args):
    from moe_gated_activation_b200.workloads import WORKLOADS
    import oracle
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    dirs = DIRS[args.dirs]
    oracle.sigmoid_table()
    per_step = min(2.0, 150.0 / max(1, args.steps + args.warmup))
    rows = _calibrate_rows(oracle, wl, dirs, per_step)
    xb, s, dyb = _oracle_sample(wl, dirs, rows)
    for _ in range(args.warmup):
        _oracle_step(oracle, xb, s, dyb, wl.N, dirs)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step(oracle, xb, s, dyb, wl.N, dirs)
    dt = time.perf_counter() - t0
    bm = byte_model(rows, wl.N, 1, dirs)
    value = args.steps * (bm["fwd"] + bm["bwd"]) / dt / 1e9
    sample = (f"rows [0, {rows}) of {wl.M} ({wl.key}) per step, forward + backward, "
              f"single-threaded C oracle")
    out = {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "impl": "reference",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(1e3 * dt / args.steps, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f32",
           "data": "synthetic (seeded torch generators)",
           "config": {"workload": f"{wl.key}: {wl.title}", "M": wl.M, "N": wl.N,
                      "groups": wl.groups, "dirs": args.dirs, "activation": "swiglu",
                      "step": "splits_to_offsets + grouped fwd + grouped bwd (dx, dscale)",
                      "parallelism": "host cores (rank 0)"},
           "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1,
                            "kind": "oracle", "sample": sample},
           "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="c2", choices=["c2", "c3", "c4", "c5"])
    ap.add_argument("--dirs", default="both", choices=list(DIRS))
    ap.add_argument("--act", default="swiglu", choices=["swiglu", "clamped", "srelu"],
                    help="activation: SwiGLU, ClampedSwiGLU (alpha 1.702, limit 7), or SReLU "
                         "(on the workload's own SReLU input; c4 has one)")
    ap.add_argument("--staged", action="store_true",
                    help="SwiGLU forward with staged rounding (silu and h rounded to bf16)")
    ap.add_argument("--scales", default="rowmajor", choices=["rowmajor", "gemm"],
                    help="E8M0 scale layout: row-major, or the GEMM-ready 128 x 4 tiles")
    ap.add_argument("--glu-interleave", type=int, default=0,
                    help="gate / up interleaved in blocks of G columns (0: [gate | up] halves)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--eager", action="store_true", help="launch eagerly instead of CUDA graphs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

"""Benchmark of the fused scaled gated activation + MXFP8 path on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
splits_to_offsets (per-expert offsets) -> grouped forward (scaled SwiGLU, MXFP8
with the requested scale directions) -> grouped backward (dgate/dup bf16, dscale,
MXFP8 of the gradient).  A single-group workload runs the same calls with one
group.  The metric is algorithmic bytes / device time (GB/s), the byte model of
the pytorch/ao PR #4743 performance table extended with the per-row scale and
the backward's bf16 dX and dscale.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c5]
                    [--dirs both|row|col] [--impl ours|reference]

The default workload is the largest single-GPU one (c5: X bf16 [131072, 16384],
32 Zipf-skewed experts).  N > 1 runs under torchrun: every rank runs its own
replica of the workload on its GPU (rows are independent; there is no exchange
step), and the device time is the max over ranks.  L2 is flushed (written then
read, 256 MiB) before every timed step, outside the timed events.
"""
from __future__ import annotations

import argparse
import hashlib
import json
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


FC2_SOURCES = ("fc2.cuh", "kern_fc2.cu")


def kernel_source_hash(kernel="act"):
    """Hash of the sources a kernel's profile depends on: the fused activation
    kernels ("act": every csrc file but the fused FC2's own) or the fused FC2
    ("fc2": its own files and the shared device helpers)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "moe_gated_activation_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if kernel == "act" and name in FC2_SOURCES:
            continue
        if kernel == "fc2" and name not in FC2_SOURCES + ("device_common.cuh", "kernels.cuh"):
            continue
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
    cur = kernel_source_hash("fc2" if kernel == "fc2_kernel" else "act")
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


# ------------------------------------------------------------------ config
def workload_config(args, wl, M, N, E, world):
    """The `config` of a bench line: the same dict for both arms."""
    return {"workload": f"{wl.key}: {wl.title}", "M": M, "N": N, "groups": E,
            "dirs": args.dirs, "scales": args.scales, "activation": args.act,
            "staged_rounding": bool(args.staged), "glu_interleave": args.glu_interleave,
            "step": "splits_to_offsets + grouped fwd + grouped bwd (dx, dscale)",
            "l2": "flushed before every timed step (256 MiB written then read), outside the "
                  "timed events",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def device_error_word():
    """The library's device error word (reading clears it): non-zero if a
    kernel gave up a bounded wait, i.e. its outputs are incomplete."""
    import ctypes
    from moe_gated_activation_b200 import _capi
    v = ctypes.c_uint32(0)
    _capi.call("moeact_device_error", ctypes.byref(v))
    return v.value


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

    # eager warm-up; the offsets of the warm-up stay for the per-kernel graphs
    for i in range(3):
        ro0, cb0, st0 = splits()
        fwd(ro0, cb0, st0)
        bwd(ro0, cb0, st0)
    torch.cuda.synchronize()
    if int(st0.item()) != 0:
        raise SystemExit(f"device status {int(st0.item())} from the warm-up step")

    def capture(body):
        """`body` captured as one CUDA graph between two event-record nodes."""
        ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                ev[0].record(side)
                out = body()
                ev[1].record(side)
        stream.wait_stream(side)
        torch.cuda.synchronize()
        return g, ev, out

    if args.eager:
        def step_body():
            ro, cb, st = splits()
            fwd(ro, cb, st)
            bwd(ro, cb, st)
            return st
        graphs = None
    else:
        # The step as one CUDA graph with event nodes only at its ends (the
        # headline); each call of the step as a graph of its own, timed the
        # same way, for the per-kernel times (an event node between two
        # kernels of one graph would add a few microseconds to each).
        def step_body():
            ro, cb, st = splits()
            fwd(ro, cb, st)
            bwd(ro, cb, st)
            return st
        graphs = {"step": capture(step_body),
                  "splits": capture(splits),
                  "fwd": capture(lambda: fwd(ro0, cb0, st0)),
                  "bwd": capture(lambda: bwd(ro0, cb0, st0))}

    def timed(name, n, record):
        """n replays of graph `name` (eager: n calls), each after an L2 flush;
        the device time of each in ms."""
        out = []
        for i in range(n):
            do_flush(i)
            if graphs is None:
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                if name == "step":
                    step_body()
                elif name == "splits":
                    splits()
                elif name == "fwd":
                    fwd(ro0, cb0, st0)
                else:
                    bwd(ro0, cb0, st0)
                e1.record(stream)
                e1.synchronize()
                ms = e0.elapsed_time(e1)
            else:
                g, ev, _ = graphs[name]
                g.replay()
                torch.cuda.synchronize()
                ms = ev[0].elapsed_time(ev[1])
            if record:
                out.append(ms)
        return out

    for name in ("step", "splits", "fwd", "bwd"):
        timed(name, args.warmup, False)
    torch.cuda.synchronize()
    sampler = ClockSampler(dev)
    with sampler:
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        sampler.active = True
        wall0 = time.perf_counter()
        times = timed("step", args.steps, True)
        torch.cuda.synchronize()
        wall = time.perf_counter() - wall0
        # per-kernel times: each call alone, the same number of replays
        parts = {k: timed(k, args.steps, True) for k in ("splits", "fwd", "bwd")}
        torch.cuda.synchronize()
        sampler.active = False
        if world > 1:
            torch.distributed.barrier()
    total_ms = max_over_ranks(sum(times), world, dev)
    # a kernel that gave up a bounded wait leaves its outputs incomplete: no number
    err = device_error_word()
    st_step = graphs["step"][2] if graphs is not None else st0
    if err != 0 or int(st_step.item()) != 0 or int(st0.item()) != 0:
        raise SystemExit(f"device error word {err:#x}, status {int(st_step.item())}: "
                         "the timed kernels did not complete their work")
    graphs = None
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    # end to end through the public API with host buffers (pinned), H2D of the
    # step's inputs and D2H of every output inside the timed region
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(mg, wl, inp, dev, dirs, S, args, world)
        if device_error_word() != 0:
            raise SystemExit("device error word set during the end-to-end run")

    peak, peak_kind = measured_peak()
    mean = lambda v: sum(v) / len(v)
    fwd_us, bwd_us = 1e3 * mean(parts["fwd"]), 1e3 * mean(parts["bwd"])
    dom = "bwd" if bwd_us >= fwd_us else "fwd"
    dom_us = bwd_us if dom == "bwd" else fwd_us
    achieved = bm[dom] / (dom_us * 1e-6) / 1e9
    kname = "act_bwd_kernel" if dom == "bwd" else "act_fwd_kernel"
    # the profiled launches are the default variant (SwiGLU, halves layout,
    # row-major scales, no staged rounding); other variants report none
    default_variant = (args.act == "swiglu" and not args.staged and not args.glu_interleave
                       and args.scales == "rowmajor")
    traffic = ncu_traffic(args.workload, kname, args.dirs) if default_variant else None

    def kstats(name):
        v = parts[name]
        us = 1e3 * mean(v)
        d = {"us": round(us, 2), "us_median": round(1e3 * statistics.median(v), 2),
             "us_min": round(1e3 * min(v), 2)}
        if name in bm and name != "splits":
            d.update(bytes=bm[name], gbs=round(bm[name] / (us * 1e-6) / 1e9, 1),
                     frac=round(bm[name] / (us * 1e-6) / 1e9 / peak, 4))
        return d

    value = whole_job_gbs(world, args.steps, step_bytes, total_ms)
    config = workload_config(args, wl, M, N, E, world)
    config.update(
        launch="eager" if args.eager else "one CUDA graph per step (event nodes at its ends only)",
        kernel_times="each call alone (its own CUDA graph, event nodes at its ends), after an "
                     "L2 flush, as many replays as timed steps; `us` is the mean, which the "
                     "roofline uses; bwd = act_bwd_kernel + dscale_reduce_kernel")
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
        "config": config,
        "roofline": {"bound": "hbm", "kernel": kname, "achieved": round(achieved, 1),
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "algorithmic_bytes": bm[dom], "time_stat": "mean"},
        "kernels": {"fwd": kstats("fwd"), "bwd": kstats("bwd"),
                    "splits_to_offsets": kstats("splits")},
        "wall_s_timed_region": round(wall, 4),
        "gpu_launches": 4 * args.steps,   # splits, fwd, bwd, dscale reduction per step
        "device_error_word": 0,
        "clocks": sampler.summary(),
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(wl, dirs, inp, budget_s=args.cpu_seconds,
                                           act=args.act, staged=args.staged)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(out))


def run_e2e(mg, wl, inp, dev, dirs, S, args, world):
    """The step through the public API with host buffers: every step copies its
    inputs (X, s, dY, m_splits) from pinned host memory to the device, runs
    splits_to_offsets, the forward and the backward, and copies every output
    back to pinned host memory.  Three streams pipeline consecutive steps
    (host->device copies of step i+1 and device->host copies of step i-1 run
    while step i computes; the two copy directions use separate engines), with
    double-buffered device inputs.  The host output buffers are double-buffered
    too when a step's outputs are small (<= 4 GiB), else shared by all steps
    (nothing reads them on the host, and the copies into them are serialised
    on one stream), which keeps pinned host memory bounded at the largest
    workloads.  Timed from the first copy in to the last copy out."""
    srelu = args.act == "srelu"
    M, N = wl.M, (wl.srelu_N if srelu else wl.N)
    rw, cw = bool(dirs & 1), bool(dirs & 2)
    gemm = args.scales == "gemm"
    fwd_api, bwd_api, fwd_extra, bwd_extra = act_api(mg, args.act, args.glu_interleave,
                                                     args.staged)

    def pinned_copy(t):
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t)
        return h

    hin = [pinned_copy(inp["x"]), pinned_copy(inp["s"]), pinned_copy(inp["dy"]),
           inp["m_splits"].clone().pin_memory()]
    h2d = sum(t.numel() * t.element_size() for t in hin)
    dbuf = [[torch.empty_like(t, device=dev) for t in hin] for _ in range(2)]
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    hout = [None, None]
    shared_out = [False]

    def step(i, in_free, out_free):
        """Enqueue step i; returns (outputs computed, outputs copied) events."""
        b = i & 1
        with torch.cuda.stream(s_in):
            if in_free[b] is not None:
                s_in.wait_event(in_free[b])
            for d, h in zip(dbuf[b], hin):
                d.copy_(h, non_blocking=True)
            loaded = torch.cuda.Event()
            loaded.record(s_in)
        xd, sd, dyd, md = dbuf[b]
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
        if hout[0] is None:
            nbytes = sum(t.numel() * t.element_size() for t in outs)
            shared_out[0] = nbytes > (4 << 30)
            hout[0] = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
            hout[1] = hout[0] if shared_out[0] else \
                [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
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
    for i in range(3):                         # warm-up: host outputs, allocator pool
        in_free[i & 1], out_free[i & 1], outs = step(i, in_free, out_free)
        keep = (keep + [outs])[-2:]
    torch.cuda.synchronize()
    d2h = sum(t.numel() * t.element_size() for t in outs)
    # a bounded number of steps (at the largest workload a step moves ~17 GB
    # over PCIe)
    steps = max(2, min(args.steps, 20 if d2h + h2d <= (4 << 30) else 6))
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
    pipe = "copy-in / compute / copy-out streams, double-buffered device inputs, " + \
        ("one host output buffer for all steps" if shared_out[0] else
         "double-buffered host outputs")
    return {"value": round(whole_job_gbs(world, steps, step_bytes, ms), 2), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(ms / steps, 4), "pipeline": pipe}


# ------------------------------------------------------------------ activation -> FC2
def measured_bf16_tflops():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured"
    except Exception:  # noqa: BLE001
        return 1590.0, "fallback"


def run_fc2(args):
    """The activation -> MXFP8 -> expert FC2 GEMM fused on the tensor cores
    (grouped_scaled_swiglu_mxfp8_fc2) on the Qwen3-MoE-like workload c3
    (65536 routed rows over 128 experts, N = 768) into an FC2 of width
    --fc2-width (the model's hidden size, 2048), with a seeded MXFP8 weight.
    One step = one launch (its own CUDA graph, event nodes at its ends) after
    an L2 flush.  Reports TFLOP/s against the fp8 dense peak (twice the
    measured bf16 GEMM peak: the tensor cores' fp8 rate is twice their bf16
    rate) and the HBM bytes of the launch against the copy peak; `saved_bytes`
    is the traffic of the quantized activation an unfused path would write
    and read back (codes + rowwise scales, twice)."""
    import moe_gated_activation_b200 as mg
    from moe_gated_activation_b200.workloads import WORKLOADS, fc2_weights, make_inputs

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    mg.init()
    wl = WORKLOADS["c3"]
    inp = make_inputs(wl, device=dev, with_dy=False)
    x, s, m = inp["x"], inp["s"], inp["m_splits"]
    M, N, H, E = wl.M, wl.N, args.fc2_width, int(m.numel())
    # uniform random code and scale bytes: the same law in any layout, so
    # they serve as the tiled weight codes and scales the kernel reads
    # without a conversion
    wc, ws = fc2_weights(E, H, N, 11, device=dev)
    ro, _, st = mg.splits_to_offsets(m.to(dev), M)
    out = torch.empty(M, H, dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def call():
        mg.grouped_scaled_swiglu_mxfp8_fc2(x, s, ro, wc, ws, status=st, out=out)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    if int(st.item()) != 0:
        raise SystemExit(f"device status {int(st.item())}")
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            ev[0].record(side)
            call()
            ev[1].record(side)
    stream.wait_stream(side)
    torch.cuda.synchronize()

    def timed(n):
        t = []
        for i in range(n):
            flush.fill_(float(i & 7))
            flush.amax()
            g.replay()
            torch.cuda.synchronize()
            t.append(ev[0].elapsed_time(ev[1]))
        return t

    timed(args.warmup)
    sampler = ClockSampler(dev)
    with sampler:
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        sampler.active = True
        times = timed(args.steps)
        sampler.active = False
        if world > 1:
            torch.distributed.barrier()
    err = device_error_word()
    if err != 0 or int(st.item()) != 0:
        raise SystemExit(f"device error word {err:#x}, status {int(st.item())}")
    total_ms = max_over_ranks(sum(times), world, dev)
    ms = total_ms / args.steps
    flops = 2.0 * M * N * H
    nonempty = int((m > 0).sum())
    hbm_bytes = 2 * M * 2 * N + 4 * M + nonempty * H * (N + N // 32) + 2 * M * H
    saved = 2 * (M * N + M * N // 32)
    bf16, kind = measured_bf16_tflops()
    fp8_peak = 2.0 * bf16
    hbm_peak, hbm_kind = measured_peak()
    tflops = world * args.steps * flops / (total_ms * 1e-3) / 1e12
    gbs = hbm_bytes / (ms * 1e-3) / 1e9
    bound = "tensor" if flops / (fp8_peak * 1e12) >= hbm_bytes / (hbm_peak * 1e9) else "hbm"
    tensor_rf = {"achieved": round(tflops, 1), "peak": round(fp8_peak, 1),
                 "peak_kind": f"2 x {kind} bf16 GEMM peak", "unit": "TFLOP/s",
                 "frac": round(tflops / fp8_peak, 4)}
    hbm_rf = {"achieved": round(gbs, 1), "peak": hbm_peak, "peak_kind": hbm_kind, "unit": "GB/s",
              "frac": round(gbs / hbm_peak, 4), "algorithmic_bytes": hbm_bytes}
    outd = {
        "metric": "fused act+MXFP8+FC2 grouped GEMM TFLOP/s (tcgen05, block-scaled E4M3)",
        "value": round(tflops, 1), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 x e4m3 -> f32 (bf16 out)",
        "data": "synthetic (seeded torch generators; c3 activation input, uniform MXFP8 weight)",
        "config": {"workload": f"c3 -> FC2: {wl.title}, FC2 width {H}", "M": M, "N": N, "H": H,
                   "groups": E, "kernel": "grouped_scaled_swiglu_mxfp8_fc2",
                   "l2": "flushed before every launch (256 MiB written then read)",
                   "launch": "one CUDA graph per launch (event nodes at its ends)"},
        # the roofline's own unit at the top level (the bound with the larger
        # floor), the other bound nested beside it
        "roofline": dict(
            {"bound": bound, "kernel": "fc2_kernel"},
            **(tensor_rf if bound == "tensor" else hbm_rf),
            **{("hbm" if bound == "tensor" else "tensor"): (hbm_rf if bound == "tensor"
                                                            else tensor_rf)},
            traffic=ncu_traffic("c3", "fc2_kernel", f"H{H}"), time_stat="mean"),
        "saved_bytes": saved,
        "us_median": round(1e3 * statistics.median(times), 2),
        "us_min": round(1e3 * min(times), 2),
        "gpu_launches": args.steps,
        "clocks": sampler.summary(),
    }
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(outd))


# ------------------------------------------------------------------ oracle timing
def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def _oracle_rows(x, s, dy, rows):
    """The first `rows` rows of the inputs (torch tensors on any device), as
    numpy bit arrays for the oracle."""
    from moe_gated_activation_b200.workloads import bf16_bits
    return (bf16_bits(x[:rows]), s[:rows].cpu().numpy().copy(), bf16_bits(dy[:rows]))


def _oracle_step(oracle, xb, s, dyb, N, dirs, act="swiglu", staged=False):
    if act == "clamped":
        oracle.clamped_fwd(xb, s, N, dirs)
        oracle.clamped_bwd(dyb, xb, s, N, dirs)
        return
    a = oracle.SRELU if act == "srelu" else oracle.SWIGLU
    oracle.act_fwd(xb, s, N, dirs, act=a, staged=staged)
    oracle.act_bwd(dyb, xb, s, N, dirs, act=a)


class OraclePool:
    """The oracle over independent 32-row slabs on `cores` host threads: the
    sample's rows are cut into one chunk of whole 32-row slabs per thread
    (a slab is a complete set of colwise blocks, so each chunk is a complete
    problem), and each thread runs the oracle's forward and backward on its
    chunk.  The oracle's C calls release the interpreter lock, so the threads
    run in parallel; the oracle itself is unchanged (single-threaded per
    call)."""

    def __init__(self, oracle, xb, s, dyb, N, dirs, act, staged, cores):
        import concurrent.futures
        rows = xb.shape[0]
        n = max(1, min(cores, rows // 32))
        per = (rows // 32 + n - 1) // n * 32
        self.chunks = [(xb[i:i + per], s[i:i + per], dyb[i:i + per])
                       for i in range(0, rows, per)]
        self.threads = len(self.chunks)
        self.ex = concurrent.futures.ThreadPoolExecutor(self.threads)
        self.args = (oracle, N, dirs, act, staged)

    def step(self):
        oracle, N, dirs, act, staged = self.args
        futs = [self.ex.submit(_oracle_step, oracle, xb, s, dyb, N, dirs, act, staged)
                for xb, s, dyb in self.chunks]
        for f in futs:
            f.result()

    def close(self):
        self.ex.shutdown()


def _sample_rows(oracle, x, s, dy, N, dirs, seconds, cores, M, act="swiglu", staged=False):
    """Rows of a sample the oracle passes over in about `seconds` on `cores`
    threads: single-thread time of 32 rows, scaled by the thread count;
    whole 32-row slabs, at least one per thread where the workload has them,
    at most 2^28 input elements (host memory)."""
    xb, sv, dyb = _oracle_rows(x, s, dy, 32)
    t0 = time.perf_counter()
    _oracle_step(oracle, xb, sv, dyb, N, dirs, act, staged)
    per32 = max(time.perf_counter() - t0, 1e-4)
    rows = int(seconds * cores / per32) * 32
    cap = max(32, ((1 << 28) // max(1, x.shape[1])) // 32 * 32)
    return max(32, min(M, rows, cap))


def cpu_baseline(wl, dirs, inp, budget_s=10.0, act="swiglu", staged=False):
    """The oracle on the first rows of the GPU arm's own inputs, on every host
    core, for about `budget_s` seconds."""
    import oracle
    oracle.sigmoid_table()
    srelu = act == "srelu"
    N = wl.srelu_N if srelu else wl.N
    cores = host_cores()
    rows = _sample_rows(oracle, inp["x"], inp["s"], inp["dy"], N, dirs, budget_s / 2, cores,
                        wl.M, act, staged)
    xb, s, dyb = _oracle_rows(inp["x"], inp["s"], inp["dy"], rows)
    pool = OraclePool(oracle, xb, s, dyb, N, dirs, act, staged, cores)
    # whole passes over the sample until the budget is spent (a workload
    # smaller than the budget is passed over several times)
    passes = 0
    t0 = time.perf_counter()
    while True:
        pool.step()
        passes += 1
        dt = time.perf_counter() - t0
        if dt >= 0.9 * budget_s:
            break
    pool.close()
    bm = byte_model(rows, N, 1, dirs, srelu=srelu)
    return {"value": round(passes * (bm["fwd"] + bm["bwd"]) / dt / 1e9, 4), "unit": "GB/s",
            "cores": pool.threads, "host_cores": cores, "kind": "oracle",
            "sample": f"rows [0, {rows}) of {wl.M} ({wl.key}, the timed arm's own inputs) x "
                      f"{passes} pass(es), {act}{' staged' if staged else ''} forward + "
                      f"backward, dirs={dirs}, {dt:.1f} s on {pool.threads} threads "
                      f"(32-row slabs)"}


def run_reference(args):
    """The reference arm: the C oracle (the only runnable definition of the
    method; the pages hold no implementation) on the machine's host cores, over
    a bounded sample of the workload's rows per step."""
    from moe_gated_activation_b200.workloads import WORKLOADS, make_inputs
    import oracle
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    dirs = DIRS[args.dirs]
    srelu = args.act == "srelu"
    N = wl.srelu_N if srelu else wl.N
    # the same seeded inputs as the GPU arm (drawn on the GPU when there is one)
    gen_dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = make_inputs(wl, device=gen_dev, srelu=srelu)
    E = int(inp["m_splits"].numel())
    oracle.sigmoid_table()
    cores = host_cores()
    per_step = min(2.0, 150.0 / max(1, args.steps + args.warmup))
    rows = _sample_rows(oracle, inp["x"], inp["s"], inp["dy"], N, dirs, per_step, cores, wl.M,
                        args.act, args.staged)
    xb, s, dyb = _oracle_rows(inp["x"], inp["s"], inp["dy"], rows)
    del inp
    pool = OraclePool(oracle, xb, s, dyb, N, dirs, args.act, args.staged, cores)
    for _ in range(args.warmup):
        pool.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        pool.step()
    dt = time.perf_counter() - t0
    pool.close()
    bm = byte_model(rows, N, 1, dirs, srelu=srelu)
    value = args.steps * (bm["fwd"] + bm["bwd"]) / dt / 1e9
    sample = (f"rows [0, {rows}) of {wl.M} ({wl.key}) per step, forward + backward, C oracle "
              f"on {pool.threads} host threads (32-row slabs)")
    out = {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "impl": "reference",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(1e3 * dt / args.steps, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f32",
           "data": "synthetic (seeded torch generators; shapes and statistics of the pages' "
                   "workloads)",
           "config": workload_config(args, wl, wl.M, N, E, 1),
           "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": pool.threads,
                            "host_cores": cores, "kind": "oracle", "sample": sample},
           "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="c5", choices=["c2", "c3", "c4", "c5"])
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
    ap.add_argument("--fc2", action="store_true",
                    help="time the activation -> MXFP8 -> FC2 GEMM fused on the tensor cores "
                         "(workload c3) instead of the activation path")
    ap.add_argument("--fc2-width", type=int, default=2048,
                    help="FC2 output width (the model's hidden size) for --fc2")
    args = ap.parse_args()
    if args.warmup < 3:
        # Fewer than three untimed steps leaves clocks and caches cold; run
        # three and report the count actually run in the JSON line.
        print(f"--warmup {args.warmup} raised to 3", file=sys.stderr)
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.fc2:
        run_fc2(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

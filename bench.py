"""Benchmark of the fused all-reduce + residual-add + RMSNorm (+FP8) epilogue.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl far|reference]

One step = one call of the whole epilogue (W-partial reduce, residual add and
new-residual write, mean square, normalise with gamma, FP8 quantisation) over
one batch of synthetic rows.  The headline workload is the prefill one: W=4
partials of 8192 x 8192 bf16 (1% outlier rows x50), residual N(0,2),
eps=1e-5, static per-tensor FP8 with scale 0.05, the new residual and the FP8
codes written (norm_out not requested).

The metric is achieved HBM GB/s of algorithmic bytes (W*T*H*2 partials +
T*H*2 residual in + H*2 gamma + T*H*2 residual out + T*H FP8 codes [+ 4T
scales] [+ T*H*2 norm_out]) and its fraction of the measured HBM peak;
tokens/s is reported beside it.  Inputs (640 MiB read per step) are larger
than the 126 MB L2, so nothing stays cached between steps.

Under torchrun (N > 1) every rank runs its own batch of rows (the rows are
independent: weak scaling, no collective on the data path); the time is the
max over ranks and `value` counts every rank's bytes.  `--impl reference`
times the CPU fp64 oracle on a bounded sample of the same workload (rank 0).
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

from reduce_residual_add_b200.inputs import WORKLOADS, Workload, as_u16, make_inputs  # noqa: E402

HEADLINE = "c4_prefill_fp8_static"
METRIC = "achieved HBM GB/s (% of B200 peak) and tokens/s of fused reduce+add+RMSNorm(+FP8)"
L2_BYTES = 126 * 10 ** 6  # B200 L2 capacity
FALLBACK_HBM_GBS = 6650.0


def algorithmic_bytes(wl: Workload, rows: int, with_norm: bool) -> int:
    T, H, W = rows, wl.H, wl.W
    b = W * T * H * 2 + H * 2
    if wl.has_residual:
        b += T * H * 2          # residual in
    b += T * H * 2              # new residual out
    if with_norm:
        b += T * H * 2
    if wl.pattern in (1, 2, 3, 4):
        b += T * H             # e4m3 codes
    if wl.pattern == 2:
        b += 4 * T             # per-token scales
    if wl.pattern == 3:
        b += 4                 # the one per-tensor scale
    if wl.pattern == 4:
        b += 4 * T * (H // wl.group_size)   # per-group scales
    return b


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML: read-only queries)
# ---------------------------------------------------------------------------

REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
           0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
           0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
           0x100: "display_clock_setting"}


class ClockSampler(threading.Thread):
    """NVML SM clock and clock-event reasons, sampled from a thread while the
    timed region runs (every `period_s`, the reasons every few samples), plus
    one sample taken as the region ends."""
    def __init__(self, device: int, period_s: float = 0.0002):
        super().__init__(daemon=True)
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._halt = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            idx = device
            try:
                idx = torch.cuda._get_nvml_device_index(device)
            except Exception:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES")
                if vis:
                    idx = int(vis.split(",")[device])
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def run(self):
        if not self.ok:
            return
        i = 0
        while not self._halt.is_set():
            self._sample(reasons=(i % 5 == 0))
            i += 1
            time.sleep(self.period)

    def _sample(self, reasons: bool = True):
        nv = self.nv
        try:
            self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
            if reasons:
                try:
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except AttributeError:
                    r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.reasons |= int(r) & ~0x1
        except Exception:
            pass

    def stop(self) -> dict:
        self._halt.set()
        if self.is_alive():
            self.join(timeout=2)
        if self.ok:
            self._sample()  # the state as the timed region ends
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": [n for b, n in REASONS.items() if self.reasons & b],
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------

def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device="cuda") -> float:
    """The largest value over ranks (the slowest rank's time)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int, device="cuda") -> float:
    """The total over ranks (bytes and rows of every rank)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------------------
# the oracle on host cores (CPU baseline and reference arm)
# ---------------------------------------------------------------------------

def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_threads(wl: Workload, rows: int, want: int) -> int:
    """Threads the oracle can use on `rows` rows: rows are independent except
    under per-tensor FP8, whose one scale spans all rows of the call."""
    return 1 if wl.pattern == 3 else max(1, min(want, rows))


def oracle_rate(wl: Workload, inp: dict, rows: int, with_norm: bool, threads: int = 1):
    """Run the fp64 oracle on the first `rows` rows, as `threads` contiguous
    row ranges side by side (the oracle is a C library called through
    ctypes, which releases the GIL during the call); return (seconds, bytes)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    threads = oracle_threads(wl, rows, threads)
    bounds = [rows * i // threads for i in range(threads + 1)]
    jobs = []
    for b, e in zip(bounds[:-1], bounds[1:]):
        ps = [as_u16(p[b:e]) for p in inp["partials"]]
        res = None if inp["residual"] is None else as_u16(inp["residual"][b:e])
        jobs.append((ps, res))
    gam = as_u16(inp["gamma"])
    oracle.lib()

    def run(job):
        oracle.fused(job[0], job[1], gam, wl.dtype, wl.eps, wl.weight_bias, wl.pattern,
                     scale_in=wl.static_scale, want_norm=with_norm, group=wl.group_size)

    t0 = time.perf_counter()
    if threads == 1:
        run(jobs[0])
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(run, jobs))
    dt = time.perf_counter() - t0
    return dt, algorithmic_bytes(wl, rows, with_norm)


def cpu_baseline(wl: Workload, inp: dict, with_norm: bool, budget_s: float = 8.0) -> dict:
    """The oracle on this host: on every allowed core (the reported value)
    and single-threaded, each on a sample of about `budget_s` seconds of
    CPU work."""
    t1, _ = oracle_rate(wl, inp, 64, with_norm)
    per_row = max(t1 / 64, 1e-9)
    rows1 = int(min(wl.T, max(64, budget_s / per_row)))
    dt1, b1 = oracle_rate(wl, inp, rows1, with_norm)
    cores = host_cores()
    rows = int(min(wl.T, max(64, budget_s * 2 / per_row)))
    used = oracle_threads(wl, rows, cores)
    dt, b = oracle_rate(wl, inp, rows, with_norm, used)
    return {"value": round(b / dt / 1e9, 4), "unit": "GB/s", "cores": used, "kind": "oracle",
            "sample": "first %d of %d rows of %s, C fp64 oracle on %d threads (one contiguous "
                      "row range each), %.2f s" % (rows, wl.T, wl.name, used, dt),
            "tokens_per_s": round(rows / dt, 2),
            "single_thread": {"value": round(b1 / dt1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                              "sample": "first %d rows, %.1f s" % (rows1, dt1),
                              "tokens_per_s": round(rows1 / dt1, 2)}}


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------

class Case:
    """Device buffers of one workload and a closure that launches one step."""

    def __init__(self, ctx, wl: Workload, inp: dict, device, with_norm: bool, stream):
        from reduce_residual_add_b200 import far
        self.far = far
        self.ctx, self.wl, self.with_norm, self.stream = ctx, wl, with_norm, stream
        T, H = wl.T, wl.H
        self.ps = [p.to(device) for p in inp["partials"]]
        self.res = None if inp["residual"] is None else inp["residual"].to(device)
        self.gam = inp["gamma"].to(device)
        dt = wl.torch_dtype
        self.rout = torch.empty(T, H, dtype=dt, device=device)
        self.nout = torch.empty(T, H, dtype=dt, device=device) if (with_norm or wl.pattern == 0) else None
        self.qout = torch.empty(T, H, dtype=torch.uint8, device=device) if wl.pattern else None
        n_scales = {2: T, 3: 1, 4: T * (H // wl.group_size if wl.group_size else 1)}.get(wl.pattern, 0)
        self.sout = (torch.empty(n_scales, dtype=torch.float32, device=device)
                     if wl.pattern in (2, 3, 4) else None)
        self.ws = (torch.empty(far.far_fp8_tensor_workspace_bytes(T), dtype=torch.uint8, device=device)
                   if wl.pattern == 3 else None)
        self.sin = (torch.tensor([wl.static_scale], dtype=torch.float32, device=device)
                    if wl.pattern == 1 else None)
        self.bytes = algorithmic_bytes(wl, T, self.nout is not None)
        self.median_launch = 0.0  # of the last time_steps(per_launch=True)

    def prepared(self):
        """The same step as a far.FarCall (arguments marshalled once)."""
        return self.far.FarCall(self.ctx, self.ps, self.res, self.gam, self.wl.eps,
                                self.wl.weight_bias, self.wl.pattern, residual_out=self.rout,
                                norm_out=self.nout, quant_out=self.qout, scale_in=self.sin,
                                scale_out=self.sout, stream=self.stream)

    def step(self):
        if self.wl.pattern == 4:
            self.far.far_fused_fp8_group(self.ctx, self.ps, self.res, self.gam, self.wl.eps,
                                         self.wl.weight_bias, group_size=self.wl.group_size,
                                         quant_out=self.qout, scale_out=self.sout,
                                         residual_out=self.rout, norm_out=self.nout,
                                         stream=self.stream)
            return
        if self.wl.pattern == 3:
            self.far.far_fused_fp8_tensor(self.ctx, self.ps, self.res, self.gam, self.wl.eps,
                                          self.wl.weight_bias, quant_out=self.qout,
                                          scale_out=self.sout, workspace=self.ws,
                                          residual_out=self.rout, norm_out=self.nout,
                                          stream=self.stream)
            return
        self.far.far_fused(self.ctx, self.ps, self.res, self.gam, self.wl.eps,
                           self.wl.weight_bias, self.wl.pattern, residual_out=self.rout,
                           norm_out=self.nout, quant_out=self.qout, scale_in=self.sin,
                           scale_out=self.sout, stream=self.stream)

    def time_steps(self, k: int, warmup: int, per_launch: bool = True, prepared: bool = False):
        """(total seconds for k back-to-back steps, mean per-launch seconds).
        prepared: launch through a far.FarCall (arguments marshalled once), for
        calls short enough that the binding's per-call marshalling would leave
        the GPU idle between the events."""
        s = self.stream
        step = self.prepared() if prepared else self.step
        for _ in range(warmup):
            step()
        torch.cuda.synchronize()
        if k == 0:
            return 0.0, 0.0
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(k)] if per_launch else None
        first, last = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        first.record(s)
        for i in range(k):
            if per_launch:
                ev[i][0].record(s)
            step()
            if per_launch:
                ev[i][1].record(s)
        last.record(s)
        torch.cuda.synchronize()
        total = first.elapsed_time(last) / 1e3
        if per_launch:
            times = [a.elapsed_time(b) / 1e3 for a, b in ev]
            mean = sum(times) / k
            self.median_launch = statistics.median(times)
        else:
            mean = total / k
        return total, mean


def replay_time(g, s, launches: int, reps: int, warm_s: float = 0.02) -> float:
    """Seconds per launch of a captured graph of `launches` calls: untimed
    replays for at least `warm_s` (clocks ramp up after the host-side set-up
    left the GPU idle), then the median of `reps` replays each timed alone."""
    t0 = time.perf_counter()
    n = 0
    while n < 2 or time.perf_counter() - t0 < warm_s:
        with torch.cuda.stream(s):      # replay() launches on the current stream
            g.replay()
        torch.cuda.synchronize()
        n += 1
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    with torch.cuda.stream(s):
        for a, b in ev:
            a.record(s)
            g.replay()
            b.record(s)
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in ev) / 1e3 / launches


def graph_time(case: Case, launches: int, reps: int = 7) -> float:
    """Seconds per launch inside a CUDA graph of `launches` calls on one
    input set (median replay)."""
    s = case.stream
    g = torch.cuda.CUDAGraph()
    case.step()
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=s):
        for _ in range(launches):
            case.step()
    t = replay_time(g, s, launches, reps)
    del g
    return t


def touched_bytes(wl: Workload, with_norm: bool) -> int:
    """Bytes one call reads and writes at its own addresses (gamma aside)."""
    return algorithmic_bytes(wl, wl.T, with_norm) - wl.H * 2


class RotatingSets:
    """`n` copies of one workload's inputs and outputs at distinct addresses,
    enough that one pass over them touches more than `min_bytes` (2x L2):
    a loop over the sets finds none of a set's bytes left in L2 from its
    previous use, as a decode step whose partials come fresh from a GEMM
    would.  Gamma is shared (one weight vector).  Every set holds the same
    seeded values, so any set's outputs are the workload's outputs."""

    def __init__(self, ctx, wl: Workload, inp: dict, device, with_norm: bool, stream,
                 min_bytes: int = 2 * L2_BYTES):
        from reduce_residual_add_b200 import far
        T, H, W = wl.T, wl.H, wl.W
        with_norm = with_norm or wl.pattern == 0
        self.n = max(2, -(-min_bytes // touched_bytes(wl, with_norm)))
        n_in = W + (1 if wl.has_residual else 0)
        dt = wl.torch_dtype
        self.inputs = torch.empty(self.n, n_in, T, H, dtype=dt, device=device)
        src = torch.stack(list(inp["partials"]) + ([inp["residual"]] if wl.has_residual else []))
        self.inputs.copy_(src.to(device).unsqueeze(0).expand_as(self.inputs))
        self.rout = torch.empty(self.n, T, H, dtype=dt, device=device)
        self.nout = torch.empty(self.n, T, H, dtype=dt, device=device) if with_norm else None
        self.qout = torch.empty(self.n, T, H, dtype=torch.uint8, device=device) if wl.pattern else None
        self.sout = (torch.empty(self.n, T, dtype=torch.float32, device=device)
                     if wl.pattern == 2 else None)
        self.gam = inp["gamma"].to(device)
        self.sin = (torch.tensor([wl.static_scale], dtype=torch.float32, device=device)
                    if wl.pattern == 1 else None)
        self.stream = stream
        self.calls = []
        for i in range(self.n):
            ps = [self.inputs[i, r] for r in range(W)]
            res = self.inputs[i, W] if wl.has_residual else None
            self.calls.append(far.FarCall(
                ctx, ps, res, self.gam, wl.eps, wl.weight_bias, wl.pattern,
                residual_out=self.rout[i], norm_out=None if self.nout is None else self.nout[i],
                quant_out=None if self.qout is None else self.qout[i], scale_in=self.sin,
                scale_out=None if self.sout is None else self.sout[i], stream=stream))

    def graph_time(self, min_launches: int = 200, reps: int = 5) -> float:
        """Seconds per call in a CUDA graph that cycles through the sets (at
        least `min_launches` calls and at least one full cycle; median
        replay)."""
        launches = max(min_launches, self.n)
        launches = -(-launches // self.n) * self.n
        s = self.stream
        for c in self.calls:
            c()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for i in range(launches):
                self.calls[i % self.n]()
        t = replay_time(g, s, launches, reps)
        del g
        return t


def e2e_time(case: Case, inp: dict, steps: int, chunk_rows: int = 0):
    """Through the public API from pinned host memory: every step copies the
    inputs host->device, runs the epilogue and copies the outputs back.
    far_fused_host does it in chunks of rows whose copies overlap the
    kernels; per-tensor FP8 (one scale over every row: no chunks) copies
    everything in, calls far_fused_fp8_tensor and copies everything out."""
    far, wl, s = case.far, case.wl, case.stream
    h_ps = [p.pin_memory() for p in inp["partials"]]
    h_res = None if inp["residual"] is None else inp["residual"].pin_memory()
    h_gam = inp["gamma"].pin_memory()
    h_rout = torch.empty(case.rout.shape, dtype=case.rout.dtype).pin_memory()
    h_q = torch.empty(case.qout.shape, dtype=torch.uint8).pin_memory() if case.qout is not None else None
    h_s = torch.empty(case.sout.shape, dtype=torch.float32).pin_memory() if case.sout is not None else None
    h_n = torch.empty(case.nout.shape, dtype=case.nout.dtype).pin_memory() if case.nout is not None else None
    h_sin = torch.tensor([wl.static_scale], dtype=torch.float32) if wl.pattern == 1 else None
    h2d = sum(p.numel() * 2 for p in h_ps) + (h_res.numel() * 2 if h_res is not None else 0) + \
        h_gam.numel() * 2 + (4 if h_sin is not None else 0)
    d2h = h_rout.numel() * 2 + (h_q.numel() if h_q is not None else 0) + \
        (h_s.numel() * 4 if h_s is not None else 0) + (h_n.numel() * 2 if h_n is not None else 0)
    mode = "far_fused_host, chunks of %s rows" % (chunk_rows or "the default")

    if wl.pattern == 3:
        mode = "copies in, far_fused_fp8_tensor, copies out"

        def one():
            with torch.cuda.stream(s):
                for d, h in zip(case.ps, h_ps):
                    d.copy_(h, non_blocking=True)
                if h_res is not None:
                    case.res.copy_(h_res, non_blocking=True)
                case.gam.copy_(h_gam, non_blocking=True)
                case.step()
                h_rout.copy_(case.rout, non_blocking=True)
                h_q.copy_(case.qout, non_blocking=True)
                h_s.copy_(case.sout, non_blocking=True)
                if h_n is not None:
                    h_n.copy_(case.nout, non_blocking=True)
    else:
        H = wl.H
        staging = torch.empty(far.far_host_staging_bytes(wl.W, H, chunk_rows), dtype=torch.uint8,
                              device=case.rout.device)
        h_flat = None if h_s is None else h_s.view(-1)

        def one():
            far.far_fused_host(case.ctx, h_ps, h_res, h_gam, wl.eps, wl.weight_bias, wl.pattern,
                               staging=staging, chunk_rows=chunk_rows, group_size=wl.group_size,
                               residual_out=h_rout, norm_out=h_n, quant_out=h_q, scale_in=h_sin,
                               scale_out=h_flat, stream=s)

    one()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s)
    for _ in range(steps):
        one()
    b.record(s)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / 1e3 / steps, h2d, d2h, mode


def code_tokens(src: str) -> str:
    """C/C++ source without its comments, whitespace runs collapsed: what the
    compiler sees, so that editing a comment keeps a measurement valid."""
    import re
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":                      # string or character literal
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            out.append(" ")
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return re.sub(r"\s+", " ", "".join(out)).strip()


def kernel_source_hash() -> str:
    """sha256 of the kernels' code (far_kernels.cu and far_internal.h without
    comments); the committed DRAM traffic is valid only for this hash."""
    h = hashlib.sha256()
    for f in ("far_kernels.cu", "far_internal.h"):
        with open(os.path.join(ROOT, "reduce_residual_add_b200", "csrc", f)) as fh:
            h.update(code_tokens(fh.read()).encode())
    return h.hexdigest()


def profiled_traffic(workload: str):
    """Per-launch DRAM bytes of the kernel from the committed ncu summary,
    or None when the kernel source changed since it was captured."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[workload]
        if e.get("source_sha256") != kernel_source_hash():
            return None
        return int(e["traffic_bytes_per_launch"])
    except Exception:
        return None


PATTERN_NAMES = {0: "ar_residual_rmsnorm", 1: "fp8_static", 2: "fp8_per_token",
                 3: "fp8_per_tensor", 4: "fp8_per_group"}


def l2_note(wl: Workload) -> str:
    read = (wl.W + (1 if wl.has_residual else 0)) * wl.T * wl.H * 2
    if read > L2_BYTES:
        return "inputs larger than L2 (%d MiB read per step vs 126 MB L2); no flush" % (read // 2 ** 20)
    return ("inputs fit in L2 (%d MiB read per step vs 126 MB L2): an L2-resident, "
            "latency-bound case" % (read // 2 ** 20))


def workload_config(wl: Workload, bytes_per_step: int, with_norm: bool, world: int) -> dict:
    """The bench line's `config` object for one workload (the same object in
    the CUDA arm and the reference arm; the launch geometry is reported
    under `roofline`)."""
    cfg = {"workload": wl.name, "W": wl.W, "T": wl.T, "H": wl.H, "dtype": wl.dtype,
           "arithmetic": "fp32 accumulation; bf16/fp16 in and out; e4m3 codes",
           "pattern": PATTERN_NAMES[wl.pattern], "norm_out": with_norm, "eps": wl.eps,
           "weight_bias": wl.weight_bias, "static_scale": wl.static_scale,
           "bytes_per_step": bytes_per_step, "rows_per_rank": wl.T,
           "l2": l2_note(wl),
           "parallelism": "rows sharded across %d rank(s), no collective" % world}
    if wl.pattern == 4:
        cfg["group_size"] = wl.group_size
    return cfg


def run_far(args, world, rank, local):
    from reduce_residual_add_b200 import build as fbuild
    from reduce_residual_add_b200 import far
    fbuild.build()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    wl = WORKLOADS[args.workload]
    if args.rows:
        wl = wl.with_(T=args.rows, outlier_frac=wl.outlier_frac)
    if args.shape:
        W, H = (int(x) for x in args.shape.split(","))
        wl = wl.with_(name="%s_W%d_H%d" % (wl.name, W, H), W=W, H=H)
    # each rank owns an independent batch of rows (seed offset by rank)
    inp = make_inputs(wl.with_(seed=wl.seed + 1000 * rank))
    stream = torch.cuda.Stream(device=device)
    ctx = far.FarContext(local)
    case = Case(ctx, wl, inp, device, args.with_norm, stream)
    launch = far.far_describe_launch(ctx, wl.T, wl.H, wl.torch_dtype, wl.W, wl.has_residual,
                                     case.nout is not None, pattern=wl.pattern)

    case.time_steps(0, args.warmup, per_launch=False)
    barrier(world)
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    total, mean_launch = case.time_steps(args.steps, 0, per_launch=True)
    clocks = sampler.stop()
    barrier(world)
    total_max = max_over_ranks(total, world)
    bytes_all = sum_over_ranks(float(case.bytes) * args.steps, world)
    rows_all = sum_over_ranks(float(wl.T) * args.steps, world)

    value = bytes_all / total_max / 1e9
    peak, peak_kind = hbm_peak()
    # the roofline takes the median launch (robust to the odd launch that
    # waits on something else); the mean is reported beside it
    achieved = case.bytes / case.median_launch / 1e9
    achieved_mean = case.bytes / mean_launch / 1e9
    e2e_s, h2d, d2h, e2e_mode = e2e_time(case, inp, args.e2e_steps, args.e2e_chunk_rows)
    e2e_s = max_over_ranks(e2e_s, world)

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_max / args.steps * 1e3, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": workload_config(wl, case.bytes, case.nout is not None, world),
        "tokens_per_s": round(rows_all / total_max, 1),
        "pct_of_peak": round(100 * value / world / peak, 2),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "peak_source": "%s (MEASURED_PEAKS.json hbm_gbs)" % peak_kind
                                    if peak_kind == "measured" else "fallback 6.65 TB/s",
                     "traffic": profiled_traffic(wl.name),
                     "kernel": ("far_decode_kernel" if launch["regime"] == 1 else
                                "far_ring_kernel" if launch["kernel"] == 1 else "far_prefill_kernel"),
                     "launch_time": "median of %d per-launch CUDA-event intervals" % args.steps,
                     "median_launch_us": round(case.median_launch * 1e6, 3),
                     "mean_launch_us": round(mean_launch * 1e6, 3),
                     "achieved_on_mean": round(achieved_mean, 2),
                     "frac_on_mean": round(achieved_mean / peak, 4),
                     "launch": launch},
        "e2e": {"value": round(case.bytes / e2e_s / 1e9, 3), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": args.e2e_steps, "ms_per_step": round(e2e_s * 1e3, 3), "path": e2e_mode},
        "gpu_launches": args.steps * (2 if wl.pattern == 3 else 1),
        "clocks": clocks,
    }

    if world == 1 and not args.no_extras:
        line["other_workloads"] = extras(ctx, device, stream)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, inp, case.nout is not None)
    ctx.close()
    if rank == 0:
        print(json.dumps(line), flush=True)


def extras(ctx, device, stream) -> dict:
    """The other synthetic workloads, one short measurement each."""
    from reduce_residual_add_b200 import far
    out = {}
    peak, _ = hbm_peak()
    for name, with_norm in (("c5_gemma_fp8_token_bf16", False), ("c5_gemma_fp8_token_fp16", False),
                            ("c5_gemma_fp8_token_bf16", True), ("c4_prefill_fp8_static", True),
                            ("c4_prefill_fp8_tensor", False), ("c4_prefill_fp8_group128", False),
                            ("c3_3d", False)):
        wl = WORKLOADS[name]
        inp = make_inputs(wl)
        case = Case(ctx, wl, inp, device, with_norm, stream)
        # a short call is launched through a prepared call: the binding's
        # marshalling (about 10 us) would otherwise sit between the events
        short = wl.pattern in (0, 1, 2) and case.bytes < L2_BYTES
        total, mean = case.time_steps(200, 20, per_launch=True, prepared=short)
        if with_norm:
            name += "+norm_out"
        med = case.median_launch
        out[name] = {"GB/s": round(case.bytes / mean / 1e9, 1),
                     "launches_per_call": 2 if wl.pattern == 3 else 1,
                     "frac": round(case.bytes / mean / 1e9 / peak, 4),
                     "us_per_call": round(mean * 1e6, 2), "tokens_per_s": round(wl.T / mean, 1),
                     "median_us_per_call": round(med * 1e6, 2),
                     "frac_on_median": round(case.bytes / med / 1e9 / peak, 4),
                     "traffic": None if with_norm else profiled_traffic(wl.name),
                     "bytes": case.bytes,
                     "stream_timing": ("far.FarCall per call, per-launch events" if short
                                       else "far binding per call, per-launch events")}
        if name == "c3_3d":
            warm = graph_time(case, 50)
            rot = RotatingSets(ctx, wl, inp, device, with_norm, stream)
            cold = rot.graph_time()
            out[name].update({
                "graph_us_per_call": round(warm * 1e6, 3),
                "cold_graph_us_per_call": round(cold * 1e6, 3),
                "cold_GB/s": round(case.bytes / cold / 1e9, 1),
                "cold_frac": round(case.bytes / cold / 1e9 / peak, 4),
                "cold_sets": rot.n,
                "timing": "graph_us_per_call: one input set replayed (L2-resident); "
                          "cold_*: a CUDA graph cycling through %d input/output sets "
                          "(%d MiB per cycle, more than 2x L2)"
                          % (rot.n, rot.n * touched_bytes(wl, True) // 2 ** 20)})
            del rot
        del case
    # the latency floor of one call: a single row of 64 elements, one partial
    wl = WORKLOADS["c1_small"].with_(name="floor_W1_T1_H64", W=1, T=1)
    case = Case(ctx, wl, make_inputs(wl), device, False, stream)
    out["floor_W1_T1_H64"] = {"graph_us_per_call": round(graph_time(case, 100) * 1e6, 3),
                              "note": "latency floor: the smallest call, same kernels and launch path"}
    del case
    for T in (1, 8, 32, 80):
        wl = WORKLOADS["c2_decode_T%d" % T]
        inp = make_inputs(wl)
        case = Case(ctx, wl, inp, device, False, stream)
        row = {}
        rot = RotatingSets(ctx, wl, inp, device, False, stream)
        for reg, nm in ((far.FAR_REGIME_AUTO, "auto"), (far.FAR_REGIME_DECODE, "cluster_kernel"),
                        (far.FAR_REGIME_PREFILL, "one_cta_per_row")):
            far.far_set_regime(ctx, reg)
            row[nm] = {"graph_us_per_call": round(graph_time(case, 200) * 1e6, 3),
                       "cold_graph_us_per_call": round(rot.graph_time() * 1e6, 3)}
        far.far_set_regime(ctx, far.FAR_REGIME_AUTO)
        row["auto"]["launch"] = far.far_describe_launch(ctx, T, wl.H, wl.torch_dtype, wl.W, True,
                                                        True)
        row["cold_sets"] = rot.n
        del rot
        call = case.prepared()
        for _ in range(50):
            call()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(case.stream)
        for _ in range(500):
            call()
        b.record(case.stream)
        torch.cuda.synchronize()
        row["auto"]["prepared_stream_us_per_call"] = round(a.elapsed_time(b) / 500 * 1e3, 3)
        far.far_set_regime(ctx, far.FAR_REGIME_AUTO)
        row["tokens_per_s_graph"] = round(T / (row["auto"]["graph_us_per_call"] * 1e-6), 1)
        row["tokens_per_s_cold_graph"] = round(T / (row["auto"]["cold_graph_us_per_call"] * 1e-6), 1)
        row["timing"] = ("graph_us_per_call: one input set replayed (L2-resident); "
                         "cold_graph_us_per_call: a CUDA graph cycling through %d sets "
                         "(more than 2x L2 per cycle); prepared_stream_us_per_call: one "
                         "far.FarCall per call in a stream (host-bound)" % row["cold_sets"])
        row["bytes"] = case.bytes
        out[wl.name] = row
        del case
    return out


def run_sp(args, world, rank, local):
    """Sequence-parallel tensor parallelism across the ranks (one per GPU):
    the batch's W = world partials are the ranks' own row-parallel outputs,
    each rank owns T / world rows of the residual; one step is the row
    exchange, the fused epilogue on the local rows (W = world partials) and
    the all-gather of the normed outputs (reduce_residual_add_b200.sp)."""
    from reduce_residual_add_b200 import build as fbuild
    from reduce_residual_add_b200 import far, sp
    import torch.distributed as dist
    fbuild.build()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    base = WORKLOADS[args.workload]
    if base.pattern not in (0, 1, 2):
        raise SystemExit("--sp takes the norm, static FP8 and per-token FP8 workloads")
    wl = base.with_(W=world, T=args.rows or base.T)
    if not sp.is_applicable(wl.T, world):
        raise SystemExit("%d rows do not split over %d ranks" % (wl.T, world))
    inp = make_inputs(wl)                       # the same draw on every rank
    b, e = sp.rows_for_rank(wl.T, world, rank)
    part = inp["partials"][rank].to(device)
    res_rows = inp["residual"][b:e].to(device) if wl.has_residual else None
    gam = inp["gamma"].to(device)
    rout = torch.empty(e - b, wl.H, dtype=wl.torch_dtype, device=device)
    sin = (torch.tensor([wl.static_scale], dtype=torch.float32, device=device)
           if wl.pattern == 1 else None)
    del inp
    ctx = far.FarContext(local)
    group = dist.group.WORLD if world > 1 else None
    if world == 1:
        import datetime
        dist.init_process_group("nccl", rank=0, world_size=1, init_method="tcp://127.0.0.1:%d"
                                % _free_port(), timeout=datetime.timedelta(seconds=120),
                                device_id=device)
        group = dist.group.WORLD
    if args.peer:
        step = sp.PeerSequenceParallelEpilogue(group, wl.T, wl.H, wl.torch_dtype, wl.pattern,
                                               device, with_norm=args.with_norm, ctx=ctx)
        step.partial.copy_(part)        # the row-parallel GEMM would write it there

        def one():
            step(res_rows, gam, wl.eps, wl.weight_bias, residual_out=rout, scale_in=sin)
    else:
        step = sp.SequenceParallelEpilogue(group, wl.T, wl.H, wl.torch_dtype, wl.pattern, device,
                                           with_norm=args.with_norm, ctx=ctx)

        def one():
            step(part, res_rows, gam, wl.eps, wl.weight_bias, residual_out=rout, scale_in=sin)
    s = torch.cuda.current_stream()

    for _ in range(args.warmup):
        one()
    dist.barrier()
    torch.cuda.synchronize()
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s)
    for _ in range(args.steps):
        one()
    z.record(s)
    torch.cuda.synchronize()
    dist.barrier()
    t = max_over_ranks(a.elapsed_time(z) / 1e3, world)
    nbytes = algorithmic_bytes(wl, wl.T, step.with_norm)
    line = {"metric": METRIC, "value": round(nbytes * args.steps / t / 1e9, 2), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(t / args.steps * 1e3, 5), "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": dict(workload_config(wl, nbytes, step.with_norm, world),
                           parallelism=("sequence parallel over %d rank(s): %s, fused epilogue "
                                        "on T/%d rows with W=%d partials, all-gather of the "
                                        "normed outputs"
                                        % (world, "the kernel reads the peers' rows directly "
                                           "(symmetric memory)" if args.peer else
                                           "row exchange (all_to_all_single)", world, world))),
            "tokens_per_s": round(wl.T * args.steps / t, 1),
            "gpu_launches": args.steps}
    ctx.close()
    del step
    dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def _free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def run_reference(args, world, rank):
    """The CPU oracle, timed on this host's cores, on the same workload."""
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    inp = make_inputs(wl)
    with_norm = args.with_norm or wl.pattern == 0   # the plain pattern always writes norm_out
    t1, _ = oracle_rate(wl, inp, 16, with_norm)
    cores = host_cores()
    budget = 90.0   # seconds of wall time for all steps
    rows = wl.T
    for _ in range(3):   # the thread count depends on the rows, the rows on the rate
        used = oracle_threads(wl, rows, cores)
        per_row = t1 / 16 / used
        rows = max(1, min(wl.T, int(budget / (args.steps + args.warmup) / per_row)))
    used = oracle_threads(wl, rows, cores)
    for _ in range(args.warmup):
        oracle_rate(wl, inp, rows, with_norm, used)
    tot_t, tot_b = 0.0, 0
    for _ in range(args.steps):
        dt, b = oracle_rate(wl, inp, rows, with_norm, used)
        tot_t += dt
        tot_b += b
    value = tot_b / tot_t / 1e9
    sample = ("first %d of %d rows of %s per step, C fp64 oracle on %d threads "
              "(one contiguous row range each)" % (rows, wl.T, wl.name, used))
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(tot_t / args.steps * 1e3, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            # the same workload object as the CUDA arm's line (no kernel launch here)
            "config": workload_config(wl, algorithmic_bytes(wl, wl.T, with_norm), with_norm, world),
            "tokens_per_s": round(rows * args.steps / tot_t, 3),
            "cpu_baseline": {"value": round(value, 5), "unit": "GB/s", "cores": used,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 5), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["far", "reference"], default="far")
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS))
    ap.add_argument("--with-norm", action="store_true", help="also write norm_out")
    ap.add_argument("--rows", type=int, default=0,
                    help="override the workload's row count (smaller cases for profiling)")
    ap.add_argument("--shape", default="",
                    help="W,H: override the workload's partial count and hidden size "
                         "(other shapes for profiling)")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--e2e-chunk-rows", type=int, default=0,
                    help="rows per chunk of far_fused_host in the e2e leg (0: the library default)")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--peer", action="store_true",
                    help="with --sp: the one-shot variant, partials read from the peers' memory")
    ap.add_argument("--sp", action="store_true",
                    help="sequence-parallel step across the ranks: each rank holds one of "
                         "W = N partials and T/N rows of the residual")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    world, rank, local = dist_setup(args.gpus)
    if args.sp:
        run_sp(args, world, rank, local)
        return
    try:
        run_far(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

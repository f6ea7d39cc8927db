"""Benchmark of the fused bf16 sum + residual + RMSNorm + per-row FP8 call.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--replays N] [--impl rrf|reference]
    python bench.py --plan-sweep reduce_rmsnorm_fp8_b200/csrc/rrf_plan_table.inc

One step is one pass of the operation over one batch of the workload: for
the default "prefill" workload, the largest single-GPU configuration, one
call of R = 8 bf16 inputs of 8192 x 8192 with the residual on (1.41 GB of
HBM traffic).  Inputs are resident in HBM when the timed region starts and
rotate over buffer sets whose total exceeds three times the L2 cache, so
every step reads cold HBM.  K steps are captured in one CUDA graph and timed
with CUDA events on the launching stream, bracketed by a barrier and a
device synchronisation on both sides; the value comes from the median of
--replays timed replays, and the time is the maximum over ranks.

value = algorithmic bytes of all ranks' steps / time, in GB/s, where one
fused call moves R*rows*cols*2 + 4*rows*cols (residual read + write) +
2*cols (gamma) + rows*cols (fp8 codes) + 4*rows (scales) bytes.

Beside the headline: every configuration's calls timed one by one (decode
1/8/32/64 x 7168, odd 37/64 x 7168, tiny, prefill), the launch floor of the
call chain, the end-to-end figure through pinned host buffers, the oracle on
one core and on all cores, and the other entry points.

Multi-GPU (torchrun, one process per GPU, NCCL only for the barrier and the
max-over-ranks timing): rows are independent, so every rank runs its own
batch with no data-path collective (weak scaling).

--impl reference times the CPU oracle (single-threaded C) on a bounded sample
of the same workload, on rank 0 only.  --plan-sweep measures the fused call's
launches on a grid of shapes and writes the library's launch table.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "fused sum+RMSNorm+FP8 achieved HBM GB/s (% of B200 peak) and us/call"
L2_FLUSH_FACTOR = 3  # rotating pool >= 3 x L2


# ---------------------------------------------------------------- helpers ---

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def shard_rows(rows: int, world: int, rank: int):
    """Contiguous row block [start, stop) of `rank` when `rows` independent
    rows are split over `world` ranks (the first rows % world ranks get one
    more)."""
    base, extra = divmod(rows, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank float over all ranks (identity without a
    process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


ROWS_OVERRIDE = None  # --rows: a subset of the workload's row counts


def workload_cases(name: str):
    """(rows, residual) of every call one step makes."""
    w = workloads.WORKLOADS[name]
    rows = ROWS_OVERRIDE if ROWS_OVERRIDE else w.rows
    return [(r, w.residual) for r in rows]


def step_bytes(name: str) -> int:
    w = workloads.WORKLOADS[name]
    return sum(workloads.fused_bytes(w.R, rows, w.cols, res) for rows, res in
               workload_cases(name))


def kernel_source_hash() -> str:
    """sha256 of the fused kernel's sources: a recorded ncu traffic figure is
    valid only for the kernel it was taken from."""
    import hashlib
    h = hashlib.sha256()
    for f in ("rrf_fused.cu", "rrf_device.cuh"):
        with open(os.path.join(ROOT, "reduce_rmsnorm_fp8_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum)
    of the fused kernel on `workload`, from profiles/fused_kernel_traffic.txt,
    or None if none is recorded for the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "fused_kernel_traffic.txt")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    src = None
    for line in lines:
        if line.startswith("kernel_source_sha256:"):
            src = line.split(":", 1)[1].strip()
        elif line and not line.startswith("#") and src == kernel_source_hash():
            parts = line.split()
            if parts[0] == workload:
                return int(parts[1])
    return None


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def fp8_peak_tflops():
    """Dense fp8 tensor peak: the measured cuBLAS bf16 burst figure times the
    nominal fp8 / bf16 ratio (4.5 / 2.25 PFLOP/s), else the fallback 1.59
    PFLOP/s bf16 times the same ratio."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            return 2.0 * float(json.load(fh)["bf16_tflops"]), "measured bf16_tflops x 2"
    except Exception:
        return 2.0 * 1590.0, "fallback bf16 x 2"


_CLOCK_POLL = r"""
import sys, time
import pynvml
pynvml.nvmlInit()
bus = sys.argv[1]
try:
    h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
except Exception:
    h = pynvml.nvmlDeviceGetHandleByIndex(int(sys.argv[2]))
print("max", pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM), flush=True)
while True:
    t = time.monotonic()
    c = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
    r = int(pynvml.nvmlDeviceGetCurrentClocksEventReasons(h))
    print(f"{t:.6f} {c} {r}", flush=True)
    time.sleep(0.0002)
"""


class ClockSampler:
    """Samples the SM clock and the active clock-event reasons of one GPU
    through NVML in a separate process (so no Python lock of this process
    can starve it), every ~0.2 ms; summary() keeps the samples taken between
    mark_start() and mark_end(), the timed region."""

    REASONS = {  # NVML clocks-event-reason bits
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting"}

    def __init__(self, index: int):
        import subprocess
        import tempfile
        import torch
        self.t0 = self.t1 = None
        bus = ""
        try:
            pr = torch.cuda.get_device_properties(index)
            bus = "%08X:%02X:%02X.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
        except Exception:
            pass
        self._out = tempfile.TemporaryFile(mode="w+")
        try:
            self._proc = subprocess.Popen([sys.executable, "-c", _CLOCK_POLL, bus, str(index)],
                                          stdout=self._out, stderr=subprocess.DEVNULL)
        except Exception:
            self._proc = None
        # wait (briefly) for the poller's first sample
        deadline = time.monotonic() + 20.0
        while self._proc is not None and time.monotonic() < deadline:
            self._out.seek(0)
            if self._out.read().count("\n") >= 2 or self._proc.poll() is not None:
                break
            time.sleep(0.05)

    def mark_start(self):
        self.t0 = time.monotonic()

    def mark_end(self):
        self.t1 = time.monotonic()

    def summary(self):
        if self._proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        self._proc.terminate()
        self._proc.wait()
        self._out.seek(0)
        max_mhz, samples, reasons = None, [], 0
        for line in self._out.read().splitlines():
            parts = line.split()
            if parts and parts[0] == "max":
                max_mhz = int(parts[1])
            elif len(parts) == 3:
                t, c, r = float(parts[0]), int(parts[1]), int(parts[2])
                if self.t0 is not None and self.t0 <= t <= self.t1:
                    samples.append(c)
                    reasons |= r
        names = [n for bit, n in self.REASONS.items() if reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(samples) if samples else None,
                "sm_max_mhz": max_mhz, "reasons": names, "samples": len(samples),
                "source": "NVML, sampled every ~0.2 ms during the timed region"}


# -------------------------------------------------------------- CUDA arm ---

class DevicePool:
    """Rotating buffer sets, all resident in HBM: for each call of the
    workload (or the listed row counts), n_sets copies of the R inputs, the
    residual, gamma and the outputs, carved as views from one allocation per
    tensor kind.  n_sets is chosen so the sets together exceed min_bytes of
    algorithmic traffic, so a set is cold in L2 when its turn comes again."""

    def __init__(self, name: str, device, min_bytes: int, rows_list=None, with_sum=False):
        import torch
        self.name = name
        w = workloads.WORKLOADS[name]
        rows_list = [r for r, _ in workload_cases(name)] if rows_list is None else rows_list
        self.cases = [workloads.make_case(name, rows, device=device) for rows in rows_list]
        per_set = sum(workloads.fused_bytes(w.R, c.rows, c.cols, c.residual is not None)
                      for c in self.cases)
        self.n_sets = n = max(2, math.ceil(min_bytes / per_set))
        self.per_set_bytes = per_set
        self.big = []
        for c in self.cases:
            shape = (n, c.rows, c.cols)
            b = {"inputs": [x.unsqueeze(0).expand(shape).contiguous() for x in c.inputs],
                 "gamma": c.gamma.unsqueeze(0).expand(n, c.cols).contiguous(),
                 "q": torch.empty(shape, dtype=torch.float8_e4m3fn, device=device),
                 "scales": torch.empty((n, c.rows, 1), dtype=torch.float32, device=device),
                 "residual": None, "res_out": None}
            if c.residual is not None:
                b["residual"] = c.residual.unsqueeze(0).expand(shape).contiguous()
                b["res_out"] = torch.empty(shape, dtype=torch.bfloat16, device=device)
            if with_sum:
                b["sum_out"] = torch.empty(shape, dtype=torch.bfloat16, device=device)
            self.big.append(b)
        self.eps, self.wo, self.ub = w.eps, w.weight_offset, w.scale_ub

    def call(self, rrf, k: int, i: int, flags: int = 0) -> int:
        """Enqueue call i of the workload on set k mod n_sets (the library's
        own launch; flags: RRF_FLAG_* overrides through the _ex entry);
        returns 1."""
        b, s = self.big[i], k % self.n_sets
        args = ([x[s] for x in b["inputs"]], b["gamma"][s], self.eps, self.wo, self.ub)
        kw = dict(residual_in=None if b["residual"] is None else b["residual"][s],
                  residual_out=None if b["res_out"] is None else b["res_out"][s],
                  q_out=b["q"][s], scales_out=b["scales"][s])
        if flags:
            rrf.rrf_sum_rmsnorm_fp8_ex(*args, **kw, flags=flags)
        else:
            rrf.rrf_sum_rmsnorm_fp8(*args, **kw)
        return 1

    def call_sum(self, rrf, k: int, i: int) -> int:
        """Enqueue the sum-only call i on set k mod n_sets; returns 1."""
        b, s = self.big[i], k % self.n_sets
        rrf.rrf_sum([x[s] for x in b["inputs"]], out=b["sum_out"][s])
        return 1

    def run_step(self, rrf, k: int) -> int:
        """Enqueue step k: every call of the workload on set k mod n_sets;
        returns the number of kernels launched."""
        return sum(self.call(rrf, k, i) for i in range(len(self.cases)))


def time_region(fn, k_steps: int, device, stream, clocks=None):
    """Device time of k_steps calls of fn(i), CUDA events on `stream`, with a
    barrier and a synchronisation on both sides; max over ranks, seconds.
    A ClockSampler is told when the region starts and ends."""
    import torch
    barrier(device)
    torch.cuda.synchronize(device)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if clocks is not None:
        clocks.mark_start()
    start.record(stream)
    for i in range(k_steps):
        fn(i)
    end.record(stream)
    torch.cuda.synchronize(device)
    if clocks is not None:
        clocks.mark_end()
    barrier(device)
    return max_over_ranks(start.elapsed_time(end) / 1e3, device)


def time_sharded(rrf, label, rows, cols, shards, device, stream, l2, peak):
    """Both phases of the sharded form on one shard [rows, cols] of a row
    split into `shards` (R = 8, residual), each over rotating buffer sets
    larger than 3 x L2; the gathered statistics are synthetic (the other
    shards' are copies of this one's)."""
    import torch
    c = workloads.make_case(label, rows, cols=cols, device=device)
    R = c.R
    pre_b = R * rows * cols * 2 + 4 * rows * cols + 2 * cols + 8 * rows
    post_b = 2 * rows * cols + 2 * cols + 8 * shards * rows + rows * cols + 4 * rows
    n = max(2, math.ceil(L2_FLUSH_FACTOR * l2 / (pre_b + post_b)))
    shape = (n, rows, cols)
    xs = [x.unsqueeze(0).expand(shape).contiguous() for x in c.inputs]
    res = c.residual.unsqueeze(0).expand(shape).contiguous()
    h = torch.empty(shape, dtype=torch.bfloat16, device=device)
    st = torch.empty((n, rows, 2), dtype=torch.float32, device=device)
    gathered = torch.empty((n, shards, rows, 2), dtype=torch.float32, device=device)
    q = torch.empty(shape, dtype=torch.float8_e4m3fn, device=device)
    sc = torch.empty((n, rows, 1), dtype=torch.float32, device=device)

    def pre(k):
        s = k % n
        rrf.rrf_sum_rmsnorm_fp8_pre([x[s] for x in xs], c.gamma, c.weight_offset,
                                    residual_in=res[s], residual_out=h[s], stats_out=st[s])
        return 1

    def post(k):
        s = k % n
        rrf.rrf_rmsnorm_fp8_post(h[s], c.gamma, gathered[s], cols * shards, c.eps,
                                 c.weight_offset, c.scale_ub, q_out=q[s], scales_out=sc[s])
        return 1

    for k in range(n):
        pre(k)
    torch.cuda.synchronize(device)
    gathered.copy_(st.unsqueeze(1).expand(n, shards, rows, 2))
    rec = {"shard": f"{label} {rows} x {cols} (1 of {shards})", "R": R}
    for name, fn, nbytes in (("pre", pre, pre_b), ("post", post, post_b)):
        reps = 100 if rows < 1024 else 10
        g, _ = capture_steps(fn, reps, device)
        g.replay()
        torch.cuda.synchronize(device)
        t = time_region(lambda _: g.replay(), 1, device, stream)
        del g
        rec[f"{name}_us"] = round(t / reps * 1e6, 3)
        rec[f"{name}_GB_s"] = round(nbytes * reps / t / 1e9, 1)
        rec[f"{name}_frac"] = round(nbytes * reps / t / 1e9 / peak, 4)
    return rec


def time_allreduce(rrf, label, rows, world, mode, device, stream, l2):
    """The multi-GPU call with all `world` ranks in one launch on this GPU
    (LocalGroup): one CUDA graph of `reps` calls, cycling through buffer sets
    larger than 3 x L2 (the residual updated in place);
    microseconds per call.  This GPU's memory stands in for the links, so the
    number bounds the kernel's own cost, not a multi-GPU call's."""
    import torch

    from reduce_rmsnorm_fp8_b200 import allreduce
    c = workloads.make_case(label, rows, R=world, device=device)
    cols = c.cols
    set_bytes = world * rows * cols * 2 * 3 + world * rows * cols
    n = max(1, math.ceil(L2_FLUSH_FACTOR * l2 / set_bytes))
    rep = lambda t: t.unsqueeze(0).repeat(n, 1, 1)  # a copy, also for n == 1
    xs = [rep(x) for x in c.inputs]                # [n, rows, cols] per rank
    rs = [rep(c.residual) for _ in range(world)]
    qs = [torch.empty((n, rows, cols), dtype=torch.float8_e4m3fn, device=device)
          for _ in range(world)]
    ss = [torch.empty((n, rows, 1), dtype=torch.float32, device=device) for _ in range(world)]
    g = allreduce.LocalGroup(world, device)

    def call(k):
        i = k % n
        g([x[i] for x in xs], c.gamma, c.eps, c.weight_offset, c.scale_ub,
          residual_in=[r[i] for r in rs], residual_out=[r[i] for r in rs],
          q_out=[q[i] for q in qs], scales_out=[s[i] for s in ss], mode=mode)
        return 1

    reps = max(50, n) if rows < 1024 else 5
    for k in range(reps):  # warm-up, eager
        call(k)
    torch.cuda.synchronize(device)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):  # the pads number the replayed calls themselves
        for k in range(reps):
            call(k)
    graph.replay()
    torch.cuda.synchronize(device)
    t = time_region(lambda _: graph.replay(), 1, device, stream)
    del graph
    sm = torch.cuda.get_device_properties(device).multi_processor_count
    m, cl, th, vpt = rrf.rrf_plan_allreduce(world, rows, cols, sm, True, mode)
    flags = rrf.rrf_device_error(clear=True)
    return {"case": f"{label} {rows} x {cols}, {world} ranks",
            "mode": "two-shot" if m == 2 else "one-shot",
            "launch": {"cluster": cl, "threads": th, "vecs_per_thread": vpt},
            "us_per_call": round(t / reps * 1e6, 3), "device_error": flags}


def time_gemm(rrf, M, N, K, device, stream, l2, hbm_peak):
    """The FP8 GEMM that consumes the per-row scales (rrf_scaled_mm_fp8), one
    CUDA graph of calls cycling through operand sets larger than 3 x L2;
    TFLOP/s against the fp8 tensor peak and algorithmic GB/s against HBM."""
    import torch
    sets_bytes = workloads.gemm_bytes(M, N, K)
    n = max(1, math.ceil(L2_FLUSH_FACTOR * l2 / sets_bytes))
    cases = [workloads.make_gemm_case(M, N, K, sub=i, device=device) for i in range(n)]
    outs = [torch.empty((M, N), dtype=torch.bfloat16, device=device) for _ in range(n)]

    def call(k):
        c = cases[k % n]
        rrf.rrf_scaled_mm_fp8(c.a, c.a_scale, c.b, c.b_scale, c.bias, out=outs[k % n])
        return 1

    for k in range(3):
        call(k)
    reps = max(n, 20 if M * N * K >= 2 ** 36 else 100)
    g, _ = capture_steps(call, reps, device)
    g.replay()
    torch.cuda.synchronize(device)
    t = time_region(lambda _: g.replay(), 1, device, stream) / reps
    del g, cases, outs
    tf = workloads.gemm_flops(M, N, K) / t / 1e12
    gbs = workloads.gemm_bytes(M, N, K) / t / 1e9
    fp8_peak, fp8_kind = fp8_peak_tflops()
    return {"shape": f"{M} x {N} x {K}", "us_per_call": round(t * 1e6, 3),
            "TFLOP_s": round(tf, 1), "tensor_frac": round(tf / fp8_peak, 4),
            "GB_s": round(gbs, 1), "hbm_frac": round(gbs / hbm_peak, 4),
            "fp8_peak_TFLOP_s": round(fp8_peak, 1), "fp8_peak_kind": fp8_kind,
            "operand_sets": n, "device_error": rrf.rrf_device_error(clear=True)}


def mx_bytes(R: int, rows: int, cols: int, residual: bool) -> int:
    """Algorithmic HBM bytes of one MX call: as the row-scaled call, with one
    E8M0 byte per 32 elements in place of one float per row."""
    return R * rows * cols * 2 + (4 * rows * cols if residual else 0) + cols * 2 \
        + rows * cols + rows * cols // 32


def time_mx(rrf, label, rows, device, stream, l2, peak):
    """The MX output (rrf_sum_rmsnorm_mxfp8) on one configuration, one CUDA
    graph of calls cycling through buffer sets larger than 3 x L2."""
    import torch
    c = workloads.make_case(label, rows, device=device)
    nbytes = mx_bytes(c.R, rows, c.cols, c.residual is not None)
    n = max(2, math.ceil(L2_FLUSH_FACTOR * l2 / nbytes))
    rep = lambda t: t.unsqueeze(0).repeat(n, *([1] * t.dim()))
    xs = [rep(x) for x in c.inputs]
    res = None if c.residual is None else rep(c.residual)
    q = torch.empty((n, rows, c.cols), dtype=torch.float8_e4m3fn, device=device)
    sc = torch.empty((n, rows, c.cols // 32), dtype=torch.uint8, device=device)

    def call(k):
        i = k % n
        r = None if res is None else res[i]
        rrf.rrf_sum_rmsnorm_mxfp8([x[i] for x in xs], c.gamma, c.eps, c.weight_offset,
                                  residual_in=r, residual_out=r, q_out=q[i], scales_mx_out=sc[i])
        return 1

    for k in range(3):
        call(k)
    reps = max(n, 100) if rows < 1024 else 10
    g, _ = capture_steps(call, reps, device)
    g.replay()
    torch.cuda.synchronize(device)
    t = time_region(lambda _: g.replay(), 1, device, stream) / reps
    del g, xs, res, q, sc
    return {"case": f"{label} {rows} x {c.cols}", "R": c.R, "us_per_call": round(t * 1e6, 3),
            "GB_s": round(nbytes / t / 1e9, 1), "frac": round(nbytes / t / 1e9 / peak, 4)}


def time_gemm_mx(rrf, M, N, K, device, stream, l2, hbm_peak):
    """The MX GEMM (rrf_scaled_mm_mxfp8) on operands with random E8M0 codes
    in [120, 134), cycling through operand sets larger than 3 x L2."""
    import numpy as np
    import torch
    nbytes = workloads.gemm_bytes(M, N, K) + (M + N) * K // 32
    n = max(1, math.ceil(L2_FLUSH_FACTOR * l2 / nbytes))
    sets = []
    for i in range(n):
        c = workloads.make_gemm_case(M, N, K, sub=i, device=device)
        rng = np.random.default_rng(200 + i)
        sa = rrf.mx_blocked(torch.from_numpy(
            rng.integers(120, 134, (M, K // 32)).astype(np.uint8)).to(device))
        sb = rrf.mx_blocked(torch.from_numpy(
            rng.integers(120, 134, (N, K // 32)).astype(np.uint8)).to(device))
        sets.append((c, sa, sb, torch.empty((M, N), dtype=torch.bfloat16, device=device)))

    def call(k):
        c, sa, sb, out = sets[k % n]
        rrf.rrf_scaled_mm_mxfp8(c.a, sa, c.b, sb, c.bias, out=out)
        return 1

    for k in range(3):
        call(k)
    reps = max(n, 20 if M * N * K >= 2 ** 36 else 100)
    g, _ = capture_steps(call, reps, device)
    g.replay()
    torch.cuda.synchronize(device)
    t = time_region(lambda _: g.replay(), 1, device, stream) / reps
    del g, sets
    tf = workloads.gemm_flops(M, N, K) / t / 1e12
    fp8_peak, fp8_kind = fp8_peak_tflops()
    return {"shape": f"{M} x {N} x {K}", "us_per_call": round(t * 1e6, 3),
            "TFLOP_s": round(tf, 1), "tensor_frac": round(tf / fp8_peak, 4),
            "GB_s": round(nbytes / t / 1e9, 1), "hbm_frac": round(nbytes / t / 1e9 / hbm_peak, 4),
            "fp8_peak_TFLOP_s": round(fp8_peak, 1), "fp8_peak_kind": fp8_kind,
            "operand_sets": n, "device_error": rrf.rrf_device_error(clear=True)}


def capture_steps(fn, n: int, device):
    """Capture fn(0) .. fn(n-1) into one CUDA graph; returns (graph, number
    of kernels fn launched)."""
    import torch
    g = torch.cuda.CUDAGraph()
    launched = 0
    torch.cuda.synchronize(device)
    with torch.cuda.graph(g):
        for i in range(n):
            launched += fn(i) or 1
    torch.cuda.synchronize(device)
    return g, launched


class _Arena:
    """Views of one byte buffer, each starting on a 256-byte boundary."""

    def __init__(self):
        self.size, self.items = 0, []

    def add(self, shape, dtype):
        import torch
        off = (self.size + 255) // 256 * 256
        n = math.prod(shape) * torch.empty((), dtype=dtype).element_size()
        self.items.append((off, n, shape, dtype))
        self.size = off + n
        return len(self.items) - 1

    def views(self, buf):
        return [buf[off:off + n].view(dtype).view(shape) for off, n, shape, dtype in self.items]


def e2e_measure(rrf, name: str, k_steps: int, warmup: int, device, stream):
    """The same metric through the public call with HOST buffers.  Every step
    copies its inputs (all calls' inputs, residuals and gammas, packed in one
    pinned host buffer) to the device in one copy, runs the calls, and reads
    all results (codes, scales, residual outputs) back to pinned host memory
    in one copy; all copies are inside the timed region.  Steps are
    double-buffered over three streams (H2D, compute, D2H), as a serving loop
    would run them, so one step's copies overlap the neighbouring steps'."""
    import torch
    w = workloads.WORKLOADS[name]
    cases = [workloads.make_case(name, rows, device=device) for rows, _ in workload_cases(name)]
    ins, outs = _Arena(), _Arena()
    slots = []
    for c in cases:
        shape = (c.rows, c.cols)
        slot = {"inputs": [ins.add(shape, torch.bfloat16) for _ in c.inputs],
                "gamma": ins.add((c.cols,), torch.bfloat16),
                "residual": ins.add(shape, torch.bfloat16) if c.residual is not None else None,
                "q": outs.add(shape, torch.uint8),
                "scales": outs.add((c.rows, 1), torch.float32),
                "res_out": outs.add(shape, torch.bfloat16) if c.residual is not None else None}
        slots.append(slot)
    h_in = torch.empty(ins.size, dtype=torch.uint8).pin_memory()
    h_out = [torch.empty(outs.size, dtype=torch.uint8).pin_memory() for _ in range(2)]
    d_in = [torch.empty(ins.size, dtype=torch.uint8, device=device) for _ in range(2)]
    d_out = [torch.empty(outs.size, dtype=torch.uint8, device=device) for _ in range(2)]
    hv = ins.views(h_in)
    dv = [ins.views(b) for b in d_in]
    ov = [outs.views(b) for b in d_out]
    for c, slot in zip(cases, slots):  # the host data of the step
        for x, i in zip(c.inputs, slot["inputs"]):
            hv[i].copy_(x)
        hv[slot["gamma"]].copy_(c.gamma)
        if slot["residual"] is not None:
            hv[slot["residual"]].copy_(c.residual)
    h2d = sum(n for _, n, _, _ in ins.items)
    d2h = sum(n for _, n, _, _ in outs.items)

    s_in, s_cmp, s_out = (torch.cuda.Stream(device) for _ in range(3))
    in_ready = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    copied_out = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    def step(k):
        b = k % 2
        with torch.cuda.stream(s_in):
            if used[b]:
                s_in.wait_event(computed[b])  # slot b's inputs are free again
            d_in[b].copy_(h_in, non_blocking=True)
            in_ready[b].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(in_ready[b])
            if used[b]:
                s_cmp.wait_event(copied_out[b])  # slot b's outputs were read
            for slot in slots:
                rrf.rrf_sum_rmsnorm_fp8(
                    [dv[b][i] for i in slot["inputs"]], dv[b][slot["gamma"]], w.eps,
                    w.weight_offset, w.scale_ub,
                    residual_in=None if slot["residual"] is None else dv[b][slot["residual"]],
                    residual_out=None if slot["res_out"] is None else ov[b][slot["res_out"]],
                    q_out=ov[b][slot["q"]].view(torch.float8_e4m3fn),
                    scales_out=ov[b][slot["scales"]])
            computed[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(computed[b])
            h_out[b].copy_(d_out[b], non_blocking=True)
            copied_out[b].record(s_out)
        used[b] = True

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize(device)
    barrier(device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    for i in range(k_steps):
        step(warmup + i)
    s_in.wait_stream(s_out)
    end.record(s_in)
    torch.cuda.synchronize(device)
    barrier(device)
    t = max_over_ranks(start.elapsed_time(end) / 1e3, device)
    return t, h2d, d2h


def _oracle_sample(name: str, rows: int):
    """The workload's inputs for the oracle: one call of `rows` rows (drawn
    with the workload's seeds), as bf16 bit patterns."""
    bits = workloads.bits
    c = workloads.make_case(name, rows, sub=0)
    return ([bits(x) for x in c.inputs], None if c.residual is None else bits(c.residual),
            bits(c.gamma), c)


def cpu_baseline(name: str, budget_s: float = 10.0):
    """The oracle, as it stands, on bounded samples of the workload: the
    single-threaded C oracle on a block of rows per call until about budget_s
    seconds, and the same per-row function on every core this process may use
    (rows split into contiguous chunks, one POSIX thread each) on a larger
    block.  Rows are independent, so GB/s over the sample is the oracle's
    throughput on the workload."""
    import oracle
    w = workloads.WORKLOADS[name]
    o = oracle.default()
    cores = o.cores()
    calls = [r for r, _ in workload_cases(name)]
    one_rows = [min(r, 8) for r in calls]
    all_rows = [min(r, 16 * cores) for r in calls]
    legs = {}
    for leg, rows_list, threads in (("one", one_rows, 1), ("all", all_rows, cores)):
        prepared = [_oracle_sample(name, r) for r in rows_list]
        nbytes = sum(workloads.fused_bytes(w.R, r, w.cols, w.residual) for r in rows_list)

        def one_step():
            for xs, res, g, c in prepared:
                if threads == 1:
                    o.sum_rmsnorm_fp8(xs, c.rows, c.cols, g, c.eps, c.weight_offset,
                                      c.scale_ub, residual=res)
                else:
                    o.sum_rmsnorm_fp8_mt(xs, c.rows, c.cols, g, c.eps, c.weight_offset,
                                         c.scale_ub, residual=res, threads=threads)

        one_step()  # warms the caches
        n, t0 = 0, time.perf_counter()
        while True:
            one_step()
            n += 1
            if time.perf_counter() - t0 >= budget_s:
                break
        dt = time.perf_counter() - t0
        sample = (f"{n} x ({', '.join(str(r) for r in rows_list)} of the "
                  f"{', '.join(str(r) for r in calls)} rows per call, R={w.R} x {w.cols} cols"
                  f"{' + residual' if w.residual else ''}), {dt:.1f} s")
        legs[leg] = {"value": round(nbytes * n / dt / 1e9, 6), "unit": "GB/s",
                     "cores": threads, "kind": "oracle", "sample": sample,
                     "rows_per_s": round(sum(rows_list) * n / dt, 1)}
    out = dict(legs["one"])
    out["sample"] += ", single-threaded C"
    out["all_cores"] = legs["all"]
    out["all_cores"]["sample"] += (f", {cores} POSIX threads (the cores of this process's "
                                   f"CPU affinity), one contiguous row chunk each")
    return out


def time_calls(rrf, name, rows, device, stream, l2, peak, flags=0, replays=11):
    """One call of a workload alone: a CUDA graph of back-to-back calls over
    its own rotating buffer sets (> 3x L2, so every call reads cold HBM),
    `replays` timed replays; the median per call, with p10 / p90."""
    import torch
    w = workloads.WORKLOADS[name]
    cp = DevicePool(name, device, L2_FLUSH_FACTOR * l2, rows_list=[rows])
    nbytes = workloads.fused_bytes(w.R, rows, w.cols, w.residual)
    reps = max(cp.n_sets, 100) if nbytes < 64 << 20 else 20
    for i in range(3):
        cp.call(rrf, i, 0, flags)
    g, _ = capture_steps(lambda k: cp.call(rrf, 3 + k, 0, flags), reps, device)
    g.replay()
    torch.cuda.synchronize(device)
    ts = sorted(time_region(lambda _: g.replay(), 1, device, stream) for _ in range(replays))
    del g, cp
    tc = ts[len(ts) // 2]
    return {"us_per_call": round(tc / reps * 1e6, 3),
            "us_p10": round(ts[len(ts) // 10] / reps * 1e6, 3),
            "us_p90": round(ts[-1 - len(ts) // 10] / reps * 1e6, 3),
            "GB_s": round(nbytes * reps / tc / 1e9, 1),
            "frac": round(nbytes * reps / tc / 1e9 / peak, 4),
            "rows_per_s": round(rows * reps / tc, 1), "bytes": nbytes}


def time_floor(rrf, device, stream, l2, replays=11):
    """The floor of a call in this benchmark's chain: the library's smallest
    kernel (rrf_sum of one 16-byte vector: one input, 8 columns) launched the
    same way (programmatic dependent launch, graph replay), each call reading
    a line of HBM that is not in L2 (a buffer larger than L2 is written
    between replays): an empty PDL kernel chain plus one cold HBM round trip
    per call."""
    import torch
    reps = 100
    x = torch.randn((reps, 2048), device=device).to(torch.bfloat16)  # 4 KB apart
    out = torch.empty((reps, 8), dtype=torch.bfloat16, device=device)
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=device)

    def call(k):
        rrf.rrf_sum([x[k, :8].view(1, 8)], out=out[k].view(1, 8))
        return 1

    for k in range(3):
        call(k)
    g, _ = capture_steps(call, reps, device)
    ts = []
    for _ in range(replays):
        flush.fill_(1)
        torch.cuda.synchronize(device)
        ts.append(time_region(lambda _: g.replay(), 1, device, stream))
    del g
    ts.sort()
    return {"us_per_call": round(ts[len(ts) // 2] / reps * 1e6, 3),
            "what": "rrf_sum of one 16-byte vector per call, cold line each call, PDL, "
                    "graph replay"}


# The calls timed one by one beside the headline: every configuration's row
# counts (decode and odd with the L2 prefetch also forced off).
CASE_CONFIGS = (("decode", (1, 8, 32, 64)), ("odd", (37, 64)), ("tiny", (4,)),
                ("prefill", (8192,)))


def run_rrf(args):
    import torch
    import torch.distributed as dist
    import reduce_rmsnorm_fp8_b200 as rrf

    rank, local_rank, world = dist_env()
    if world != args.gpus and rank == 0:
        print(f"note: --gpus {args.gpus} but WORLD_SIZE {world}; using WORLD_SIZE",
              file=sys.stderr)
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    props = torch.cuda.get_device_properties(device)
    l2 = props.L2_cache_size
    sm = props.multi_processor_count
    peak, peak_kind = measured_peaks()

    name = args.workload
    w = workloads.WORKLOADS[name]
    pool = DevicePool(name, device, L2_FLUSH_FACTOR * l2)
    stream = torch.cuda.current_stream(device)

    # ---- warm-up (eager), then K steps captured in one CUDA graph, timed
    # as the median of several replays (the graph removes the host's
    # per-launch cost from the device timeline)
    for i in range(args.warmup):
        pool.run_step(rrf, i)
    torch.cuda.synchronize(device)
    graph, launches = capture_steps(lambda i: pool.run_step(rrf, args.warmup + i),
                                    args.steps, device)
    graph.replay()  # one untimed replay: graph upload
    torch.cuda.synchronize(device)
    clocks = ClockSampler(device.index)
    clocks.mark_start()
    times = [time_region(lambda _: graph.replay(), 1, device, stream)
             for _ in range(args.replays)]
    clocks.mark_end()
    clock_info = clocks.summary()  # stops the poller
    del graph
    t = statistics.median(times)
    n_sets = pool.n_sets
    per_step = step_bytes(name)
    value = world * per_step * args.steps / t / 1e9
    kernel_us = t / launches * 1e6
    calls_per_step = len(workload_cases(name))
    del pool
    torch.cuda.empty_cache()

    # ---- end to end through host buffers
    e2e = None
    if not args.no_e2e:
        ke = args.e2e_steps
        te, h2d, d2h = e2e_measure(rrf, name, ke, 3, device, torch.cuda.Stream(device))
        e2e = {"value": round(world * per_step * ke / te / 1e9, 3), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": round(te / ke * 1e3, 4), "steps": ke,
               "how": "rrf_sum_rmsnorm_fp8 on device copies of pinned host buffers: one "
                      "H2D and one D2H copy per step, double-buffered over three streams"}
        torch.cuda.empty_cache()

    # ---- every configuration's calls one by one, and the launch floor
    cases = []
    floor = None
    if not args.no_breakdown:
        for cname, rows_list in CASE_CONFIGS:
            wc = workloads.WORKLOADS[cname]
            for rows in rows_list:
                rec = {"workload": cname, "R": wc.R, "rows": rows, "cols": wc.cols,
                       "residual": wc.residual}
                rec.update(time_calls(rrf, cname, rows, device, stream, l2, peak))
                cl, th, vpt, pf = rrf.rrf_plan_fused_ex(wc.R, rows, wc.cols, sm,
                                                        residual=wc.residual)
                rec["launch"] = {"cluster": cl, "threads": th, "vecs_per_thread": vpt,
                                 "prefetch": pf}
                if cname in ("decode", "odd"):
                    rec["no_prefetch"] = time_calls(rrf, cname, rows, device, stream, l2, peak,
                                                    flags=rrf.RRF_FLAG_NO_PREFETCH)["us_per_call"]
                cases.append(rec)
                torch.cuda.empty_cache()
        floor = time_floor(rrf, device, stream, l2)

    # ---- the sum-only / fused sweep over the b12x payload sizes (R=4, 4096 cols)
    sweep = None
    if not args.no_secondary:
        sweep = []
        ws = workloads.WORKLOADS["sweep"]
        for rows in ws.rows:
            sp = DevicePool("sweep", device, L2_FLUSH_FACTOR * l2, rows_list=[rows],
                            with_sum=True)
            rec = {"rows": rows, "payload_KiB": rows * ws.cols * 2 // 1024}
            for op, fn, nbytes in (
                    ("sum", sp.call_sum, workloads.sum_bytes(ws.R, rows, ws.cols)),
                    ("fused", sp.call, workloads.fused_bytes(ws.R, rows, ws.cols, False))):
                for i in range(3):
                    fn(rrf, i, 0)
                reps = 200
                gs, _ = capture_steps(lambda k, fn=fn: fn(rrf, 3 + k, 0), reps, device)
                gs.replay()
                torch.cuda.synchronize(device)
                ts = sorted(time_region(lambda _: gs.replay(), 1, device, stream)
                            for _ in range(5))
                del gs
                rec[f"{op}_us"] = round(ts[2] / reps * 1e6, 3)
                rec[f"{op}_GB_s"] = round(nbytes * reps / ts[2] / 1e9, 1)
            sweep.append(rec)
            del sp
        torch.cuda.empty_cache()
        # the sum alone at the prefill size (8 inputs of 8192 x 8192)
        pf = DevicePool("prefill", device, 2 * l2, with_sum=True)
        for i in range(3):
            pf.call_sum(rrf, i, 0)
        kp = 20
        gs, _ = capture_steps(lambda k: pf.call_sum(rrf, k, 0), kp, device)
        gs.replay()
        torch.cuda.synchronize(device)
        ts = sorted(time_region(lambda _: gs.replay(), 1, device, stream) for _ in range(5))
        del gs, pf
        torch.cuda.empty_cache()
        bs = workloads.sum_bytes(8, 8192, 8192)
        sweep.append({"rows": 8192, "cols": 8192, "R": 8, "sum_us": round(ts[2] / kp * 1e6, 2),
                      "sum_GB_s": round(bs * kp / ts[2] / 1e9, 1),
                      "sum_frac": round(bs * kp / ts[2] / 1e9 / peak, 4)})

    # ---- the sharded form, one shard of 8 (the all-gather between the phases
    # is not on one GPU): decode 32 x 7168 -> 896 columns, prefill 8192 x 8192
    # -> 1024 columns, R = 8 with residual
    sharded = None
    if not args.no_secondary:
        sharded = []
        for label, rows, cols in (("decode", 32, 896), ("prefill", 8192, 1024)):
            sharded.append(time_sharded(rrf, label, rows, cols, 8, device, stream, l2, peak))
        torch.cuda.empty_cache()

    # ---- the multi-GPU call, all ranks emulated in one launch on this GPU
    emulated = None
    if not args.no_secondary:
        emulated = [time_allreduce(rrf, label, rows, ranks, mode, device, stream, l2)
                    for label, rows, ranks, mode in (("decode", 1, 8, 0), ("decode", 8, 8, 0),
                                                     ("decode", 64, 8, 0), ("decode", 64, 8, 1),
                                                     ("prefill", 8192, 8, 0))]
        torch.cuda.empty_cache()

    # ---- the MX output (per-32-element scales)
    mx = None
    if not args.no_secondary:
        mx = [time_mx(rrf, label, rows, device, stream, l2, peak)
              for label, rows in (("decode", 1), ("decode", 8), ("decode", 32), ("decode", 64),
                                  ("prefill", 8192))]
        torch.cuda.empty_cache()

    # ---- the FP8 GEMMs that consume the per-row and the MX scales
    gemm = gemm_mx = None
    if not args.no_secondary:
        gemm = [time_gemm(rrf, M, 7168, 7168, device, stream, l2, peak) for M in (1, 8, 32, 64)]
        gemm.append(time_gemm(rrf, 8192, 8192, 8192, device, stream, l2, peak))
        torch.cuda.empty_cache()
        gemm_mx = [time_gemm_mx(rrf, M, N, N, device, stream, l2, peak)
                   for M, N in ((1, 7168), (8, 7168), (32, 7168), (64, 7168), (8192, 8192))]
        torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(name)

    if rank == 0:
        achieved = per_step * args.steps / t / 1e9
        rows_list = [r for r, _ in workload_cases(name)]
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(t / args.steps * 1e3, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "io": "bf16 inputs/residual/gamma -> e4m3fn codes + f32 scales + bf16 residual",
            "data": "synthetic (seeded splitmix64 + Box-Muller, drawn on the GPU)",
            "impl": "rrf",
            "config": {"workload": f"{name}: R={w.R}, cols={w.cols}, rows {rows_list} per "
                                   f"step, residual={'on' if w.residual else 'off'}",
                       "R": w.R, "cols": w.cols, "rows": rows_list,
                       "bytes_per_step": per_step,
                       "l2": f"inputs larger than L2: {n_sets} rotating buffer sets, "
                             f"{n_sets * per_step >> 20} MiB of traffic > "
                             f"{L2_FLUSH_FACTOR}x L2 ({l2 >> 20} MiB)",
                       "launch": "auto (rrf_sum_rmsnorm_fp8)",
                       "timing": f"K steps captured in one CUDA graph; the median of "
                                 f"{args.replays} timed replays (CUDA events)",
                       "replay_ms": [round(x * 1e3, 4) for x in times],
                       "parallelism": f"dp{world}"},
            "us_per_call": round(t / launches * 1e6, 3),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                         "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "traffic": recorded_traffic(name),
                         "traffic_note": "ncu dram__bytes_read.sum + dram__bytes_write.sum "
                                         "per launch (profiles/fused_kernel_traffic.txt); "
                                         "null when not recorded for these kernel sources",
                         "peak_kind": f"{peak_kind} hbm_gbs",
                         "kernel": "fused_kernel (rrf_fused.cu)",
                         "avg_launch_us": round(kernel_us, 3),
                         "bytes_per_launch": round(per_step / calls_per_step)},
            "gpu_launches": launches,
            "clocks": clock_info,
            "e2e": e2e,
            "cases": cases,
            "floor": floor,
            "sweep": sweep,
            "sharded": sharded,
            "allreduce_emulated": emulated,
            "mx": mx,
            "gemm_fp8": gemm,
            "gemm_mxfp8": gemm_mx,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier(device_ids=[device.index])
        dist.destroy_process_group()


def run_reference(args):
    """The oracle as the reference arm: rank 0 times it on the host cores.
    Each step is a bounded sample of one step of the workload: the first
    2 x cores rows of every call, split into contiguous chunks over one
    POSIX thread per core (the oracle's row-parallel driver of its per-row
    function; rows are independent, so GB/s over the sample is the oracle's
    throughput on the workload)."""
    rank, _, world = dist_env()
    if rank != 0:
        return
    name = args.workload
    w = workloads.WORKLOADS[name]
    import oracle
    o = oracle.default()
    cores = o.cores()
    rows_list = [min(r, 2 * cores) for r, _ in workload_cases(name)]
    prepared = [_oracle_sample(name, r) for r in rows_list]
    per_step = sum(workloads.fused_bytes(w.R, r, w.cols, w.residual) for r in rows_list)

    def step():
        for xs, res, g, c in prepared:
            o.sum_rmsnorm_fp8_mt(xs, c.rows, c.cols, g, c.eps, c.weight_offset, c.scale_ub,
                                 residual=res, threads=cores)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = per_step * args.steps / dt / 1e9
    sample = (f"first {', '.join(str(r) for r in rows_list)} rows of the "
              f"{len(rows_list)} call(s) per step, {cores} POSIX threads (the cores of this "
              f"process's CPU affinity), one contiguous row chunk each")
    line = {"metric": METRIC, "value": round(value, 6), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": f"{name}: R={w.R}, cols={w.cols}, rows {list(w.rows)} "
                                   f"per step, residual={'on' if w.residual else 'off'}",
                       "sample": sample},
            "cpu_baseline": {"value": round(value, 6), "unit": "GB/s", "cores": cores,
                             "kind": "oracle", "sample": f"{args.steps} steps, {sample}"},
            "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ launch sweep ---

SWEEP_RB = (2, 4, 8, 16)
SWEEP_COLS = (1024, 2048, 4096, 7168, 8192, 16384)
SWEEP_ROWS = (1, 2, 4, 8, 16, 32, 37, 48, 64, 96, 128, 192, 256, 512, 1024, 2048, 8192)
SWEEP_CLUSTERS = (1, 2, 3, 4, 5, 6, 7, 8, 12, 16)
SWEEP_MAX_BYTES = 1600 << 20  # shapes moving more per call are left out


def write_plan_table(out_inc: str, best, gpu: str, sms: int, seconds: float) -> None:
    """The launch table the library compiles: a header comment, then one
    RRF_PLAN(input bound, residual, cols, rows, cluster, prefetch, us) line
    per (rb, residual, cols, rows, cluster, prefetch, us) of `best`."""
    with open(out_inc, "w") as fh:
        fh.write(f"""// rrf_plan_table.inc -- measured launches of the fused call, one
// RRF_PLAN(input bound, residual, cols, rows, cluster, prefetch, us per call)
// per shape: the cluster size and L2-prefetch setting that ran fastest.
// Written by `python bench.py --plan-sweep <this file>` on a {gpu}
// ({sms} SMs), {time.strftime('%Y-%m-%d')}, in {seconds:.0f} s; every
// measurement is in the .json the sweep writes beside its output.  Do not
// edit by hand.
""")
        for rb, res, cols, rows, C, pf, us in best:
            fh.write(f"RRF_PLAN({rb}, {res}, {cols}, {rows}, {C}, {pf}, {us:.3f}f)\n")


def plan_sweep(out_inc: str, rbs=SWEEP_RB, cols_list=SWEEP_COLS, rows_list=SWEEP_ROWS):
    """Measure every launch of the fused call (cluster size x L2 prefetch on
    and off) on a grid of shapes and write the fastest per shape as the
    library's launch table (rrf_plan_table.inc: one RRF_PLAN line per shape)
    plus every measurement beside it (<out>.json).  Each launch is timed as
    the median of five graph replays of back-to-back calls over rotating
    buffer sets larger than 3x L2 (cold HBM, as the benchmark's calls).
    Inputs: the sweep workload's distributions (N(0,1), gamma N(1, 0.1)),
    R = the input bound."""
    import torch
    import reduce_rmsnorm_fp8_b200 as rrf
    device = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(device)
    props = torch.cuda.get_device_properties(device)
    l2 = props.L2_cache_size
    flags_of = {1: rrf.RRF_FLAG_PREFETCH, 0: rrf.RRF_FLAG_NO_PREFETCH}
    records, best = [], []
    t_start = time.perf_counter()
    for rb in rbs:
        for res in (0, 1):
            for cols in cols_list:
                for rows in rows_list:
                    nbytes = workloads.fused_bytes(rb, rows, cols, bool(res))
                    if nbytes > SWEEP_MAX_BYTES:
                        continue
                    c = workloads.make_case("sweep", rows, R=rb, cols=cols, residual=bool(res),
                                            device=device)
                    n_sets = max(2, math.ceil(L2_FLUSH_FACTOR * l2 / nbytes))
                    shape = (n_sets, rows, cols)
                    xs = [x.unsqueeze(0).expand(shape).contiguous() for x in c.inputs]
                    rin = c.residual.unsqueeze(0).expand(shape).contiguous() if res else None
                    rout = torch.empty(shape, dtype=torch.bfloat16, device=device) if res \
                        else None
                    q = torch.empty(shape, dtype=torch.float8_e4m3fn, device=device)
                    sc = torch.empty((n_sets, rows, 1), dtype=torch.float32, device=device)
                    calls = int(min(100, max(8, 1.5e-3 / (nbytes / 5e12 + 3e-6))))

                    def call(k, C, pf):
                        i = k % n_sets
                        rrf.rrf_sum_rmsnorm_fp8_ex(
                            [x[i] for x in xs], c.gamma, c.eps, c.weight_offset, c.scale_ub,
                            residual_in=None if rin is None else rin[i],
                            residual_out=None if rout is None else rout[i], q_out=q[i],
                            scales_out=sc[i], variant=1 if C == 1 else 2,
                            cluster_size=0 if C == 1 else C, flags=flags_of[pf])
                        return 1

                    meas = []
                    for C in SWEEP_CLUSTERS:
                        if C > 1 and cols // 8 // C < 32:
                            continue
                        for pf in (0, 1):
                            try:
                                for i in range(3):
                                    call(i, C, pf)
                            except rrf.RrfError:
                                break  # the block cannot hold this cluster's slice
                            g, _ = capture_steps(lambda k: call(3 + k, C, pf), calls, device)
                            g.replay()
                            torch.cuda.synchronize(device)
                            ts = sorted(time_region(lambda _: g.replay(), 1, device, stream)
                                        for _ in range(5))
                            del g
                            us = ts[2] / calls * 1e6
                            meas.append((us, C, pf))
                            records.append({"rb": rb, "residual": res, "cols": cols,
                                            "rows": rows, "cluster": C, "prefetch": pf,
                                            "us": round(us, 4),
                                            "GB_s": round(nbytes / us / 1e3, 1)})
                    us, C, pf = min(meas)
                    best.append((rb, res, cols, rows, C, pf, us))
                    del xs, rin, rout, q, sc, c
                    print(f"sweep rb={rb} res={res} cols={cols} rows={rows}: C={C} "
                          f"prefetch={pf} {us:.3f} us", file=sys.stderr, flush=True)
                torch.cuda.empty_cache()
    took = time.perf_counter() - t_start
    write_plan_table(out_inc, best, props.name, props.multi_processor_count, took)
    with open(os.path.splitext(out_inc)[0] + ".json", "w") as fh:
        json.dump({"gpu": props.name, "sms": props.multi_processor_count,
                   "clusters": SWEEP_CLUSTERS, "records": records}, fh)
    print(json.dumps({"plan_sweep": out_inc, "shapes": len(best), "measurements": len(records),
                      "seconds": round(took, 1)}), flush=True)


def run_gemm_only(M: int, N: int, K: int, mx: bool = False):
    """One GEMM shape through time_gemm or time_gemm_mx (3 eager calls, then
    graph replays), for profiling; prints its record."""
    import torch

    import reduce_rmsnorm_fp8_b200 as rrf
    device = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(device)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    fn, key = (time_gemm_mx, "gemm_mxfp8") if mx else (time_gemm, "gemm_fp8")
    rec = fn(rrf, M, N, K, device, stream, l2, measured_peaks()[0])
    print(json.dumps({key: rec}), flush=True)


def run_one_secondary(key, fn, *args):
    """One secondary measurement alone (profiling runs); prints its record."""
    import torch

    import reduce_rmsnorm_fp8_b200 as rrf
    device = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(device)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    if fn is time_sharded:
        rec = fn(rrf, *args, device, stream, l2, measured_peaks()[0])
    else:
        rec = fn(rrf, *args, device, stream, l2)
    print(json.dumps({key: rec}), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description="fused sum + RMSNorm + FP8 benchmark")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["rrf", "reference"], default="rrf")
    ap.add_argument("--workload", choices=sorted(workloads.WORKLOADS), default="prefill")
    ap.add_argument("--replays", type=int, default=5,
                    help="timed replays of the K-step graph (the value is their median)")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--rows", type=int, nargs="*", default=None,
                    help="only these row counts of the workload (profiling runs)")
    ap.add_argument("--no-breakdown", action="store_true",
                    help="skip the per-call breakdown")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--gemm", type=int, nargs=3, metavar=("M", "N", "K"), default=None,
                    help="time only the FP8 GEMM of this shape (profiling runs)")
    ap.add_argument("--gemm-mx", type=int, nargs=3, metavar=("M", "N", "K"), default=None,
                    help="time only the MX GEMM of this shape (profiling runs)")
    ap.add_argument("--allreduce", nargs=4, metavar=("WORKLOAD", "ROWS", "RANKS", "MODE"),
                    default=None, help="time only the multi-GPU call, all ranks in one launch "
                                       "(MODE 0 auto, 1 one-shot, 2 two-shot; profiling runs)")
    ap.add_argument("--sharded", nargs=4, metavar=("WORKLOAD", "ROWS", "COLS", "SHARDS"),
                    default=None, help="time only the two phases of the sharded form on one "
                                       "shard (profiling runs)")
    ap.add_argument("--plan-sweep", metavar="OUT_INC", default=None,
                    help="measure the fused call's launches on a grid of shapes and write "
                         "the launch table (reduce_rmsnorm_fp8_b200/csrc/rrf_plan_table.inc; "
                         "rebuild the library afterwards) and OUT_INC's .json")
    ap.add_argument("--plan-sweep-shapes", nargs=3, metavar=("RB", "COLS", "ROWS"),
                    default=None, help="comma lists restricting the sweep's grid")
    args = ap.parse_args(argv)
    global ROWS_OVERRIDE
    if args.rows:
        ROWS_OVERRIDE = tuple(args.rows)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.plan_sweep is not None:
        grid = {}
        if args.plan_sweep_shapes:
            lists = [tuple(int(v) for v in x.split(",")) for x in args.plan_sweep_shapes]
            grid = dict(rbs=lists[0], cols_list=lists[1], rows_list=lists[2])
        plan_sweep(args.plan_sweep, **grid)
    elif args.gemm is not None:
        run_gemm_only(*args.gemm)
    elif args.gemm_mx is not None:
        run_gemm_only(*args.gemm_mx, mx=True)
    elif args.allreduce is not None:
        w, rows, ranks, mode = args.allreduce
        run_one_secondary("allreduce_emulated", time_allreduce, w, int(rows), int(ranks),
                          int(mode))
    elif args.sharded is not None:
        w, rows, cols, shards = args.sharded
        run_one_secondary("sharded", time_sharded, w, int(rows), int(cols), int(shards))
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_rrf(args)


if __name__ == "__main__":
    main()

"""Benchmark of the BitLinear training hot path (fwd + bwd) on B200.

One step = one pass of the whole hot path over one batch:
  S1 + S2 bl_quantize (2 launches: |W| partial sums with part of the token
  rows, then gamma and the codes with the other rows) -> S3 bl_forward
  -> S4 bl_backward with its x_hat workspace (for N >= 2048 one launch makes
  x_hat, then dX and dW in one launch)                   (4 or 5 launches)

Default workload: the up-projection BitLinear 2560 -> 6912 at 8 x 512 tokens
(M=4096, K=2560, N=6912; x, dY bf16 ~ N(0,1), W bf16 kaiming-uniform).
Metric: effective TOPS = 6 M N K / step time (plus ms per step and the
roofline fraction of the dominant kernel).

Timing: W >= 3 untimed warm-up steps, then exactly K timed steps on
resident inputs. L2 is flushed (256 MiB written, then read back, so that no
dirty line is left) before every step, outside the timed events; each step is bracketed by CUDA events on the launching
stream (the headline); a second pass of K steps puts events between the C-ABI
calls (`ms_isolated` per kernel: one launch after a flush, with the launch
latency an event in front of it costs). The per-kernel times the roofline
fractions use come from CUDA graphs of 16 back-to-back calls of one stage over
4 rotating sets of inputs and outputs (more than L2 between reuses), replayed
between two events: each launch's average duration in a stream. For N > 1
(torchrun, one rank per GPU) the step is the data-parallel one: every rank
runs the path on its own tokens (weak scaling) with the same W, and the
partial dW are summed over the ranks by an NCCL all-reduce inside the timed
step (the path's one exchange); the job time is the max over ranks.

`--impl reference` times the CPU oracle (the only reference this path has)
on a bounded sample of the same workload, on the host cores.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import WORKLOADS, workload_inputs  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_OVER_BF16 = 2.0  # nominal dense ratio (4.5 / 2.25 PFLOP/s)
KERNEL_SOURCES = ["ternary_weight_quantization_b200/csrc/k_quant.cu",
                  "ternary_weight_quantization_b200/csrc/k_gemm.cu",
                  "ternary_weight_quantization_b200/csrc/bl_device.cuh",
                  "ternary_weight_quantization_b200/csrc/bl_abs_sum.cuh"]


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash():
    """Hash of the kernel sources' code (line comments and blank lines
    dropped, so editing a comment does not invalidate captured counters)."""
    import hashlib
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            for line in f:
                code = line.split("//", 1)[0].rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def load_traffic(workload):
    """Per-launch DRAM bytes from a committed ncu capture, if it matches the
    current kernel sources (else None)."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except Exception:
        return {}
    if t.get("source_hash") != kernel_source_hash():
        return {}
    return t.get("workloads", {}).get(workload, {})


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons with NVML in a background thread."""

    BAD = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}

    def __init__(self, device_index, period_s=0.005):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.period = period_s
            self.ok = True
        except Exception:
            self.ok = False

    def _reason_names(self, mask):
        nv = self.nv
        table = {
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "hw_power_brake_slowdown": getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }
        return {k for k, v in table.items() if mask & v}

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                try:
                    mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    mask = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.reasons |= self._reason_names(mask)
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t:
            self._stop.set()
            self._t.join()
        s = sorted(self.samples)
        med = s[len(s) // 2] if s else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(s), "source": "nvml" if self.ok else "unavailable"}

    def rejected(self, rec):
        return bool(self.BAD & set(rec["reasons"]))


# ----------------------------------------------------------------- multi-rank aggregation

def job_time_ms(local_ms: float, world: int, device=None) -> float:
    """Device time of the whole job: the max over ranks (all ranks call)."""
    if world <= 1:
        return float(local_ms)
    t = torch.tensor([float(local_ms)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_tops(ops_per_rank_step: float, world: int, steps: int, job_ms: float) -> float:
    """Whole-job throughput: every rank's work divided by the job time."""
    return ops_per_rank_step * world * steps / (job_ms * 1e-3) / 1e12


# ----------------------------------------------------------------- our arm

STAGES = ["quantize", "forward", "backward"]


def launches_per_step(N):
    """S1 sums (+ S2 rows); S1 codes (+ S2 rows); S3; S4: dX and dW in one
    launch, after one that makes x_hat in the backward's workspace where dW
    has N >= 2048 features (below that the library rebuilds x_hat instead)."""
    return 5 if N >= 2048 else 4


def stage_work(M, N, K, w_bytes):
    """Algorithmic work per launch group: bytes for the HBM passes, ops for GEMMs."""
    return {
        "quantize": {"bound": "hbm", "bytes": N * K * w_bytes + N * K // 4 + 4 + M * K * 2 + M * K + 4 * M},
        "forward": {"bound": "tensor", "ops": 2 * M * N * K, "dtype": "int8"},
        "backward": {"bound": "tensor", "ops": 4 * M * N * K, "dtype": "bf16"},
    }


def stage_graph_ms(bl, x, w, dy, M, N, K, dev, n_sets=4, calls=16, reps=5):
    """Per-call device time of each stage: `calls` back-to-back C-ABI calls of
    the stage, over n_sets rotating copies of its inputs and outputs (between
    two uses of one set the other sets move well over the 126 MB of L2),
    captured in one CUDA graph and replayed between two events after an L2
    flush; the median over `reps` replays, divided by `calls`. This is each
    launch's average duration inside a stream of launches, without host launch
    gaps or the cost of an event around every launch."""
    sets = []
    for _ in range(n_sets):
        b = bl.StepBuffers.allocate(M, N, K, torch.bfloat16, device=dev)
        xs, ws_, dys = x.clone(), w.clone(), dy.clone()
        bl.bl_quantize(ws_, xs, b.w_packed, b.gamma, b.xq, b.sx, b.workspace)
        sets.append((xs, ws_, dys, b))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    calls_of = {
        "quantize": lambda t: bl.bl_quantize(t[1], t[0], t[3].w_packed, t[3].gamma, t[3].xq, t[3].sx, t[3].workspace),
        "forward": lambda t: bl.bl_forward(t[3].xq, t[3].sx, t[3].w_packed, t[3].gamma, t[3].y, None),
        "backward": lambda t: bl.bl_backward(t[2], t[3].xq, t[3].sx, t[3].w_packed, t[3].gamma, t[3].dX, t[3].dW,
                                             False, workspace=t[3].bwd_workspace),
    }
    out = {}
    for name, call in calls_of.items():
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            for i in range(n_sets):
                call(sets[i])
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            for i in range(calls):
                call(sets[i % n_sets])
        ts = []
        for r in range(reps + 1):
            flush.fill_(r & 0xFF)
            flush.view(torch.int64).max()
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            g.replay()
            e.record()
            torch.cuda.synchronize(dev)
            if r > 0:
                ts.append(s.elapsed_time(e) / calls)
        del g
        out[name] = sorted(ts)[len(ts) // 2]
    if bl.bl_get_last_error() != 0:
        raise RuntimeError("device error during the per-stage graph timing")
    del sets, flush
    torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world, local_rank):
    import ternary_weight_quantization_b200 as bl
    from ternary_weight_quantization_b200.dp import dp_step

    bl.load_library()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = WORKLOADS[args.workload]
    M, K, N = wl.M, wl.K, wl.N
    # every rank: its own tokens and output gradients, the same W
    x_cpu, w_cpu, dy_cpu = workload_inputs(args.workload, seed=rank)
    if rank != 0:
        w_cpu = workload_inputs(args.workload, seed=0)[1]
    x, w, dy = x_cpu.to(dev), w_cpu.to(dev), dy_cpu.to(dev)
    bufs = bl.StepBuffers.allocate(M, N, K, torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def flush_l2(i):
        # Write a buffer twice the size of L2, then read it back: no workload
        # data stays in L2 and no dirty line is left for the timed kernels to
        # write back.
        flush.fill_(i & 0xFF)
        flush.view(torch.int64).max()

    def step(evs=None):
        if not evs:
            dp_step(x, w, dy, bufs, stream=stream)  # world 1: no exchange
            return
        evs[0].record(stream)
        bl.bl_quantize(w, x, bufs.w_packed, bufs.gamma, bufs.xq, bufs.sx, bufs.workspace, stream)
        evs[1].record(stream)
        bl.bl_forward(bufs.xq, bufs.sx, bufs.w_packed, bufs.gamma, bufs.y, None, stream)
        evs[2].record(stream)
        bl.bl_backward(dy, bufs.xq, bufs.sx, bufs.w_packed, bufs.gamma, bufs.dX, bufs.dW, False, stream,
                       workspace=bufs.bwd_workspace)
        evs[3].record(stream)
        if world > 1:
            with torch.cuda.stream(stream):
                torch.distributed.all_reduce(bufs.dW)
            evs[4].record(stream)

    for i in range(args.warmup):
        flush_l2(i)
        step()
    torch.cuda.synchronize(dev)
    if bl.bl_get_last_error() != 0:
        raise RuntimeError("device error during warm-up")

    # The step's C-ABI calls captured once into a CUDA graph (their tensor maps
    # and launch shapes are fixed by the buffers), then replayed: one host
    # launch per step instead of the Python-side issue of every call, which
    # on a slow host leaves gaps between the step's kernels. Every kernel of
    # the step runs on every replay. The all-reduce of N > 1 is issued after
    # each replay, outside the graph.
    def compute(st):
        bl.bl_quantize(w, x, bufs.w_packed, bufs.gamma, bufs.xq, bufs.sx, bufs.workspace, st)
        bl.bl_forward(bufs.xq, bufs.sx, bufs.w_packed, bufs.gamma, bufs.y, None, st)
        bl.bl_backward(dy, bufs.xq, bufs.sx, bufs.w_packed, bufs.gamma, bufs.dX, bufs.dW, False, st,
                       workspace=bufs.bwd_workspace)

    graph = None
    if not args.eager:
        graph = torch.cuda.CUDAGraph()
        # thread-local capture: CUDA calls of other threads (the process
        # group's watchdog under torchrun) do not invalidate the capture
        with torch.cuda.graph(graph, capture_error_mode="thread_local"):
            compute(torch.cuda.current_stream(dev))
        torch.cuda.synchronize(dev)

    def graph_step():
        graph.replay()
        if world > 1:
            torch.distributed.all_reduce(bufs.dW)

    for i in range(args.warmup if graph is not None else 0):
        flush_l2(i)
        graph_step()
    torch.cuda.synchronize(dev)

    def timed(per_stage, replay=False):
        """K steps, L2 flushed before each. per_stage: events between the C-ABI
        calls (kernel breakdown); otherwise events only around each step, so
        consecutive kernels keep their programmatic-launch overlap. replay:
        the step as the captured graph (plus the all-reduce for N > 1)."""
        n_ev = len(STAGES) + 1 + (world > 1) if per_stage else 2
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        for i in range(args.steps):
            flush_l2(i)
            if per_stage:
                step(evs[i])
            else:
                evs[i][0].record(stream)
                graph_step() if replay else step()
                evs[i][1].record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        names = STAGES + (["allreduce"] if world > 1 else [])
        per = {s: 0.0 for s in names}
        total = 0.0
        for e in evs:
            if per_stage:
                for j, st in enumerate(names):
                    per[st] += e[j].elapsed_time(e[j + 1])
            total += e[0].elapsed_time(e[-1])
        return total, per

    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    sampler.start()
    total_ms, _ = timed(False, graph is not None)
    clocks = sampler.stop()
    remeasured = False
    if sampler.rejected(clocks):
        sampler = ClockSampler(dev.index if dev.index is not None else 0)
        sampler.start()
        total_ms, _ = timed(False, graph is not None)
        clocks = sampler.stop()
        remeasured = True
    eager_ms = timed(False)[0] if graph is not None else total_ms
    del graph
    breakdown_ms, per_stage = timed(True)
    clocks["remeasured"] = remeasured
    graph_ms = stage_graph_ms(bl, x, w, dy, M, N, K, dev)
    if bl.bl_get_last_error() != 0:
        raise RuntimeError("device error during the timed region")

    job_ms = job_time_ms(total_ms, world, dev)
    eager_job_ms = job_time_ms(eager_ms, world, dev)

    e2e = measure_e2e(bl, args, dev, stream, bufs, x_cpu, w_cpu, dy_cpu, world)
    if rank != 0:
        return None

    ops_step = 6.0 * M * N * K
    ms_per_step = job_ms / args.steps
    value = job_tops(ops_step, world, args.steps, job_ms)
    peaks, peak_src = load_peaks()
    work = stage_work(M, N, K, 2 if wl.w_dtype == torch.bfloat16 else 4)
    traffic = load_traffic(args.workload)
    kernels = {}
    roof_ms = 0.0
    for s in STAGES:
        ms = graph_ms[s]
        wk = work[s]
        if wk["bound"] == "hbm":
            ach = wk["bytes"] / (ms * 1e-3) / 1e9
            peak = peaks["hbm_gbs"]
            unit = "GB/s"
            roof_ms += wk["bytes"] / (peak * 1e9) * 1e3
        else:
            ach = wk["ops"] / (ms * 1e-3) / 1e12
            peak = peaks["bf16_tflops"] * (INT8_OVER_BF16 if wk["dtype"] == "int8" else 1.0)
            unit = "TOPS" if wk["dtype"] == "int8" else "TFLOP/s"
            roof_ms += wk["ops"] / (peak * 1e12) * 1e3
        kernels[s] = {"ms": round(ms, 5), "achieved": round(ach, 1), "unit": unit, "peak": peak,
                      "frac": round(ach / peak, 4), "share": round(graph_ms[s] / sum(graph_ms[t] for t in STAGES), 4),
                      "ms_isolated": round(per_stage[s] / args.steps, 5), "traffic": traffic.get(s)}
    dom = max(STAGES, key=lambda s: graph_ms[s])
    dk = kernels[dom]
    roofline = {"kernel": dom, "bound": work[dom]["bound"], "achieved": dk["achieved"], "peak": dk["peak"],
                "unit": "GB/s" if work[dom]["bound"] == "hbm" else "TFLOP/s", "frac": dk["frac"],
                "traffic": dk["traffic"], "peak_source": f"{peak_src} (burst bf16"
                + (" x2 nominal int8/bf16 ratio" if work[dom].get("dtype") == "int8" else "") + ")"
                if work[dom]["bound"] == "tensor" else f"{peak_src} hbm copy"}
    out = {
        "metric": "bitlinear_fwd_bwd_effective_tops", "value": round(value, 2), "unit": "TOPS",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8/bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, "M": M, "K": K, "N": N,
                   "x": f"bf16 [{M},{K}] N(0,1)" + (" + 1% x20 outliers" if wl.outliers else ""),
                   "W": f"{'bf16' if wl.w_dtype == torch.bfloat16 else 'f32'} [{N},{K}] {wl.w_init}",
                   "dY": f"bf16 [{M},{N}] N(0,1)", "global_batch_tokens": M * world,
                   "l2": "flushed before every step (256 MiB write then read, outside the timed events)",
                   "parallelism": f"dp{world}: token shards, dW all-reduce (NCCL) in the step"
                   if world > 1 else "single GPU"},
        "roofline": roofline,
        "step_roofline_frac": round(roof_ms / ms_per_step, 4),
        "launch": "one CUDA graph replay per step (the step's C-ABI calls captured once)"
        if not args.eager else "the step's C-ABI calls issued from Python every step",
        "ms_per_step_eager": round(eager_job_ms / args.steps, 5),
        "kernel_breakdown_ms_per_step": round(breakdown_ms / args.steps, 5),
        "kernels": kernels,
        **({"allreduce_ms_per_step": round(per_stage["allreduce"] / args.steps, 5),
            "allreduce_bytes": bufs.dW.numel() * bufs.dW.element_size()} if world > 1 else {}),
        "e2e": e2e,
        "gpu_launches": launches_per_step(N) * args.steps,
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args.workload, budget_tokens=args.cpu_tokens)
    return out


def measure_e2e(bl, args, dev, stream, bufs, x_cpu, w_cpu, dy_cpu, world):
    """Same metric through the C ABI with host buffers: every step copies its
    inputs (x, W, dY) from pinned host memory to the device, runs the step
    (`dp_step`, the public call) and copies its results (y, dX, dW) back, all
    inside the timed region. Steps are pipelined the way a training loop
    feeds a GPU: two sets of device buffers, the host-to-device copies on one
    stream, the step on another and the device-to-host copies on a third, so
    that step i's results travel back while step i + 1's inputs travel in
    (PCIe is full duplex) and the step's kernels run between them; events
    order each set's copies, step and read-back."""
    from ternary_weight_quantization_b200.dp import dp_step

    M, K = x_cpu.shape
    N = w_cpu.shape[0]
    hin = [(x_cpu.pin_memory(), w_cpu.pin_memory(), dy_cpu.pin_memory())]
    hin.append(tuple(t.clone().pin_memory() for t in hin[0]))
    sets = [(torch.empty_like(x_cpu, device=dev), torch.empty_like(w_cpu, device=dev),
             torch.empty_like(dy_cpu, device=dev), bl.StepBuffers.allocate(M, N, K, bufs.dW.dtype, device=dev))
            for _ in range(2)]
    hout = [tuple(torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (st[3].y, st[3].dX, st[3].dW))
            for st in sets]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    s_run = stream
    steps = max(3, min(args.steps, 20))
    freed = [None, None]  # event: the set's previous results have left the device

    def one(i):
        k = i % 2
        (x, w, dy, b), (xh, wh, dyh), (yh, dxh, dwh) = sets[k], hin[k], hout[k]
        if freed[k] is not None:
            s_in.wait_event(freed[k])
        with torch.cuda.stream(s_in):
            x.copy_(xh, non_blocking=True)
            w.copy_(wh, non_blocking=True)
            dy.copy_(dyh, non_blocking=True)
        ready = torch.cuda.Event()
        ready.record(s_in)
        s_run.wait_event(ready)
        dp_step(x, w, dy, b, stream=s_run)
        done = torch.cuda.Event()
        done.record(s_run)
        s_out.wait_event(done)
        with torch.cuda.stream(s_out):
            yh.copy_(b.y, non_blocking=True)
            dxh.copy_(b.dX, non_blocking=True)
            dwh.copy_(b.dW, non_blocking=True)
        freed[k] = torch.cuda.Event()
        freed[k].record(s_out)

    for i in range(2):
        one(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    for i in range(steps):
        one(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_run)
    end.record(s_out)
    torch.cuda.synchronize(dev)
    ms = job_time_ms(start.elapsed_time(end), world, dev)
    h2d = sum(tt.numel() * tt.element_size() for tt in hin[0])
    d2h = sum(tt.numel() * tt.element_size() for tt in hout[0])
    del sets
    torch.cuda.empty_cache()
    return {"value": round(job_tops(6.0 * M * N * K, world, steps, ms), 3), "unit": "TOPS",
            "ms_per_step": round(ms / steps, 4), "steps": steps,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipelining": "two buffer sets; H2D, step and D2H on three streams (step i's D2H overlaps step i+1's H2D)"}


# ----------------------------------------------------------------- oracle (CPU)

def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [i.get("num_threads", 0) for i in info if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


_INPUT_CACHE = {}


def oracle_sample(workload, m_tokens, n_rows):
    """Run the oracle's fwd+bwd on the first m_tokens tokens and n_rows output
    features of the workload (full K). Returns (seconds, ops)."""
    import numpy as np
    from oracle import bitlinear_ref as ref

    if workload not in _INPUT_CACHE:
        _INPUT_CACHE[workload] = workload_inputs(workload)
    x, w, dy = _INPUT_CACHE[workload]
    x = x[:m_tokens]
    w = w[:n_rows]
    dy = dy[:m_tokens, :n_rows].contiguous()

    def b(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    w_is_bf16 = w.dtype == torch.bfloat16
    t0 = time.perf_counter()
    ref.bitlinear_step(b(x), b(w) if w_is_bf16 else w.numpy(), b(dy), w_is_bf16)
    dt = time.perf_counter() - t0
    return dt, 6.0 * x.shape[0] * w.shape[0] * x.shape[1]


def cpu_baseline(workload, budget_tokens=512):
    wl = WORKLOADS[workload]
    m = min(budget_tokens, wl.M)
    dt, ops = oracle_sample(workload, m, wl.N)
    return {"value": round(ops / dt / 1e12, 6), "unit": "TOPS", "cores": _blas_threads(), "kind": "oracle",
            "seconds": round(dt, 3),
            "sample": f"first {m} of {wl.M} tokens, all {wl.N} output features, K={wl.K} "
                      f"(S1 on the full weight); TOPS = 6*{m}*{wl.N}*{wl.K} / time"}


def run_reference(args):
    wl = WORKLOADS[args.workload]
    m, n = min(64, wl.M), min(512, wl.N)
    for _ in range(args.warmup):
        oracle_sample(args.workload, m, n)
    total = 0.0
    ops = 0.0
    for _ in range(args.steps):
        dt, o = oracle_sample(args.workload, m, n)
        total += dt
        ops += o
    value = ops / total / 1e12
    sample = f"first {m} of {wl.M} tokens and first {n} of {wl.N} output features, K={wl.K}, per step"
    return {
        "impl": "reference", "metric": "bitlinear_fwd_bwd_effective_tops", "value": round(value, 6), "unit": "TOPS",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "M": wl.M, "K": wl.K, "N": wl.N},
        "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": _blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------- main

def run_stack(args, rank, world, local_rank):
    """Layer-stack mode: the 8-layer stack workload (8 BitLinear layers alternating
    2560 -> 6912 -> 2560, 2048 tokens). One step = the forward of every layer
    (bl_quantize + bl_forward, only the 2-bit / INT8 state kept) and the
    backward of every layer in reverse (bl_backward, dX feeding the layer
    below). Reports the step time, effective TOPS and the peak device memory."""
    import ternary_weight_quantization_b200 as bl
    from ternary_weight_quantization_b200.stack import BitLinearStack
    from workloads import STACKS, stack_inputs

    bl.load_library()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    M, dims = STACKS[args.stack]
    x_cpu, ws_cpu, dy_cpu = stack_inputs(M, dims, seed=rank)
    torch.cuda.reset_peak_memory_stats(dev)
    base = torch.cuda.memory_allocated(dev)
    x, dy = x_cpu.to(dev), dy_cpu.to(dev)
    ws = [w.to(dev) for w in ws_cpu]
    st = BitLinearStack.allocate(M, dims, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(s=stream):
        st.forward(x, ws, s)
        st.backward(dy, True, s)

    for i in range(args.warmup):
        flush.fill_(i & 0xFF)
        flush.view(torch.int64).max()
        step()
    torch.cuda.synchronize(dev)
    if bl.bl_get_last_error() != 0:
        raise RuntimeError("device error during warm-up")
    peak_mb = (torch.cuda.max_memory_allocated(dev) - base - flush.numel()) / 1e6
    # the step's calls captured once into a CUDA graph and replayed (every
    # kernel of the step on every replay), as in the single-layer mode
    graph = None
    if not args.eager:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, capture_error_mode="thread_local"):
            step(torch.cuda.current_stream(dev))
        torch.cuda.synchronize(dev)

    def timed(replay):
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            flush.view(torch.int64).max()
            evs[i][0].record(stream)
            graph.replay() if replay else step()
            evs[i][1].record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        return sum(e[0].elapsed_time(e[1]) for e in evs)

    if graph is not None:
        timed(True)  # warm-up replays
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    sampler.start()
    total = timed(graph is not None)
    clocks = sampler.stop()
    eager_total = timed(False) if graph is not None else total
    del graph
    if bl.bl_get_last_error() != 0:
        raise RuntimeError("device error during the timed region")
    job_ms = job_time_ms(total, world, dev)
    eager_job_ms = job_time_ms(eager_total, world, dev)
    if rank != 0:
        return None
    ops_step = 6.0 * M * sum(k * n for k, n in zip(dims[:-1], dims[1:]))
    saved = sum(L.xq.numel() + 4 * L.sx.numel() + L.w_packed.numel() + 4 for L in st.layers)
    return {
        "metric": "bitlinear_stack_fwd_bwd_effective_tops", "value": round(job_tops(ops_step, world, args.steps,
                                                                                     job_ms), 2),
        "unit": "TOPS", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(job_ms / args.steps, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8/bf16", "data": "synthetic",
        "config": {"workload": args.stack, "M": M, "dims": dims, "layers": len(dims) - 1,
                   "l2": "flushed before every step (256 MiB written, then read back)",
                   "parallelism": f"dp{world} independent replicas" if world > 1 else "single GPU"},
        "launch": "one CUDA graph replay per step (the step's C-ABI calls captured once)"
        if not args.eager else "the step's C-ABI calls issued from Python every step",
        "ms_per_step_eager": round(eager_job_ms / args.steps, 5),
        "peak_device_memory_mb": round(peak_mb, 1),
        "saved_state_mb": round(saved / 1e6, 2),
        "gpu_launches": sum(launches_per_step(n) for n in dims[1:]) * args.steps,
        "clocks": clocks,
    }


def run_few_tokens(args, rank, world, local_rank):
    """Few-token mode: the forward alone at M in --few-tokens on the
    up-projection weight (N 6912, K 2560). With a handful of tokens it is
    bound by reading the packed codes once, so the line reports achieved
    HBM GB/s (codes + q + s_x read, y written) against the measured copy
    bandwidth, per M: from back-to-back launches in a CUDA graph, each on
    another copy of the weight, and (ms_isolated) from single launches."""
    import ternary_weight_quantization_b200 as bl
    from workloads import make_inputs

    bl.load_library()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    N, K = 6912, 2560
    _, w, _ = make_inputs(8, K, N, seed=rank)
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device=dev)
    gamma = torch.empty(1, dtype=torch.float32, device=dev)
    ws = torch.empty(max(bl.bl_quantize_weight_workspace_size(N, K), 16), dtype=torch.uint8, device=dev)
    bl.bl_quantize_weight(w.to(dev), packed, gamma, ws)
    copies = [packed.clone() for _ in range(48)]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    peaks, peak_src = load_peaks()
    rows = {}
    for M in [int(v) for v in args.few_tokens.split(",")]:
        x, _, _ = make_inputs(M, K, 8, seed=rank + M)
        xq = torch.empty((M, K), dtype=torch.int8, device=dev)
        sx = torch.empty(M, dtype=torch.float32, device=dev)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        bl.bl_quantize_act(x.to(dev), xq, sx)
        times = []
        for i in range(args.warmup + args.steps):
            flush.fill_(i & 0xFF)
            flush.view(torch.int64).max()
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            bl.bl_forward(xq, sx, packed, gamma, y)
            e.record()
            torch.cuda.synchronize(dev)
            if i >= args.warmup:
                times.append(s.elapsed_time(e))
        ms_iso = sum(times) / len(times)
        # back-to-back launches, each on its own copy of the packed weight
        # (48 copies, 212 MB: none is in L2 when its turn comes), captured in
        # a CUDA graph: the launch duration in a stream of decode launches
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            for c in copies[:2]:
                bl.bl_forward(xq, sx, c, gamma, y)
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            for c in copies:
                bl.bl_forward(xq, sx, c, gamma, y)
        gt = []
        for r in range(6):
            flush.fill_(r & 0xFF)
            flush.view(torch.int64).max()
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            g.replay()
            e.record()
            torch.cuda.synchronize(dev)
            if r > 0:
                gt.append(s.elapsed_time(e) / len(copies))
        del g
        ms = sorted(gt)[len(gt) // 2]
        nbytes = N * K // 4 + M * K + 4 * M + 4 + M * N * 2
        gbs = nbytes / (ms * 1e-3) / 1e9
        rows[str(M)] = {"ms": round(ms, 5), "bytes": nbytes, "achieved_gbs": round(gbs, 1),
                        "frac": round(gbs / peaks["hbm_gbs"], 4), "ms_isolated": round(ms_iso, 5)}
    if bl.bl_get_last_error() != 0:
        raise RuntimeError("device error")
    if rank != 0:
        return None
    return {"metric": "bitlinear_forward_few_tokens_gbs", "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "dtype": "int8", "data": "synthetic",
            "config": {"workload": "up_proj weight, forward only", "N": N, "K": K,
                       "l2": "ms: CUDA graph of 48 back-to-back launches, each on its own copy of the packed "
                             "weight (212 MB in all), after a flush; ms_isolated: one launch after a flush "
                             "(256 MiB written, then read back)"},
            "peak_gbs": peaks["hbm_gbs"], "peak_source": f"{peak_src} hbm copy", "by_tokens": rows}


def run_signsgd(args, rank, world, local_rank):
    """Sign-gradient data-parallel mode at up_proj: every rank quantises its
    tokens, runs forward and backward with the 2-bit codes it holds -- the
    backward writing dX and the sign words of dW, not dW
    (bl_backward_signs) -- and sends the words to rank 0, which alone holds
    the master W, votes, updates W and re-ternarises (bl_signsgd_apply: the
    vote, the update and the |W| sums in one sweep, then the code launch) and
    broadcasts the new codes. The line reports the whole step (6 M N K per
    rank over the max-over-ranks time), the same step unfused
    (`unfused_ms_per_step`: dW written and packed by bl_sign_pack, then
    bl_sign_vote, bl_signsgd_update and bl_quantize_weight) and, per
    sign-gradient call, achieved HBM GB/s against the copy bandwidth."""
    import ternary_weight_quantization_b200 as bl
    from ternary_weight_quantization_b200.signsgd import SignBuffers, SignOps, signsgd_dp_step
    from workloads import workload_inputs

    bl.load_library()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    x_cpu, w_cpu, dy_cpu = workload_inputs("up_proj", seed=rank)
    M, K = x_cpu.shape
    N = w_cpu.shape[0]
    holder = rank == 0
    x, dy = x_cpu.to(dev), dy_cpu.to(dev)
    master = w_cpu.to(dev) if holder else None
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device=dev)
    gamma = torch.empty(1, dtype=torch.float32, device=dev)
    ws = torch.empty(max(bl.bl_quantize_weight_workspace_size(N, K), 16), dtype=torch.uint8, device=dev)
    xq = torch.empty((M, K), dtype=torch.int8, device=dev)
    sx = torch.empty(M, dtype=torch.float32, device=dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    dW = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    buf = SignBuffers.allocate(N, K, world, holder, dev)
    lr = 2.0 ** -12
    if holder:
        bl.bl_quantize_weight(master, packed, gamma, ws)
    if world > 1:
        torch.distributed.broadcast(packed, src=0)
        torch.distributed.broadcast(gamma, src=0)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    words = torch.empty((N, K // 32), dtype=torch.int32, device=dev)
    bws = torch.empty(max(bl.bl_backward_workspace_size(M, N, K), 16), dtype=torch.uint8, device=dev)

    def step():
        bl.bl_quantize_act(x, xq, sx)
        bl.bl_forward(xq, sx, packed, gamma, y)
        bl.bl_backward_signs(dy, xq, sx, packed, gamma, dX, words, workspace=bws)
        signsgd_dp_step(None, packed, gamma, lr, master_W=master, workspace=ws if holder else None, buffers=buf,
                        words=words)

    three_calls = SignOps(apply=None)

    def step_unfused():
        bl.bl_quantize_act(x, xq, sx)
        bl.bl_forward(xq, sx, packed, gamma, y)
        bl.bl_backward(dy, xq, sx, packed, gamma, dX, dW, workspace=bws)
        signsgd_dp_step(dW, packed, gamma, lr, master_W=master, workspace=ws if holder else None, buffers=buf,
                        ops=three_calls)

    # the two forms of the step alternate, so that both see the same clocks
    times = {step: [], step_unfused: []}
    for i in range(args.warmup + args.steps):
        for fn in (step, step_unfused):
            flush.fill_(i & 0xFF)
            flush.view(torch.int64).max()
            if world > 1:
                torch.distributed.barrier()
            torch.cuda.synchronize(dev)
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record(stream)
            fn()
            e.record(stream)
            torch.cuda.synchronize(dev)
            if i >= args.warmup:
                times[fn].append(s.elapsed_time(e))
    job_ms = job_time_ms(sum(times[step]) / len(times[step]), world, dev)
    unfused_ms = job_time_ms(sum(times[step_unfused]) / len(times[step_unfused]), world, dev)

    # breakdown of the holder's sign-gradient kernels (events between the calls)
    peaks, peak_src = load_peaks()
    kern = {}
    if holder:
        calls = {
            "sign_pack": (lambda: bl.bl_sign_pack(dW, words), N * K * 2 + N * K // 8),
            "sign_vote": (lambda: bl.bl_sign_vote(buf.gathered, buf.direction), world * N * K // 8 + N * K // 4),
            "signsgd_update": (lambda: bl.bl_signsgd_update(master, buf.direction, 0.0),
                               2 * N * K * 2 + N * K // 4),
            "quantize_weight": (lambda: bl.bl_quantize_weight(master, packed, gamma, ws), N * K * 2 + N * K // 4),
            # vote + update + new codes: words read, W read and written once, codes written
            "signsgd_apply": (lambda: bl.bl_signsgd_apply(buf.gathered, master, 0.0, packed, gamma, ws),
                              world * N * K // 8 + 2 * N * K * 2 + N * K // 4),
        }
        for name, (fn, nbytes) in calls.items():
            ts = []
            for i in range(args.warmup + min(args.steps, 50)):
                flush.fill_(i & 0xFF)
                flush.view(torch.int64).max()
                s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                s.record(stream)
                fn()
                e.record(stream)
                torch.cuda.synchronize(dev)
                if i >= args.warmup:
                    ts.append(s.elapsed_time(e))
            ms = sum(ts) / len(ts)
            gbs = nbytes / (ms * 1e-3) / 1e9
            kern[name] = {"ms": round(ms, 5), "bytes": nbytes, "achieved_gbs": round(gbs, 1),
                          "frac": round(gbs / peaks["hbm_gbs"], 4)}
    if bl.bl_get_last_error() != 0:
        raise RuntimeError("device error")
    if rank != 0:
        return None
    ops = 6.0 * M * N * K
    return {"metric": "bitlinear_signsgd_dp_step_tops", "value": round(job_tops(ops, world, 1, job_ms), 2),
            "unit": "TOPS", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(job_ms, 5),
            "unfused_ms_per_step": round(unfused_ms, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8/bf16",
            "data": "synthetic",
            "config": {"workload": "up_proj, sign-gradient data-parallel step", "M": M, "K": K, "N": N,
                       "ranks": world, "lr": lr, "masters": "bf16 on rank 0 only",
                       "l2": "flushed before every step (256 MiB written, then read back)"},
            "peak_gbs": peaks["hbm_gbs"], "peak_source": f"{peak_src} hbm copy", "kernels": kern}


def run_lm(args, rank, world, local_rank):
    """Decoder-LM mode: the 4-layer LM of workloads/lm.py trained through the
    library (every projection a BitLinear call; the rest plain PyTorch in
    fp64, the precision the LM oracle keeps it in) for
    its 50 steps on each rank (independent replicas). Reports tokens per
    second (batch x sequence per step over the mean device time of a step,
    the first step excluded) and the largest |loss - oracle loss| over the
    steps against the stored oracle curve."""
    from ternary_weight_quantization_b200.lm import train_lm
    from workloads.lm import LM_CONFIG, lm_batches, lm_init

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = LM_CONFIG
    losses, ms = train_lm(lm_init(cfg, seed=0), lm_batches(cfg, seed=0), cfg, dev, timing=True)
    job_ms = job_time_ms(ms, world, dev)
    worst = None
    gold_path = os.path.join(ROOT, "tests", "golden", "lm_oracle_losses.json")
    if os.path.exists(gold_path):
        with open(gold_path) as f:
            gold = json.load(f)["losses"]
        worst = max(abs(a - b) for a, b in zip(losses, gold))
    if rank != 0:
        return None
    tokens = cfg.batch * cfg.seq
    return {"metric": "bitlinear_lm_train_tokens_per_s", "value": round(tokens * world / (job_ms * 1e-3), 1),
            "unit": "tokens/s", "n_gpus": world, "steps": cfg.steps, "warmup": 1, "ms_per_step": round(job_ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8/bf16 BitLinear, fp64 rest",
            "data": "synthetic",
            "config": {"workload": "4-layer decoder LM", "layers": cfg.layers, "d": cfg.d, "heads": cfg.heads,
                       "ffn": cfg.ffn, "vocab": cfg.vocab, "seq": cfg.seq, "batch": cfg.batch, "lr": cfg.lr},
            "loss_first": round(losses[0], 6), "loss_last": round(losses[-1], 6),
            "max_abs_dloss_vs_oracle": None if worst is None else round(worst, 6)}


def run_extras(args, local_rank):
    """The other workloads' lines in short form, measured in the same run on
    the same GPU (N = 1 only): the down-projection step, the 8-layer stack
    (step time and peak memory), the few-token forward, the sign-gradient
    step and the decoder LM (throughput and its largest loss gap to the
    stored oracle curve). Each keeps its own mode's timing rules with fewer
    steps; the headline line above is unaffected."""
    import copy
    short = copy.copy(args)
    short.steps, short.warmup = min(args.steps, 20), max(3, min(args.warmup, 5))
    extras = {}

    def keep(line, keys):
        return {k: line[k] for k in keys if k in line}

    down = copy.copy(short)
    down.workload, down.no_cpu_baseline = "down_proj", True
    line = run_ours(down, 0, 1, local_rank)
    extras["down_proj"] = keep(line, ["value", "unit", "ms_per_step", "ms_per_step_eager", "roofline", "kernels",
                                      "clocks"])
    st = copy.copy(short)
    st.stack = "stack8"
    line = run_stack(st, 0, 1, local_rank)
    extras["stack8"] = keep(line, ["value", "unit", "ms_per_step", "ms_per_step_eager", "peak_device_memory_mb",
                                   "saved_state_mb",
                                   "config", "clocks"])
    ft = copy.copy(short)
    ft.few_tokens = "1,2,4,8,16"
    line = run_few_tokens(ft, 0, 1, local_rank)
    extras["few_tokens"] = keep(line, ["by_tokens", "peak_gbs", "config"])
    line = run_signsgd(copy.copy(short), 0, 1, local_rank)
    extras["signsgd"] = keep(line, ["value", "unit", "ms_per_step", "unfused_ms_per_step", "kernels"])
    line = run_lm(copy.copy(short), 0, 1, local_rank)
    extras["lm"] = keep(line, ["value", "unit", "ms_per_step", "loss_first", "loss_last", "max_abs_dloss_vs_oracle",
                               "dtype"])
    torch.cuda.empty_cache()
    return extras


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["up_proj", "down_proj", "tiny"], default="up_proj")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="issue the step's calls from Python every step instead of replaying a CUDA graph of them")
    ap.add_argument("--cpu-tokens", type=int, default=4096)
    ap.add_argument("--stack", choices=["stack8"], default=None,
                    help="layer-stack mode (prints its own line instead of the single-layer one)")
    ap.add_argument("--lm", action="store_true",
                    help="decoder-LM training mode (prints its own line)")
    ap.add_argument("--signsgd", action="store_true",
                    help="sign-gradient data-parallel step mode (prints its own line)")
    ap.add_argument("--few-tokens", default=None,
                    help="forward-only mode at these token counts, e.g. 1,8,16 (prints its own line)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other workloads' short measurements after the headline (N = 1)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        if args.stack:
            out = run_stack(args, rank, world, local_rank)
        elif args.few_tokens:
            out = run_few_tokens(args, rank, world, local_rank)
        elif args.signsgd:
            out = run_signsgd(args, rank, world, local_rank)
        elif args.lm:
            out = run_lm(args, rank, world, local_rank)
        else:
            out = run_ours(args, rank, world, local_rank)
            if world == 1 and not args.no_extras and out is not None:
                out["other_workloads"] = run_extras(args, local_rank)
        if rank == 0 and out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Benchmark of the persistent warp-specialized BF16 GEMM (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload square8192|square4096|llm_up|llm_down|edge4099|edge8192x256|
                                edge127x8191|recsys|square256|all]

A step is one GEMM (one call: the persistent kernel, plus the alignment pre-pass copies when
an operand needs them) over the workload's synthetic inputs, already resident in HBM.
Timing: W untimed warm-up steps; the step is captured into a CUDA graph, and each of the K
timed steps is one replay between two CUDA events on the launching stream.  Workloads whose
data are smaller than twice the L2 cache get a 256 MiB write and a 256 MiB read between steps
(L2 flushed: cold and clean), outside the events; larger ones run back to back.  The K steps are bracketed by a
barrier and a device synchronize; the time is the max over ranks.  The line reports the mean
(value, ms_per_step), median and minimum step time.  A separate sustained leg replays the
step back to back for a few seconds (the part settles at its power cap) and is compared with
the measured sustained peak.  Multi-GPU runs are independent replicas (the GEMM needs no
exchange): value = total FLOPs of all ranks / max time.  `--impl reference` times the fp64
CPU oracle (rank 0 only) on a bounded sample of the same workload.
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
from typing import NamedTuple

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GEMM TFLOP/s (bf16 in, fp32 acc) and % of B200 dense BF16 peak"
UNIT = "TFLOP/s"
SPEC_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
L2_BYTES = 126 * 2 ** 20
FLUSH_BYTES = 256 * 2 ** 20


class Workload(NamedTuple):
    desc: str
    batch: int
    M: int
    N: int
    K: int
    out: str          # "f32", "bf16" or "f16"
    alpha: float
    beta: float
    std_a: float
    std_b: float
    dist: str         # "normal" or "uniform"
    idx: int          # configuration index (seeds)
    in_dtype: str = "bf16"  # operand type: "bf16" or "f16"
    n_unique: int = 0       # > 0: deduplicated batch, X holds this many distinct entries and
                            # item b uses entry b * n_unique // batch (consecutive items share)


# name -> Workload(description, batch, M, N, K, out, alpha, beta, std_a, std_b, dist, config
# index[, operand type])
WORKLOADS = {
    "square256": ("single GEMM M=N=K=256, U[-1,1], fp32 out", 1, 256, 256, 256, "f32", 1.0, 0.0,
                  1.0, 1.0, "uniform", 0),
    "square4096": ("square GEMM M=N=K=4096, N(0,1), bf16 out", 1, 4096, 4096, 4096, "bf16", 1.0, 0.0,
                   1.0, 1.0, "normal", 1),
    "square8192": ("square GEMM M=N=K=8192, N(0,1), bf16 out", 1, 8192, 8192, 8192, "bf16", 1.0, 0.0,
                   1.0, 1.0, "normal", 1),
    "llm_up": ("LLM MLP up-proj M=16384 N=28672 K=8192, act N(0,1), W N(0,0.02), bf16 out", 1, 16384,
               28672, 8192, "bf16", 1.0, 0.0, 1.0, 0.02, "normal", 2),
    "llm_down": ("LLM MLP down-proj M=16384 N=8192 K=28672, act N(0,1), W N(0,0.02), bf16 out", 1,
                 16384, 8192, 28672, "bf16", 1.0, 0.0, 1.0, 0.02, "normal", 2),
    "edge4099": ("edge GEMM M=N=K=4099 packed ld, alpha=0.5 beta=1, bf16 C in place", 1, 4099, 4099,
                 4099, "bf16", 0.5, 1.0, 1.0, 1.0, "normal", 3),
    "edge8192x256": ("edge GEMM M=8192 N=256 K=4096, alpha=0.5 beta=1, bf16 C in place", 1, 8192, 256,
                     4096, "bf16", 0.5, 1.0, 1.0, 1.0, "normal", 3),
    "edge127x8191": ("edge GEMM M=127 N=8191 K=2048 packed ld, alpha=0.5 beta=1, bf16 C in place", 1,
                     127, 8191, 2048, "bf16", 0.5, 1.0, 1.0, 1.0, "normal", 3),
    "recsys": ("batched shared-W GEMM Y[b]=W X[b], b<2048, W 256x512 N(0,1/sqrt(512)), X[b] 512x128 "
               "N(0,1), bf16 out", 2048, 256, 128, 512, "bf16", 1.0, 0.0, 512 ** -0.5, 1.0, "normal", 4),
    "recsys_dedup128": ("batched shared-W GEMM Y[b]=W X[index[b]], b<2048 as 16 requests of 128 items "
                        "sharing one feature entry (16 distinct X entries), W 256x512, X 512x128, bf16 out",
                        2048, 256, 128, 512, "bf16", 1.0, 0.0, 512 ** -0.5, 1.0, "normal", 4, "bf16", 16),
    "recsys_dedup4": ("batched shared-W GEMM Y[b]=W X[index[b]], b<2048 with 4 items per distinct entry "
                      "(512 distinct X entries), W 256x512, X 512x128, bf16 out",
                      2048, 256, 128, 512, "bf16", 1.0, 0.0, 512 ** -0.5, 1.0, "normal", 4, "bf16", 512),
    "square8192_f16": ("square GEMM M=N=K=8192, fp16 operands N(0,1), fp32 acc, fp16 out", 1, 8192, 8192,
                       8192, "f16", 1.0, 0.0, 1.0, 1.0, "normal", 1, "f16"),
    "square4096_f16": ("square GEMM M=N=K=4096, fp16 operands N(0,1), fp32 acc, fp16 out", 1, 4096, 4096,
                       4096, "f16", 1.0, 0.0, 1.0, 1.0, "normal", 1, "f16"),
}
WORKLOADS = {k: Workload(*v) for k, v in WORKLOADS.items()}
DEFAULT_WORKLOAD = "square8192"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "dsl_persistent_warp_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the current
    kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d.get(workload)
        if e and e.get("kernel_source_hash") == kernel_source_hash():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


def algorithmic_bytes(w) -> float:
    _, batch, M, N, K, out, alpha, beta, *_ = w
    es = 4 if out == "f32" else 2
    a = M * K * 2  # W / A read once
    b = (w.n_unique or batch) * N * K * 2  # X: the distinct entries only when deduplicated
    c = batch * M * N * es * (2 if beta != 0.0 else 1)
    idx = batch * 4 if w.n_unique else 0
    return float(a + b + c + idx)


def executed_flops(w) -> float:
    """FLOPs the kernels execute: 2*M*N*K per distinct entry for a deduplicated batch, else per
    item.  The reported TFLOP/s always count 2*M*N*K per item (the workload's logical work)."""
    return 2.0 * (w.n_unique or w.batch) * w.M * w.N * w.K


def launches_per_step(w) -> int:
    """Kernels of this library one call enqueues: the GEMM, plus one alignment pre-pass copy per
    operand whose leading dimension is not a multiple of 8 elements (packed ld here)."""
    _, batch, M, N, K, *_ = w
    n = 2 if w.n_unique else 1  # the deduplicated form also groups the items by entry
    if K % 8:
        n += 1  # A (lda = K)
    if (N if batch > 1 else K) % 8:
        n += 1  # B (ldb = K, or ldx = N for the batched form)
    return n


class ClockSampler(threading.Thread):
    """Samples SM clock and clock-event reasons through NVML while the timed region runs
    (every 0.5 ms by default)."""

    REASONS = {
        "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
        "hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
        "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
        "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
        "hw_power_brake_slowdown": "nvmlClocksEventReasonHwPowerBrakeSlowdown",
        "applications_clocks_setting": "nvmlClocksEventReasonApplicationsClocksSetting",
        "sync_boost": "nvmlClocksEventReasonSyncBoost",
    }

    def __init__(self, torch_dev: int, period_s: float = 0.0005):
        super().__init__(daemon=True)
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.ok = False
        self._halt = threading.Event()
        try:
            import pynvml
            import torch
            self.nv = pynvml
            pynvml.nvmlInit()
            p = torch.cuda.get_device_properties(torch_dev)
            bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - reported in the JSON
            self.err = repr(e)

    def run(self):
        if not self.ok:
            return
        nv = self.nv
        while not self._halt.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, const in self.REASONS.items():
                    if mask & getattr(nv, const, 0):
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def stop(self):
        self._halt.set()
        self.join(timeout=2)
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "err", "")}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


def dist_setup(n_gpus: int):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        if not dist.is_initialized():
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest of the ranks' values (every rank takes part; NCCL or gloo)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(flops_per_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: the FLOPs of all ranks' timed steps over the slowest rank's time."""
    return flops_per_step * steps * world / (max_ms * 1e-3) / 1e12


def make_inputs(w, torch):
    """Seeded synthetic inputs on the device (packed leading dimensions)."""
    from synth import matrix_bf16, seed_for
    batch, M, N, K, idx = w.batch, w.M, w.N, w.K, w.idx
    tdt = torch.float16 if w.in_dtype == "f16" else torch.bfloat16

    def draw(seed, rows, cols, std):
        return matrix_bf16(seed, rows, cols, dist=w.dist, std=std, dtype=w.in_dtype)

    def dev(bits, shape, dt=tdt):
        return torch.from_numpy(bits.view(np.int16)).view(dt).reshape(shape).cuda()

    if batch == 1:
        A = draw(seed_for(idx, "A"), M, K, w.std_a)
        B = draw(seed_for(idx, "B"), N, K, w.std_b)
        dA, dB = dev(A, (M, K)), dev(B, (N, K))
    else:
        nx = w.n_unique or batch
        A = draw(seed_for(idx, "W"), M, K, w.std_a)
        B = draw(seed_for(idx, "X"), nx * K, N, w.std_b)
        dA, dB = dev(A, (M, K)), dev(B, (nx, K, N))
    host = {"A": A, "B": B}
    if w.n_unique:
        host["index"] = dedup_index(w)
    odt = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[w.out]
    shape = (M, N) if batch == 1 else (batch, M, N)
    if w.beta != 0.0:
        Cb = matrix_bf16(seed_for(idx, "C"), batch * M, N)
        dC = dev(Cb, shape, torch.bfloat16).to(odt)
    else:
        dC = torch.empty(shape, dtype=odt, device="cuda")
    return dA, dB, dC, host


def dedup_index(w) -> np.ndarray:
    """Item b of a deduplicated workload uses distinct entry b * n_unique // batch."""
    return (np.arange(w.batch, dtype=np.int64) * w.n_unique // w.batch).astype(np.int32)


def needs_flush(w) -> bool:
    """Data smaller than twice the L2 cache would stay cached from step to step: flush it."""
    return algorithmic_bytes(w) < 2 * L2_BYTES


class L2Flush:
    """Empties L2 before a step: a write of a buffer larger than L2, then a read of a second one,
    so the step starts with none of its data cached and no dirty line left over from the flush
    for it to write back."""

    def __init__(self, torch):
        self.w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        self.r = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
        self.acc = torch.empty((), dtype=torch.float32, device="cuda")

    def __call__(self, i):
        self.w.fill_(i & 0x7F)
        self.acc.copy_(self.r.sum())


def time_steps(torch, run_step, steps, stream, flush_buf=None):
    """Device time (ms) of each of `steps` calls of run_step, each between two CUDA events on
    `stream`; with `flush_buf` (an L2Flush), L2 is flushed before every step, outside the
    events.  The host enqueues ahead of the device, so no host latency falls between a step's
    events."""
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for i in range(steps):
        if flush_buf is not None:
            flush_buf(i)
        starts[i].record(stream)
        run_step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    return [s.elapsed_time(e) for s, e in zip(starts, ends)]


def timed_region(torch, step, args, stream, flush, world, local):
    """The K timed steps.  The step is captured into a CUDA graph (eagerly if capture fails) and
    launched twice untimed (a graph holding workspace allocations maps them on first launch).
    Back-to-back workloads (no flush): the K steps are one replay of a graph of K steps between
    two events, so consecutive GEMMs start without a launch gap; each step's own time (median,
    min) comes from a second pass of single-step replays.  Flushed workloads: each step is timed
    on its own after the flush.  NVML clocks are sampled over the timed region.
    Returns (timed_ms, per-step ms, clocks, single-step graph or None, graph used)."""
    graph = None
    if not args.eager:
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                step()
            torch.cuda.synchronize()
            for _ in range(2):
                graph.replay()
            torch.cuda.synchronize()
        except Exception:
            graph = None
            torch.cuda.synchronize()
    run = graph.replay if graph is not None else step
    graph_k = None
    if flush is None and graph is not None:
        try:
            graph_k = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph_k):
                for _ in range(args.steps):
                    step()
            torch.cuda.synchronize()
            graph_k.replay()
            torch.cuda.synchronize()
        except Exception:
            graph_k = None
            torch.cuda.synchronize()
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    if graph_k is not None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        graph_k.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        timed_ms = e0.elapsed_time(e1)
    else:
        step_ms = time_steps(torch, run, args.steps, stream, flush)
        timed_ms = sum(step_ms)
    barrier(world)
    clocks = sampler.stop()
    if graph_k is not None:
        step_ms = time_steps(torch, run, args.steps, stream, flush)
    del graph_k
    return timed_ms, step_ms, clocks, graph, graph is not None


def run_ours(args, w, wname):
    import torch
    import dsl_persistent_warp_b200 as pw

    world, rank, local = dist_setup(args.gpus)
    batch, M, N, K, out, alpha, beta = w.batch, w.M, w.N, w.K, w.out, w.alpha, w.beta
    flops = 2.0 * batch * M * N * K
    dA, dB, dC, host = make_inputs(w, torch)
    dI = torch.from_numpy(host["index"]).cuda() if w.n_unique else None

    def step(A=dA, B=dB, C=dC, I=dI):
        if batch == 1:
            pw.gemm_bf16(A, B, C, alpha=alpha, beta=beta)
        elif w.n_unique:
            pw.gemm_bf16_batched_shared_w_dedup(A, B, I, C, alpha=alpha, beta=beta)
        else:
            pw.gemm_bf16_batched_shared_w(A, B, C, alpha=alpha, beta=beta)

    stream = torch.cuda.current_stream()
    tuned = None
    if args.autotune:
        # The library's autotuner measures its configuration space on these operands first;
        # the timed calls then take the configuration it recorded.
        c = pw.capi
        out_t = {"f32": c.GEMM_OUT_F32, "bf16": c.GEMM_OUT_BF16, "f16": c.GEMM_OUT_F16}[out]
        form = 0 if batch == 1 else 2 if w.n_unique else 1
        st, best_us = c.gemm_autotune(1 if w.in_dtype == "f16" else 0, form, batch, w.n_unique, M, N, K,
                                      dA.data_ptr(), K, dB.data_ptr(), K if batch == 1 else N,
                                      0 if batch == 1 else K * N, dI.data_ptr() if dI is not None else None,
                                      dC.data_ptr(), N, 0 if batch == 1 else M * N, out_t, alpha, beta,
                                      stream.cuda_stream)
        if st != c.GEMM_OK:
            raise RuntimeError(f"gemm_autotune: {c.gemm_bf16_status_string(st)}")
        step()
        torch.cuda.synchronize()
        tuned = dict(zip(("plan", "splits", "csplit", "group_m"), c.gemm_last_config()), tuner_us=round(best_us, 2))
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if pw.device_status() != 0:
        raise RuntimeError("kernel reported a bounded-wait timeout during warm-up")
    config_used = dict(zip(("plan", "splits", "csplit", "group_m"), pw.capi.gemm_last_config()))

    # Host cost of one call through the public API (Python wrapper, C ABI, planning, cached
    # tensor maps, launch), measured on eager calls that the device runs back to back; and of
    # the C entry point alone (pointers prepared once, one ctypes call per GEMM).
    n_host = max(3, min(args.steps, 20))
    t0 = time.perf_counter()
    for _ in range(n_host):
        step()
    host_us = (time.perf_counter() - t0) * 1e6 / n_host
    torch.cuda.synchronize()
    host_c_us = None
    if batch == 1:
        c = pw.capi
        a = (M, N, K, dA.data_ptr(), K, dB.data_ptr(), K, dC.data_ptr(), N,
             {"f32": c.GEMM_OUT_F32, "bf16": c.GEMM_OUT_BF16, "f16": c.GEMM_OUT_F16}[out], alpha, beta,
             stream.cuda_stream)
        fn = c.LIB.gemm_f16 if w.in_dtype == "f16" else c.LIB.gemm_bf16
        t0 = time.perf_counter()
        for _ in range(n_host):
            fn(*a)
        host_c_us = (time.perf_counter() - t0) * 1e6 / n_host
        torch.cuda.synchronize()
    flush = L2Flush(torch) if needs_flush(w) else None
    eager_ms = time_steps(torch, step, n_host, stream, flush)

    timed_ms, step_ms, clocks, graph, used_graph = timed_region(torch, step, args, stream, flush, world, local)
    if pw.device_status() != 0:
        raise RuntimeError("kernel reported a bounded-wait timeout in the timed region")
    total_ms = max_over_ranks(timed_ms, world)
    value = aggregate_tflops(flops, args.steps, world, total_ms)
    avg_launch_ms = timed_ms / args.steps
    run = graph.replay if graph is not None else step

    # Sustained leg: the same step back to back for a few seconds, so that the part reaches its
    # power-capped steady state; compared with the measured sustained peak.
    sustained = None
    if args.sustained_seconds > 0 and world == 1:
        n_sus = max(3, int(args.sustained_seconds / max(avg_launch_ms * 1e-3, 1e-6)))
        sampler2 = ClockSampler(local, period_s=0.005)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        sampler2.start()
        e0.record(stream)
        for _ in range(n_sus):
            run()
        e1.record(stream)
        torch.cuda.synchronize()
        sus_clocks = sampler2.stop()
        sus_ms = e0.elapsed_time(e1)
        sustained = {"value": round(flops * n_sus / (sus_ms * 1e-3) / 1e12, 2), "unit": UNIT, "steps": n_sus,
                     "seconds": round(sus_ms * 1e-3, 3), "clocks": sus_clocks,
                     "l2": "back to back, no flush"}
    used_graph = graph is not None
    flushed = flush is not None
    del graph

    # End to end through the public API with host buffers: every step copies its inputs from
    # pinned host memory, runs the GEMM and reads its result back, all inside the timed region.
    # Steps are pipelined over two device buffer sets and three streams (upload, compute,
    # download), so step i+1's upload overlaps step i's GEMM and step i-1's download.
    hA = torch.from_numpy(host["A"].view(np.int16)).view(dA.dtype).reshape(dA.shape).pin_memory()
    hB = torch.from_numpy(host["B"].view(np.int16)).view(dB.dtype).reshape(dB.shape).pin_memory()
    hC0 = dC.cpu().pin_memory() if beta != 0.0 else None
    hI = torch.from_numpy(host["index"]).pin_memory() if w.n_unique else None
    sets = [(dA, dB, dC, dI), (torch.empty_like(dA), torch.empty_like(dB), torch.empty_like(dC),
                               torch.empty_like(dI) if dI is not None else None)]
    hCs = [torch.empty(dC.shape, dtype=dC.dtype).pin_memory() for _ in range(2)]
    s_up, s_mm, s_down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_mm = [torch.cuda.Event() for _ in range(2)]
    ev_down = [torch.cuda.Event() for _ in range(2)]
    e2e_steps = max(2, min(args.steps, 10))

    def e2e_run(n):
        for i in range(n):
            k = i % 2
            a, bm, c, ix = sets[k]
            with torch.cuda.stream(s_up):
                if i >= 2:
                    s_up.wait_event(ev_mm[k])    # set k's inputs no longer read
                    s_up.wait_event(ev_down[k])  # set k's C already downloaded
                a.copy_(hA, non_blocking=True)
                bm.copy_(hB, non_blocking=True)
                if hC0 is not None:
                    c.copy_(hC0, non_blocking=True)
                if hI is not None:
                    ix.copy_(hI, non_blocking=True)
                ev_up[k].record(s_up)
            with torch.cuda.stream(s_mm):
                s_mm.wait_event(ev_up[k])
                if i >= 2:
                    s_mm.wait_event(ev_down[k])
                step(a, bm, c, ix)
                ev_mm[k].record(s_mm)
            with torch.cuda.stream(s_down):
                s_down.wait_event(ev_mm[k])
                hCs[k].copy_(c, non_blocking=True)
                ev_down[k].record(s_down)
        for st in (s_up, s_mm, s_down):
            stream.wait_stream(st)

    e2e_run(2)  # warm-up of the pipeline
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for st in (s_up, s_mm, s_down):
        st.wait_stream(stream)
    e2e_run(e2e_steps)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    h2d = (hA.numel() * 2 + hB.numel() * 2 + (hC0.numel() * hC0.element_size() if hC0 is not None else 0)
           + (hI.numel() * 4 if hI is not None else 0))
    d2h = hCs[0].numel() * hCs[0].element_size()
    e2e_value = aggregate_tflops(flops, e2e_steps, world, e2e_ms)
    del sets

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, host, budget_s=args.cpu_seconds)

    peaks, peak_kind = load_peaks()
    peak_t = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_ts = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    peak_b = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    # Roofline of the step's dominant kernel: tensor-bound above the ridge point
    # (peak FLOP/s / peak bytes/s), HBM-bound below it.  fp16 and bf16 have the same dense
    # tensor rate (kind::f16), so the bf16 peaks serve both.
    abytes = algorithmic_bytes(w)
    hbm_bound = executed_flops(w) / abytes < peak_t * 1e12 / (peak_b * 1e9)
    if hbm_bound:
        achieved, peak, r_unit = abytes / (avg_launch_ms * 1e-3) / 1e9, peak_b, "GB/s"
        peak_desc = f"HBM copy bandwidth ({peak_kind})"
    else:
        achieved, peak, r_unit = executed_flops(w) / (avg_launch_ms * 1e-3) / 1e12, peak_t, "TFLOP/s"
        peak_desc = f"{w.in_dtype} dense, burst ({peak_kind}; the bf16 figure: same tensor rate)"
    traffic = recorded_traffic(wname)
    res = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 5),
        "median_ms": round(statistics.median(step_ms), 5),
        "min_ms": round(min(step_ms), 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.in_dtype,
        "data": "synthetic",
        "config": {
            "workload": w.desc,
            "name": wname,
            "batch": batch, "M": M, "N": N, "K": K,
            "in": w.in_dtype, "out": out, "alpha": alpha, "beta": beta,
            "l2": "flushed before every step (256 MiB write, then 256 MiB read; outside the events)" if flushed else
                  "inputs larger than L2 (steps back to back)",
            "cold_l2": flushed,
            **({"n_unique": w.n_unique, "flops": "counted per item (2*M*N*K per item), as for the "
                "expanded batch; the distinct entries' GEMMs do batch/n_unique times fewer"}
               if w.n_unique else {}),
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "kernel_config": config_used,
            "autotuned": tuned,
            "timing": ("value: one replay of a graph of the K steps between two events; "
                       "median/min: single-step replays" if (used_graph and not flushed) else
                       "cuda-graph replay of one step, events around each replay" if used_graph else
                       "eager, events around each step"),
        },
        "pct_of_peak": {
            "of_measured_burst": round(100.0 * value / world / peak_t, 2),
            "of_spec_2250": round(100.0 * value / world / SPEC_BF16_TFLOPS, 2),
            "peak_source": peak_kind,
        },
        "roofline": {
            "bound": "hbm" if hbm_bound else "tensor",
            "achieved": round(achieved, 2),
            "peak": peak,
            "unit": r_unit,
            "frac": round(achieved / peak, 4),
            "traffic": traffic,
            "algorithmic_bytes": abytes,
            "peak_kind": peak_desc,
        },
        "eager": {"ms_per_step": round(statistics.mean(eager_ms), 5),
                  "median_ms": round(statistics.median(eager_ms), 5),
                  "host_us_per_call": round(host_us, 2),
                  "host_us_per_call_c_abi": None if host_c_us is None else round(host_c_us, 2),
                  "calls": n_host},
        "e2e": {"value": round(e2e_value, 3), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "steps": e2e_steps,
                "pipeline": "2 buffer sets; upload, GEMM and download on separate streams"},
        "gpu_launches": args.steps * launches_per_step(w),  # timed region of `value`
        "clocks": clocks,
    }
    if sustained is not None:
        sustained["frac_of_sustained_peak"] = round(sustained["value"] / peak_ts, 4)
        sustained["sustained_peak"] = peak_ts
        res["sustained"] = sustained
    if cpu is not None:
        res["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def cpu_baseline(w, host, budget_s=15.0):
    """The fp64 oracle, as it stands, on a bounded row sample of the same workload."""
    import oracle
    desc, batch, M, N, K, out, alpha, beta, *_ = w
    A, B = host["A"], host["B"]

    def run_rows(nrows):
        rows = list(range(nrows))
        t0 = time.perf_counter()
        if batch == 1:
            oracle.gemm(A, B, M=M, N=N, K=K, rows=rows, in_dtype=w.in_dtype)
        elif w.n_unique:
            nb = max(1, nrows // M)
            oracle.gemm_batched_dedup(A, B, host["index"][:nb], n_x=w.n_unique, M=M, N=N, K=K,
                                      stride_x=K * N, in_dtype=w.in_dtype)
        else:
            nb = max(1, nrows // M)
            oracle.gemm_batched(A, B[: nb * K], batch=nb, M=M, N=N, K=K, stride_x=K * N,
                                in_dtype=w.in_dtype)
        return time.perf_counter() - t0

    if batch == 1:
        t = run_rows(min(M, 4))
        per_row = max(t / min(M, 4), 1e-6)
        nrows = int(max(1, min(M, budget_s / per_row)))
        dt = run_rows(nrows)
        flops = 2.0 * nrows * N * K
        sample = f"{nrows} of {M} output rows (all {N} columns, full K={K})"
    else:
        t = run_rows(M)
        nb = int(max(1, min(batch, budget_s / max(t, 1e-6))))
        dt = run_rows(nb * M)
        flops = 2.0 * nb * M * N * K
        sample = f"{nb} of {batch} batches (full {M}x{N}x{K} each)"
    return {"value": round(flops / dt / 1e12, 6), "unit": UNIT, "cores": oracle.threads(),
            "kind": "oracle", "sample": sample, "seconds": round(dt, 2)}


def run_reference(args, w, wname):
    """The fp64 CPU oracle timed on the host cores (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from synth import matrix_bf16, seed_for
    desc, batch, M, N, K, out, alpha, beta, std_a, std_b, dist, idx = w[:12]
    # bounded sample: at most ~`ref_seconds` of CPU work over warmup + steps.
    total_steps = args.steps + args.warmup
    per_step_s = max(0.02, args.ref_seconds / max(total_steps, 1))
    # Rows of A are a prefix of its seeded stream, so only the rows a step can use are drawn.
    a_rows = min(M, 1024)
    A = matrix_bf16(seed_for(idx, "A" if batch == 1 else "W"), a_rows, K, dist=dist, std=std_a,
                    dtype=w.in_dtype)
    if batch == 1:
        B = matrix_bf16(seed_for(idx, "B"), N, K, dist=dist, std=std_b, dtype=w.in_dtype)
    else:
        B = matrix_bf16(seed_for(idx, "X"), K, N, dist=dist, std=std_b, dtype=w.in_dtype)
    c0 = matrix_bf16(seed_for(idx, "C"), a_rows, N) if beta != 0.0 else None

    def one(nrows):
        rows = list(range(nrows))
        if batch == 1:
            oracle.gemm(A, B, M=a_rows, N=N, K=K, c0=c0, alpha=alpha, beta=beta, rows=rows,
                        in_dtype=w.in_dtype)
        else:
            oracle.gemm(A, B, M=a_rows, N=N, K=K, b_kmajor=False, rows=rows, in_dtype=w.in_dtype)

    t0 = time.perf_counter()
    one(1)
    per_row = max(time.perf_counter() - t0, 1e-6)
    nrows = int(max(1, min(a_rows, per_step_s / per_row)))
    for _ in range(args.warmup):
        one(nrows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one(nrows)
    dt = time.perf_counter() - t0
    flops = 2.0 * nrows * N * K * args.steps
    value = flops / dt / 1e12
    sample = f"{nrows} of {M} output rows per step (all {N} columns, full K={K})" + (
        f", one of {batch} batches" if batch > 1 else "")
    res = {
        "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(dt * 1e3 / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": desc, "name": wname, "batch": batch, "M": M, "N": N, "K": K,
                   "in": w.in_dtype, "out": out, "alpha": alpha, "beta": beta,
                   "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": oracle.threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(res), flush=True)


def run_vendor(args, w, wname):
    """Vendor context: the same workload through torch.matmul / addmm (cuBLAS), timed with the
    same routine as ours (timed_region, L2 flush included).  Rank 0 only; not a target and not
    part of the product path."""
    import torch

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    desc, batch, M, N, K, out, alpha, beta, *_ = w
    base = {"metric": METRIC, "unit": UNIT, "impl": "vendor (torch.matmul, cuBLAS)",
            "config": {"workload": desc, "name": wname}}
    if out == "f32":
        # cuBLAS through torch has no 16-bit-in / fp32-out GEMM without converting the operands
        print(json.dumps({**base, "unavailable": "fp32 output from 16-bit operands"}), flush=True)
        return
    torch.cuda.set_device(0)
    dA, dB, dC, host = make_inputs(w, torch)
    dI = torch.from_numpy(host["index"]).long().cuda() if w.n_unique else None

    def step():
        if w.n_unique:
            # the distinct entries once, then each item's copy of its entry's result
            torch.index_select(torch.matmul(dA, dB), 0, dI, out=dC)
        elif batch > 1:
            torch.matmul(dA, dB, out=dC)
        elif beta != 0.0:
            dC.addmm_(dA, dB.t(), beta=beta, alpha=alpha)
        elif alpha != 1.0:
            torch.mm(dA, dB.t(), out=dC).mul_(alpha)
        else:
            torch.mm(dA, dB.t(), out=dC)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    flush = L2Flush(torch) if needs_flush(w) else None
    stream = torch.cuda.current_stream()
    timed_ms, step_ms, clocks, graph, used_graph = timed_region(torch, step, args, stream, flush, 1, 0)
    del graph
    flops = 2.0 * batch * M * N * K
    res = {**base, "value": round(flops * args.steps / (timed_ms * 1e-3) / 1e12, 2), "n_gpus": 1,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(timed_ms / args.steps, 5),
           "median_ms": round(statistics.median(step_ms), 5), "min_ms": round(min(step_ms), 5),
           "higher_is_better": True, "dtype": w.in_dtype, "data": "synthetic", "cold_l2": flush is not None,
           "clocks": clocks}
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference", "vendor"], default="ours",
                    help="ours: this library; reference: the CPU oracle; vendor: torch.matmul (cuBLAS)")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=sorted(WORKLOADS) + ["all"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU seconds for the oracle baseline sample")
    ap.add_argument("--ref-seconds", type=float, default=90.0,
                    help="CPU seconds for the whole --impl reference run")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true", help="time eager calls instead of a graph replay")
    ap.add_argument("--autotune", action="store_true",
                    help="run the library's autotuner on the workload before timing it")
    ap.add_argument("--sustained-seconds", type=float, default=None,
                    help="length of the back-to-back sustained leg (default: 3 s for tensor-bound "
                         "workloads, 0 otherwise)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    names = sorted(WORKLOADS) if args.workload == "all" else [args.workload]
    sustained_arg = args.sustained_seconds
    for n in names:
        if sustained_arg is None:
            w = WORKLOADS[n]
            args.sustained_seconds = 3.0 if executed_flops(w) / algorithmic_bytes(w) > 263 else 0.0
        if args.impl == "reference":
            run_reference(args, WORKLOADS[n], n)
        elif args.impl == "vendor":
            run_vendor(args, WORKLOADS[n], n)
        else:
            run_ours(args, WORKLOADS[n], n)


if __name__ == "__main__":
    main()

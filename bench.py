#!/usr/bin/env python
"""Benchmark of the ConvRot W4A8 codebook linear forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

A step is one pass of the whole hot path over one batch: rotate + quantise
the activations, then the fused decode GEMV (M <= 8) or decode + tcgen05
GEMM (M > 8), epilogue included.  The default workload is the decode batch
M = 8, N = K = 4096; the metric is the weight bytes the layer streams
(4.5 bits per weight + per-channel scales + codebook) per second.  A
second block ("prefill") reports the M = 2048, N = K = 4096 prefill step in
int8 TOPS.

Timing: inputs live in HBM before the timed region; R rotating copies of the
layer and activations (more bytes than the 126 MB L2) are cycled so every
step streams its weights from HBM; the K timed steps are one CUDA-graph
replay bracketed by CUDA events on the capturing stream, with a barrier and a
synchronize on both sides; multi-GPU runs report the max over ranks.  SM
clocks and throttle reasons are sampled through NVML during the timed region.

Under torchrun every rank runs its own replica of the layer on its own batch
(weak scaling, no data-path collective); the only collectives are the
barrier and the max over ranks of the timings.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "W4A8 GEMV weight GB/s & % HBM roofline (M≤8); prefill int8 TOPS & % peak"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
INT8_OVER_BF16 = 2.0  # nominal dense ratio (4.5 vs 2.25 PFLOP/s)


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="c5_m8_8k")
    p.add_argument("--prefill-workload", default="c5_m16384_8k")
    p.add_argument("--gemv-extra", default="c1_decode_m1_1k,c2_decode_m8_4k,c5_m1_8k,c5_m2_8k,c5_m4_8k",
                   help="comma-separated decode workloads reported beside the headline (empty: none)")
    p.add_argument("--prefill-extra", default="c3_prefill_2k_4k,c4_mlp_up,c4_mlp_down",
                   help="comma-separated prefill workloads reported beside the prefill block (empty: none)")
    p.add_argument("--backward-workload", default="c3_prefill_2k_4k")
    p.add_argument("--only", default=None,
                   choices=["headline", "decode-transient", "quantiser", "int8-peak", "rotate-quant", "prefill"],
                   help="run one piece alone (profiling runs): the headline step and GEMV, the prefill weight "
                        "transient, the offline quantiser, the INT8 rate kernel, the rotate+quantise kernel on "
                        "the prefill workload's activations, or the prefill block of --prefill-workload")
    p.add_argument("--no-prefill", action="store_true")
    p.add_argument("--no-grouped", action="store_true")
    p.add_argument("--no-swiglu", action="store_true")
    p.add_argument("--no-backward", action="store_true")
    p.add_argument("--swiglu-workload", default="c4_mlp_up")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=10.0)
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def weight_bytes(N, K):
    """Algorithmic weight traffic of one decode pass: packed codes (K/2 per
    row), fp8 group scales (K/16 per row), fp32 channel scales, fp32 codebook."""
    return N * (K // 2) + N * (K // 16) + 4 * N + 64


def gemv_launch_bytes(M, N, K):
    """Algorithmic bytes of one GEMV launch: the weight stream, the int8
    activation rows and scales it reads, and the bf16 output it writes."""
    return weight_bytes(N, K) + M * K + 4 * M + 2 * M * N


GEMV_SOURCES = ("k_gemv.cuh", "cr_device.cuh")
KERNEL_LAUNCHES = 200  # chained launches over which a roofline kernel's duration is averaged


def source_digest(files):
    """Short digest of kernel sources, to tell whether recorded counters are
    still those of the current kernel."""
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "w4a8_codebook_quantized_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def prior_traffic(kernel_tag, sources=GEMV_SOURCES):
    """DRAM bytes per launch recorded from an ncu capture of the current kernel
    (profiles/<tag>.traffic), or None when there is none or the kernel's
    sources changed since it was taken."""
    path = os.path.join(ROOT, "profiles", f"{kernel_tag}.traffic")
    value, digest = None, None
    try:
        with open(path) as f:
            for line in f:
                if line.startswith("dram_bytes_per_launch:"):
                    value = float(line.split(":", 1)[1])
                elif line.startswith("source_digest:"):
                    digest = line.split(":", 1)[1].strip()
    except OSError:
        return None
    if digest != source_digest(sources):
        return None
    return value


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML while running."""

    def __init__(self, index: int, period: float = 0.002):
        self.index, self.period = index, period
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            self.h = nv.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.ok = True
            self._sample()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        except Exception:
            self.ok = False
        return self

    def _sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        names = {
            "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
            "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
            "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
        }
        for k, bit in names.items():
            if r & bit:
                self.reasons.add(k)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._t.join()
            try:
                self._sample()
            except Exception:
                pass

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": float(self.max_mhz),
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ---------------------------------------------------------------- distributed

def dist_setup(backend: str = "nccl"):
    """Join the torchrun process group (one process per GPU) when WORLD_SIZE > 1.
    Returns (world, rank, local_rank)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value: float, world: int) -> float:
    """The slowest rank's timing: every multi-GPU number is the max over ranks."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(bytes_per_step_per_rank: float, steps: int, world: int, max_seconds: float) -> float:
    """Whole-job throughput in GB/s: every rank streams its own replica's
    weights each step (weak scaling), divided by the slowest rank's time."""
    return world * bytes_per_step_per_rank * steps / max_seconds / 1e9


def rank_seed(seed: int, rank: int) -> int:
    """Each rank draws its own layer and batch (independent replicas)."""
    return seed + 1000 * rank


# ---------------------------------------------------------------- our arm

class Sets:
    """R rotating device copies of one workload (layer + activations)."""

    def __init__(self, case, rank, min_bytes=int(1.25 * L2_BYTES)):
        import torch

        import w4a8_codebook_quantized_b200 as cr
        from w4a8_codebook_quantized_b200 import inputs
        self.case = case
        M, N, K = case.M, case.N, case.K
        per_set = weight_bytes(N, K) + 2 * M * K
        self.R = max(2, int(math.ceil(min_bytes / per_set)))
        layer = inputs.layer(N, K, rank_seed(case.seed, rank))
        x = inputs.activations(M, K, rank_seed(case.seed, rank), case.dist)
        q = torch.from_numpy(layer.qdata).cuda()
        s = torch.from_numpy(layer.srel).cuda()
        self.cb = torch.from_numpy(layer.codebook).cuda()
        ws = torch.from_numpy(layer.s_channel).cuda()
        xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
        self.q = [q.clone() for _ in range(self.R)]
        self.s = [s.clone() for _ in range(self.R)]
        self.ws = [ws.clone() for _ in range(self.R)]
        self.x = [xd.clone() for _ in range(self.R)]
        self.rows = cr.gemv_rows(M) if M <= cr.CR_GEMV_MAX_M else M
        self.xq = [torch.empty(self.rows, K, dtype=torch.int8, device="cuda") for _ in range(self.R)]
        self.xs = [torch.empty(self.rows, dtype=torch.float32, device="cuda") for _ in range(self.R)]
        self.out = [torch.empty(M, N, dtype=torch.bfloat16, device="cuda") for _ in range(self.R)]
        self.lin = [cr.W4A8Linear(self.q[r], self.s[r], self.cb, self.ws[r]) for r in range(self.R)]
        self.x_host = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
        self.out_host = torch.empty(M, N, dtype=torch.bfloat16).pin_memory()

    def step(self, i):
        """One decode step through a prepared layer (W4A8Linear.forward =
        cr_w4a8_plan_forward): the rotate+quant kernel and the decode GEMV."""
        r = i % self.R
        self.lin[r].forward(self.x[r], out=self.out[r], xq_work=self.xq[r], xs_work=self.xs[r])

    def contraction_only(self, i):
        """The dominant kernel alone: the prepared layer's decode GEMV on the
        quantised activations (W4A8Linear.gemv = cr_w4a8_plan_gemv)."""
        r = i % self.R
        self.lin[r].gemv(self.xq[r], self.xs[r], m=self.case.M, out=self.out[r])

    def e2e_step(self, i):
        """Through the public API with host buffers: a prepared W4A8Linear
        layer's forward_host (the C-ABI call cr_w4a8_plan_forward_host), which
        queues the H2D copy of x from pinned memory, the forward and the D2H
        copy of y."""
        r = i % self.R
        self.lin[r].forward_host(self.x_host, self.out_host, self.x[r], self.out[r], self.xq[r], self.xs[r])


def upload_graph(g, stream):
    """Upload an instantiated CUDA graph to the device before its timed
    replay; otherwise the first replay pays for the upload (about 1.5 us per
    launch of a 200-launch graph).  Nothing of the graph runs."""
    from cuda.bindings import runtime as rt
    exe = rt.cudaGraphExec_t(init_value=g.raw_cuda_graph_exec())
    err = rt.cudaGraphUpload(exe, rt.cudaStream_t(init_value=stream.cuda_stream))[0]
    if err != rt.cudaError_t.cudaSuccess:
        raise RuntimeError(f"cudaGraphUpload failed: {err}")


def graph_time(fn, steps, warmup, world, sampler_index=None):
    """Capture `steps` calls of fn(i) in one CUDA graph and time one replay
    of it; return (seconds of the timed replay, clocks).  Warm-up: `warmup`
    eager calls, then the same graph replayed untimed until at least `warmup`
    steps have run through it (at least once: a graph's first replay pays
    one-time costs, about 15 us for a 20-step decode graph, that every later
    replay of it does not)."""
    import torch
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(max(1, warmup)):
            fn(i)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(steps):
            fn(i)
    upload_graph(g, stream)
    with torch.cuda.stream(stream):
        for _ in range(max(1, -(-max(1, warmup) // steps))):
            g.replay()
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    clocks = ClockSampler(sampler_index if sampler_index is not None else torch.cuda.current_device())
    with clocks:
        with torch.cuda.stream(stream):
            e0.record(stream)
            g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    secs = e0.elapsed_time(e1) / 1000.0
    del g
    return secs, clocks.summary()


def eager_time(fn, steps, warmup, world):
    import torch
    stream = torch.cuda.current_stream()
    for i in range(max(1, warmup)):
        fn(i)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(steps):
        fn(i)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    return e0.elapsed_time(e1) / 1000.0


def cpu_baseline(case, seconds):
    """The oracle, as it stands, on the host: full forward passes of the
    workload, single-threaded, repeated for about `seconds`."""
    import oracle
    from w4a8_codebook_quantized_b200 import inputs
    layer = inputs.layer(case.N, case.K, case.seed)
    M = case.M
    rows = M
    if M > 64:  # prefill-size batches: a row sample (rows are independent)
        rows = 16
    x = inputs.activations(rows, case.K, case.seed, case.dist)
    oracle.lib()
    n, t0 = 0, time.perf_counter()
    while True:
        oracle.linear(x, layer.qdata, layer.srel, layer.codebook, layer.s_channel, threads=1)
        n += 1
        if time.perf_counter() - t0 >= seconds:
            break
    el = time.perf_counter() - t0
    per_pass = el / n
    # the same oracle with its contraction spread over every host core it may
    # use (rows are independent, so the result is the same)
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    n2, t1 = 0, time.perf_counter()
    while True:
        oracle.linear(x, layer.qdata, layer.srel, layer.codebook, layer.s_channel, threads=cores)
        n2 += 1
        if time.perf_counter() - t1 >= seconds / 2:
            break
    per_pass_all = (time.perf_counter() - t1) / n2

    def rate(t):
        if M <= 8:
            return weight_bytes(case.N, case.K) / t / 1e9
        return 2.0 * rows * case.N * case.K / t / 1e12

    if M <= 8:
        unit, sample = "GB/s", f"{n} full forward passes of the workload (M={M}, N={case.N}, K={case.K})"
    else:
        unit, sample = "TOPS", f"{n} passes over {rows} of {M} token rows (N={case.N}, K={case.K})"
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            model = next((l.split(":", 1)[1].strip() for l in f if l.startswith("model name")), None)
    except OSError:
        pass
    return {"value": rate(per_pass), "unit": unit, "cores": 1, "kind": "oracle", "sample": sample,
            "seconds": round(el, 3),
            "all_cores": {"value": rate(per_pass_all), "cores": cores, "passes": n2,
                          "note": "the oracle's int32 contraction split over rows on every allowed core"},
            "cpu_model": model}


def gemv_block(case, args, world, rank, local, pk, sets=None):
    """One decode workload: the whole step (rotate+quant launch + GEMV
    launch) as one CUDA-graph replay of K steps, and the GEMV kernel alone
    the same way (its roofline).  Rotating copies of layer + activations
    larger than L2 make every step stream its weights from HBM."""
    if sets is None:
        sets = Sets(case, rank)
    M, N, K = case.M, case.N, case.K
    secs, clocks = graph_time(sets.step, args.steps, args.warmup, world, local)
    secs = max_over_ranks(secs, world)
    wb = weight_bytes(N, K)
    # the kernel's own duration: a chain of at least KERNEL_LAUNCHES launches
    # in one graph, so that the graph's start-up is not charged to a short
    # chain's few launches
    klaunches = max(args.steps, KERNEL_LAUNCHES)
    ksecs, _ = graph_time(sets.contraction_only, klaunches, args.warmup, world, local)
    ksecs = max_over_ranks(ksecs, world)
    per_launch = ksecs / klaunches
    achieved = gemv_launch_bytes(M, N, K) / per_launch / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / pk["hbm_gbs"], 4), "traffic": prior_traffic(f"gemv_kernel_{case.name}"),
                "kernel": "cr::gv::gemv_kernel", "peak_source": f"{pk['source']} (hbm_gbs)",
                "algorithmic_bytes_per_launch": gemv_launch_bytes(M, N, K),
                "us_per_launch": round(per_launch * 1e6, 3), "launches_timed": klaunches}
    return {"workload": f"{case.name}: decode batch M={M}, N={N}, K={K}, rot 256, group 16, seed {case.seed}",
            "value": round(aggregate_value(wb, args.steps, world, secs), 2), "unit": "GB/s",
            "us_per_step": round(secs / args.steps * 1e6, 3),
            "l2": f"rotating {sets.R} copies of layer+activations ({sets.R * (wb + 2 * M * K) / 2**20:.0f} MiB)",
            "roofline": roofline, "_secs": secs, "_clocks": clocks, "_sets": sets}


def measure_int8_peak(world):
    """The dense INT8 tensor-core rate of this GPU: the library's
    measurement kernel (resident shared-memory operands, tcgen05 kind::i8 on
    CTA pairs, the prefill GEMM's instruction shape), timed with CUDA events;
    the best of several launches of about 2 ms."""
    import torch

    import w4a8_codebook_quantized_b200 as cr
    stream = torch.cuda.Stream()
    iters = 4096
    with torch.cuda.stream(stream):
        ops = cr.cr_mma_i8_peak(iters, stream=stream)
        stream.synchronize()
        # size the launch to about 2 ms
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        cr.cr_mma_i8_peak(iters, stream=stream)
        e1.record(stream)
        stream.synchronize()
        t = e0.elapsed_time(e1) / 1000.0
        iters = int(min(1 << 20, max(1024, iters * 2e-3 / max(t, 1e-6))))
        best, times = None, []
        for _ in range(5):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            ops = cr.cr_mma_i8_peak(iters, stream=stream)
            e1.record(stream)
            stream.synchronize()
            times.append(e0.elapsed_time(e1) / 1000.0)
    cr.cr_check_device_error(stream)
    t = min(times)
    t = max_over_ranks(t, world)
    return {"value": round(ops / t / 1e12, 1), "unit": "TOPS", "iters": iters, "ms_per_launch": round(t * 1e3, 4),
            "kernel": "cr::pk::mma_i8_peak_kernel (tcgen05.mma.cta_group::2.kind::i8, M=N=256, K=32, operands "
                      "resident in shared memory, one cluster of two CTAs per SM pair)",
            "launches": len(times)}


def run_ours(args):
    import torch

    import w4a8_codebook_quantized_b200 as cr
    from w4a8_codebook_quantized_b200 import inputs
    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    cr.lib()
    if args.only in ("decode-transient", "quantiser", "int8-peak", "rotate-quant"):
        return run_only(args, world, rank, local)
    pk = peaks()
    if args.only == "prefill":
        # the prefill block of --prefill-workload alone (its INT8 fraction
        # against the measured bf16 rate x the nominal ratio)
        blk = run_prefill(args, world, rank, pk, None, args.prefill_workload)
        cr.cr_check_device_error()
        if rank == 0:
            print(json.dumps({"only": "prefill", **blk}), flush=True)
        return
    case = inputs.CASES[args.workload]
    if case.M > 8:
        raise SystemExit("the headline workload must be a decode batch (M <= 8)")
    M, N, K = case.M, case.N, case.K

    # headline: the whole step (rotate+quant launch + GEMV launch), graph-replayed
    head = gemv_block(case, args, world, rank, local, pk)
    secs, clocks, sets = head.pop("_secs"), head.pop("_clocks"), head.pop("_sets")
    wb = weight_bytes(N, K)
    value = aggregate_value(wb, args.steps, world, secs)

    # end to end through the public API with host buffers
    # warm-up covers every rotating layer at least twice (first calls encode
    # each prepared layer's activation map)
    esecs = eager_time(sets.e2e_step, args.steps, max(args.warmup, 2 * sets.R), world)
    esecs = max_over_ranks(esecs, world)
    e2e = {"value": round(aggregate_value(wb, args.steps, world, esecs), 2), "unit": "GB/s",
           "h2d_bytes_per_step": 2 * M * K, "d2h_bytes_per_step": 2 * M * N,
           "ms_per_step": round(esecs / args.steps * 1e3, 5),
           "path": "W4A8Linear.forward_host (bound call, cr_w4a8_host_call_run), eager: x from pinned host memory "
                   "by a copy kernel, rotate+quant, GEMV storing y into pinned host memory (3 launches)"}
    del sets

    gemv_extra = []
    if args.only != "headline":
        for name in [w for w in args.gemv_extra.split(",") if w and w != args.workload]:
            blk = gemv_block(inputs.CASES[name], args, world, rank, local, pk)
            for k in ("_secs", "_clocks", "_sets"):
                blk.pop(k)
            gemv_extra.append(blk)
            torch.cuda.empty_cache()

    int8_peak = None
    prefill = prefill_extra = None
    if not args.no_prefill and args.only != "headline":
        int8_peak = measure_int8_peak(world)
        prefill = run_prefill(args, world, rank, pk, int8_peak, args.prefill_workload)
        torch.cuda.empty_cache()
        prefill_extra = []
        for name in [w for w in args.prefill_extra.split(",") if w and w != args.prefill_workload]:
            prefill_extra.append(run_prefill(args, world, rank, pk, int8_peak, name))
            torch.cuda.empty_cache()

    grouped = None
    if not args.no_grouped and args.only != "headline":
        grouped = run_grouped(args, world, rank, local, inputs.CASES["c2_decode_m8_4k"])

    swiglu = None
    if not args.no_swiglu and args.only != "headline":
        swiglu = run_swiglu(args, world, rank, pk)

    backward = None
    if not args.no_backward and args.only != "headline":
        backward = run_backward(args, world, rank, pk)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(case, args.cpu_seconds)

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(secs / args.steps * 1e3, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "s8", "data": "synthetic",
        "config": {"workload": head["workload"],
                   "path": "W4A8Linear.forward (cr_w4a8_plan_forward, a prepared layer) = rotate+quant kernel + fused "
                           "decode GEMV kernel",
                   "l2": head["l2"] + " > 126 MiB L2",
                   "timing": "one CUDA-graph replay of K steps (graph uploaded beforehand), CUDA events on the capture "
                             "stream; warm-up: W eager steps, then the same graph replayed untimed (at least W steps, "
                             "at least one replay: a graph's first replay pays one-time costs)",
                   "parallelism": f"replica x{world}"},
        "roofline": head["roofline"], "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": 2 * args.steps,
        "clocks": clocks, "gemv_extra": gemv_extra, "int8_peak": int8_peak, "prefill": prefill,
        "prefill_extra": prefill_extra, "grouped": grouped, "swiglu": swiglu, "ste_backward": backward,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_prefill(args, world, rank, pk, int8_peak, workload):
    """One prefill workload: the step through cr_w4a8_linear (rotate+quant
    overlapped with the weight decode, then the tcgen05 GEMM); the GEMM
    kernel alone (cr_gemm_s8 on the decoded weight: the roofline, against the
    INT8 rate measured in this run) and the cr_w4a8_gemm call (decode + GEMM)
    beside it.  Each replay follows a 256 MiB L2 flush (outside the events)."""
    import torch

    import w4a8_codebook_quantized_b200 as cr
    from w4a8_codebook_quantized_b200 import inputs
    case = inputs.CASES[workload]
    M, N, K = case.M, case.N, case.K
    layer = inputs.layer(N, K, rank_seed(case.seed, rank))
    x = inputs.activations(M, K, rank_seed(case.seed, rank), case.dist)
    q = torch.from_numpy(layer.qdata).cuda()
    s = torch.from_numpy(layer.srel).cuda()
    cb = torch.from_numpy(layer.codebook).cuda()
    ws = torch.from_numpy(layer.s_channel).cuda()
    xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    del x
    xq = torch.empty(M, K, dtype=torch.int8, device="cuda")
    xs = torch.empty(M, dtype=torch.float32, device="cuda")
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    steps = max(3, min(args.steps, 50))

    def step():
        cr.cr_w4a8_linear(xd, q, s, cb, ws, out=out, xq_work=xq, xs_work=xs)

    for i in range(max(3, args.warmup)):
        step()
    # the GEMM kernel alone runs through cr_gemm_s8 on the weight decoded once
    # beforehand (the same kernel and arguments cr_w4a8_gemm launches after
    # its decode)
    w8 = cr.cr_w4a8_decode_int8(q, s, cb)
    cr.cr_gemm_s8(xq, xs, w8, ws, out=out)
    torch.cuda.synchronize()
    ts, tc, tg = flushed_medians([step, lambda: cr.cr_w4a8_gemm(xq, xs, q, s, cb, ws, out=out),
                                  lambda: cr.cr_gemm_s8(xq, xs, w8, ws, out=out)], steps)
    del w8
    t, tc, tg = max_over_ranks(ts, world), max_over_ranks(tc, world), max_over_ranks(tg, world)
    ops = 2.0 * M * N * K
    achieved = ops / tg / 1e12
    if int8_peak is not None:
        peak_tops, src = int8_peak["value"], "measured in this run (int8_peak: tcgen05 kind::i8 rate kernel)"
    else:
        peak_tops, src = pk["bf16_tflops"] * INT8_OVER_BF16, \
            f"{pk['source']} bf16_tflops x {INT8_OVER_BF16} (nominal int8/bf16 ratio)"
    return {"workload": f"{case.name}: prefill M={M}, N={N}, K={K}", "value": round(world * ops / t / 1e12, 2),
            "unit": "TOPS", "ms_per_step": round(t * 1e3, 4), "steps": steps,
            "l2": "256 MiB write between steps, outside the timed events",
            "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak_tops, 1),
                         "unit": "TOPS", "frac": round(achieved / peak_tops, 4), "traffic": None,
                         "kernel": "tcgen05 int8 GEMM + epilogue (cr_gemm_s8 on the decoded int8 weight)",
                         "peak_source": src, "us_per_call": round(tg * 1e6, 2),
                         "frac_of_bf16x2": round(achieved / (pk["bf16_tflops"] * INT8_OVER_BF16), 4)},
            "gemm_call": {"what": "cr_w4a8_gemm: weight decode to an int8 transient + the same GEMM",
                          "us": round(tc * 1e6, 2), "tops": round(ops / tc / 1e12, 1),
                          "frac": round(ops / tc / 1e12 / peak_tops, 4)}}


def run_only(args, world, rank, local):
    """Single pieces for profiling runs (one JSON line each)."""
    import torch

    import w4a8_codebook_quantized_b200 as cr
    from w4a8_codebook_quantized_b200 import inputs
    out = {"only": args.only}
    if args.only == "int8-peak":
        out.update(measure_int8_peak(world))
    elif args.only == "decode-transient":
        # the prefill's int8 weight transient on an [8192, 4096] layer: two
        # warm launches, then 20 back to back in one CUDA graph, timed with
        # CUDA events
        N, K = 8192, 4096
        layer = inputs.layer(N, K, 1)
        q, s, cb = (torch.from_numpy(a).cuda() for a in (layer.qdata, layer.srel, layer.codebook))
        w8 = torch.empty(N, K, dtype=torch.int8, device="cuda")
        for _ in range(2):
            cr.cr_w4a8_decode_int8(q, s, cb, w8)
        torch.cuda.synchronize()
        t = replay_time(lambda: cr.cr_w4a8_decode_int8(q, s, cb, w8, stream=torch.cuda.current_stream()), 20)
        out.update({"N": N, "K": K, "us": round(t * 1e6, 2),
                    "gb_per_s": round(N * K * (0.5 + 1 / 16 + 1) / t / 1e9, 1)})
    elif args.only == "rotate-quant":
        # the rotate+quantise kernel alone on the activations of the prefill
        # workload: two warm launches, then 20 back to back in one CUDA
        # graph, timed with CUDA events (each reads 2 bytes and writes 1 byte
        # per element, plus the row scales; the 20 launches reuse one input,
        # so it comes from L2 after the first)
        case = inputs.CASES[args.prefill_workload]
        M, K = case.M, case.K
        x = torch.from_numpy(inputs.activations(M, K, case.seed, case.dist).view(np.int16)).cuda() \
            .view(torch.bfloat16)
        xq = torch.empty(M, K, dtype=torch.int8, device="cuda")
        xs = torch.empty(M, dtype=torch.float32, device="cuda")
        for _ in range(2):
            cr.cr_rotate_quant_act(x, xq=xq, xs=xs)
        torch.cuda.synchronize()
        t = replay_time(lambda: cr.cr_rotate_quant_act(x, xq=xq, xs=xs, stream=torch.cuda.current_stream()), 20)
        out.update({"workload": case.name, "M": M, "K": K, "us": round(t * 1e6, 2),
                    "gb_per_s": round((3 * M * K + 4 * M) / t / 1e9, 1)})
    elif args.only == "quantiser":
        # the offline quantiser and the stochastic re-assignment on an
        # [8192, 4096] rotated weight
        N, K = 8192, 4096
        w = torch.from_numpy(inputs.rotated_weights(N, K, 1)).cuda()
        cb = torch.tensor(inputs.FIXED_CODEBOOK, dtype=torch.float32, device="cuda")
        u = torch.from_numpy(inputs.uniforms(N, K, 1)).cuda()
        q, s, ch, _ = cr.cr_w4a8_quantize_rotated(w, cb)
        cr.cr_w4a8_assign_codes(w, s, ch, cb, u, q)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        cr.cr_w4a8_quantize_rotated(w, cb, q, s, ch)
        e1.record()
        torch.cuda.synchronize()
        out.update({"N": N, "K": K, "quantize_us": round(e0.elapsed_time(e1) * 1e3, 1)})
    cr.cr_check_device_error()
    if rank == 0:
        print(json.dumps(out), flush=True)


def replay_time(fn, n):
    """fn() captured n times in one CUDA graph (uploaded first), replayed
    once after a warm replay; seconds per call by CUDA events on the replay
    stream."""
    import torch
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(n):
            fn()
    upload_graph(g, stream)
    with torch.cuda.stream(stream):
        g.replay()
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        g.replay()
        e1.record(stream)
    stream.synchronize()
    del g
    return e0.elapsed_time(e1) / 1000.0 / n


def flushed_medians(fns, steps):
    """Each fn() captured once as a CUDA graph (uploaded first) and replayed
    `steps` times, a 256 MiB L2 flush before every replay outside the CUDA
    events on the replay stream; the median seconds of each."""
    import torch
    stream = torch.cuda.Stream()
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    graphs = []
    for fn in fns:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        upload_graph(g, stream)
        graphs.append(g)
    res = []
    with torch.cuda.stream(stream):
        for g in graphs:
            t = []
            for i in range(steps):
                flush.fill_(i & 0xFF)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                g.replay()
                e1.record(stream)
                torch.cuda.synchronize()
                t.append(e0.elapsed_time(e1) / 1000.0)
            res.append(statistics.median(t))
    del graphs
    return res


def run_swiglu(args, world, rank, pk):
    """A gate/up projection stored with interleaved rows (N = 2F), SwiGLU fused
    into the GEMM epilogue (cr_w4a8_linear_swiglu, out [M, F]) against the
    plain forward of the same layer (cr_w4a8_linear, out [M, N])."""
    import torch

    import w4a8_codebook_quantized_b200 as cr
    from w4a8_codebook_quantized_b200 import inputs
    case = inputs.CASES[args.swiglu_workload]
    M, N, K = case.M, case.N, case.K
    layer = inputs.layer(N, K, rank_seed(case.seed, rank))
    x = inputs.activations(M, K, rank_seed(case.seed, rank), case.dist)
    q, s, cb, ws = (torch.from_numpy(a).cuda() for a in (layer.qdata, layer.srel, layer.codebook, layer.s_channel))
    xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    xq = torch.empty(M, K, dtype=torch.int8, device="cuda")
    xs = torch.empty(M, dtype=torch.float32, device="cuda")
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    out_sw = torch.empty(M, N // 2, dtype=torch.bfloat16, device="cuda")
    fused = lambda: cr.cr_w4a8_linear_swiglu(xd, q, s, cb, ws, out=out_sw, xq_work=xq, xs_work=xs)
    plain = lambda: cr.cr_w4a8_linear(xd, q, s, cb, ws, out=out, xq_work=xq, xs_work=xs)
    for _ in range(max(3, args.warmup)):
        fused()
        plain()
    steps = max(3, min(args.steps, 20))
    tf, tp = flushed_medians([fused, plain], steps)
    tf, tp = max_over_ranks(tf, world), max_over_ranks(tp, world)
    ops = 2.0 * M * N * K
    return {"workload": f"{case.name} as interleaved gate/up: M={M}, N=2F={N}, K={K}, out [M, {N // 2}]",
            "value": round(world * ops / tf / 1e12, 2), "unit": "TOPS", "ms_per_step": round(tf * 1e3, 4),
            "plain_forward": {"value": round(world * ops / tp / 1e12, 2), "ms_per_step": round(tp * 1e3, 4)},
            "steps": steps, "l2": "256 MiB write between steps, outside the timed events"}


def run_backward(args, world, rank, pk):
    """The straight-through input gradient on the prefill shape: dx [M, K] =
    grad [M, N] @ (w8 * s_channel in bf16), cr_w4a8_ste_backward (the codes
    decoded again into a bf16 transient, then the tcgen05 bf16 GEMM)."""
    import torch

    import w4a8_codebook_quantized_b200 as cr
    from w4a8_codebook_quantized_b200 import inputs
    case = inputs.CASES[args.backward_workload]
    M, N, K = case.M, case.N, case.K
    layer = inputs.layer(N, K, rank_seed(case.seed, rank))
    q, s, cb, ws = (torch.from_numpy(a).cuda() for a in (layer.qdata, layer.srel, layer.codebook, layer.s_channel))
    g = torch.from_numpy(np.random.default_rng(rank_seed(case.seed, rank)).standard_normal((M, N))
                         .astype(np.float32)).to(torch.bfloat16).cuda()
    dx = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    call = lambda: cr.cr_w4a8_ste_backward(g, q, s, cb, ws, dx=dx)
    for _ in range(max(3, args.warmup)):
        call()
    steps = max(3, min(args.steps, 20))
    (t,) = flushed_medians([call], steps)
    t = max_over_ranks(t, world)
    flops = 2.0 * M * N * K
    peak = pk["bf16_tflops"]
    return {"workload": f"{case.name} backward: grad [{M}, {N}] @ w [{N}, {K}]",
            "value": round(world * flops / t / 1e12, 2), "unit": "TFLOP/s", "ms_per_step": round(t * 1e3, 4),
            "steps": steps, "l2": "256 MiB write between steps, outside the timed events",
            "roofline": {"bound": "tensor", "achieved": round(flops / t / 1e12, 1), "peak": round(peak, 1),
                         "unit": "TFLOP/s", "frac": round(flops / t / 1e12 / peak, 4),
                         "peak_source": f"{pk['source']} bf16_tflops",
                         "kernel": "cr_w4a8_ste_backward call (bf16 weight transient + tcgen05 bf16 GEMM)"}}


GROUPED_NS = (4096, 1024, 1024)  # q, k, v of an attention block with 8-way grouped k/v heads


def run_grouped(args, world, rank, local, case):
    """Three layers fed the same decode batch (q/k/v): cr_w4a8_linear_grouped
    (one rotate+quant, one grouped GEMV launch) against three
    cr_w4a8_linear calls, in weight GB/s of the three layers together."""
    import torch

    import w4a8_codebook_quantized_b200 as cr
    from w4a8_codebook_quantized_b200 import inputs
    M, K = case.M, case.K
    wb = sum(weight_bytes(n, K) for n in GROUPED_NS)
    R = max(2, int(math.ceil(1.25 * L2_BYTES / wb)))
    cb = torch.from_numpy(inputs.codebook()).cuda()
    base = []
    for i, n in enumerate(GROUPED_NS):
        ly = inputs.layer(n, K, rank_seed(case.seed + 10 + i, rank))
        base.append(tuple(torch.from_numpy(a).cuda() for a in (ly.qdata, ly.srel, ly.s_channel)))
    sets = [[tuple(t.clone() for t in ly) for ly in base] for _ in range(R)]
    x = inputs.activations(M, K, rank_seed(case.seed, rank), case.dist)
    xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    rows = cr.gemv_rows(M)
    xq = torch.empty(rows, K, dtype=torch.int8, device="cuda")
    xs = torch.empty(rows, dtype=torch.float32, device="cuda")
    outs = [torch.empty(M, n, dtype=torch.bfloat16, device="cuda") for n in GROUPED_NS]

    def grouped_step(i):
        cr.cr_w4a8_linear_grouped(xd, cb, sets[i % R], outs=outs, xq_work=xq, xs_work=xs)

    def separate_step(i):
        for (q, s, ws), o in zip(sets[i % R], outs):
            cr.cr_w4a8_linear(xd, q, s, cb, ws, out=o, xq_work=xq, xs_work=xs)

    tg, _ = graph_time(grouped_step, args.steps, args.warmup, world, local)
    ts, _ = graph_time(separate_step, args.steps, args.warmup, world, local)
    tg, ts = max_over_ranks(tg, world), max_over_ranks(ts, world)
    return {"workload": f"q/k/v of the decode batch: M={M}, K={K}, N={'+'.join(map(str, GROUPED_NS))}",
            "value": round(aggregate_value(wb, args.steps, world, tg), 2), "unit": "GB/s",
            "us_per_step": round(tg / args.steps * 1e6, 3),
            "separate_calls": {"value": round(aggregate_value(wb, args.steps, world, ts), 2),
                               "us_per_step": round(ts / args.steps * 1e6, 3)},
            "gpu_launches_per_step": 2, "l2": f"rotating {R} copies of the three layers"}


# ---------------------------------------------------------------- reference arm

def run_reference(args):
    """The oracle (plain CPU C) timed as the reference arm on the same workload."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from w4a8_codebook_quantized_b200 import inputs
    case = inputs.CASES[args.workload]
    M, N, K = case.M, case.N, case.K
    layer = inputs.layer(N, K, case.seed)
    x = inputs.activations(M, K, case.seed, case.dist)
    oracle.lib()
    # one step = one full forward pass, or a row sample of the layer when K
    # full passes would not finish in about two minutes
    t0 = time.perf_counter()
    oracle.linear(x, layer.qdata, layer.srel, layer.codebook, layer.s_channel, threads=1)
    one = time.perf_counter() - t0
    budget = 120.0
    frac = 1.0
    if one * (args.steps + args.warmup) > budget:
        frac = max(1.0 / 64, budget / (one * (args.steps + args.warmup)))
    rows = max(16, int(N * frac) // 16 * 16)
    sub = inputs.Layer(layer.qdata[:rows], layer.srel[:rows], layer.s_channel[:rows], layer.codebook)
    for _ in range(args.warmup):
        oracle.linear(x, sub.qdata, sub.srel, sub.codebook, sub.s_channel, threads=1)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.linear(x, sub.qdata, sub.srel, sub.codebook, sub.s_channel, threads=1)
    el = time.perf_counter() - t0
    wb = weight_bytes(rows, K)
    value = wb * args.steps / el / 1e9
    sample = (f"each step: full forward of M={M}, K={K} over {rows} of the {N} output rows "
              f"({'whole layer' if rows == N else 'row sample'})")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "s8", "data": "synthetic",
            "config": {"workload": f"{case.name}: decode batch M={M}, N={N}, K={K}, rot 256, group 16, seed {case.seed}",
                       "parallelism": "host CPU, 1 thread"},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

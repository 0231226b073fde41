#!/usr/bin/env python
"""Benchmark of the Mixtral top-2 sparse-MoE layer on B200 through libmoe's C ABI.

One step = one moe_layer_forward over one batch of the workload (router, grouping,
expert SwiGLU FFN on tensor cores, combine).  The default run's headline is the
prefill batch of the Mixtral-8x7B layer (T=4096, d=4096, h=14336, E=8, k=2, bf16),
whose GEMM1 (+SwiGLU) is reported against the bf16 tensor-core peak; the decode
batch (T=16, weight streaming against HBM bandwidth), the skewed-routing and
long-context (T=32768) layers and the prefill backward pass are then timed under
the same rules and reported under ``workloads`` in the same line.
``--workload NAME`` times one workload only.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--backward]
    python bench.py --impl reference ...     # the CPU oracle, timed on host cores

Under torchrun (N > 1) every rank runs its own batch with replicated weights (tokens
are independent, so the work shards with no collective in the data path); the step
time is the max over ranks and ``value`` counts the tokens of all ranks.

Printed: one JSON line (rank 0).  The expert weights (2.8 GB) are larger than L2 and
are streamed every step, so no L2 flush is inserted between steps.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s and % of roofline (bf16 TC peak prefill; HBM GB/s decode)"
UNIT = "tokens/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILES = os.path.join(ROOT, "profiles")
CSRC = os.path.join(ROOT, "sparse_mixture_experts_26_b200", "csrc")
# Dominant kernel of each regime and the file that holds it.
DOMINANT = {
    "decode": ("decode_ffn_fused_kernel (gate/up + silu*gate + split-K down, one cooperative "
               "launch, weight streaming)",
               "decode_ffn_fused", os.path.join(CSRC, "decode_gemm_sm100.cu")),
    "grouped": ("grouped_gemm_kernel<SwiGLU> (GEMM1 + silu*gate epilogue)",
                "grouped_gemm_swiglu", os.path.join(CSRC, "grouped_gemm_sm100.cu")),
    "pair": ("grouped_gemm_pair_kernel<SwiGLU> (CTA-pair GEMM1 + silu*gate epilogue)",
             "grouped_gemm_pair_swiglu", os.path.join(CSRC, "grouped_gemm_pair_sm100.cu")),
}
DECODE_MAX_TOKENS = 128   # up to here the library runs the weight-streaming kernels
PAIR_MIN_TOKENS = 512     # ... and to the CTA-pair kernels here (1024 grouped rows)


# ------------------------------------------------------------------ ranks
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(backend: str):
    import datetime

    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (the slowest rank sets the step time)."""
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ peaks / profiles
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def source_digest(path: str) -> str:
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def ncu_traffic(kernel_tag: str, workload: str, source: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the
    current kernel source (its ``source_sha256_16`` line matches); else None."""
    p = os.path.join(PROFILES, f"{kernel_tag}_{workload}.md")
    if not os.path.exists(p):
        return None
    text = open(p).read()
    m = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    h = re.search(r"source_sha256_16:\s*([0-9a-f]+)", text)
    if not m or not h or h.group(1) != source_digest(source):
        return None
    return float(m.group(1))


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the GPU works."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            phys = device_index
            if vis:
                ids = [v.strip() for v in vis.split(",") if v.strip()]
                if device_index < len(ids) and ids[device_index].isdigit():
                    phys = int(ids[device_index])
            self._h = pynvml.nvmlDeviceGetHandleByIndex(phys)
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None
        self.period = period_s

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append(mhz)
                for name, bit in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ oracle timing
def oracle_tokens_per_s(inp_cpu, sample_tokens, budget_s: float, backward: bool = False):
    """Time the CPU oracle (as it stands) on ``sample_tokens`` tokens of the workload,
    repeating until ``budget_s`` seconds; returns (tokens/s, threads, repeats).  With
    ``backward`` the oracle's gradient pass (which runs its own forward) is timed."""
    from oracle import moe_oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max((p.get("num_threads", 1) for p in threadpool_info()
                       if p.get("user_api") == "blas"), default=1)
    except Exception:
        threads = os.cpu_count() or 1
    x = inp_cpu["x"][:sample_tokens]
    dy = backward_dy_cpu(x.shape)
    t0 = time.perf_counter()
    reps = 0
    while True:
        if backward:
            O.moe_layer_backward(x, inp_cpu["Wg"], inp_cpu["W1"], inp_cpu["W3"], inp_cpu["W2"],
                                 dy)
        else:
            O.moe_layer(x, inp_cpu["Wg"], inp_cpu["W1"], inp_cpu["W3"], inp_cpu["W2"])
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return reps * sample_tokens / dt, int(threads), reps, dt


def backward_dy(T: int, d: int, seed: int = 4242):
    """The seeded upstream gradient dL/dy of the backward benchmark (bf16 values)."""
    import torch
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return torch.randn(T, d, generator=g).to(torch.bfloat16)


def backward_dy_cpu(shape):
    return backward_dy(*shape).float().numpy()


def cpu_copy(inp):
    """Exact host copies of the inputs as float32 numpy arrays (bf16 widens exactly)."""
    return {k: v.float().cpu().numpy() for k, v in inp.items()}


# ------------------------------------------------------------------ workload config
def workload_config(wl, extra=None):
    cfg = {
        "workload": f"{wl.name}: Mixtral-8x7B MoE layer, T={wl.T} d={wl.d} h={wl.h} "
                    f"E={wl.E} top-{wl.k}, {wl.dtype}" if wl.d == 4096 else wl.note,
        "T": wl.T, "d": wl.d, "h": wl.h, "E": wl.E, "k": wl.k, "seed": wl.seed,
        "routing": wl.kind,
        "l2": f"no flush: inputs larger than L2 ({3 * wl.E * wl.d * wl.h * 2 / 1e9:.1f} GB of "
              "expert weights streamed per step)",
    }
    if extra:
        cfg.update(extra)
    return cfg


def algorithmic_bytes_gemm1(wl, touched: int) -> int:
    """W1 and W3 of every touched expert, the gathered rows read, H written."""
    P = wl.T * wl.k
    return touched * 2 * wl.h * wl.d * 2 + P * wl.d * 2 + P * wl.h * 2


DECODE_SPLIT_K = 8  # partial sums the small-batch down projection writes


def algorithmic_bytes_ffn_decode(wl, touched: int) -> int:
    """Whole small-batch FFN: every touched expert's W1, W3, W2 once, the gathered rows
    read, H written and read back, and the split-K fp32 partials written."""
    P = wl.T * wl.k
    return (touched * 3 * wl.h * wl.d * 2 + P * wl.d * 2 + 2 * P * wl.h * 2
            + DECODE_SPLIT_K * P * wl.d * 4)


def algorithmic_flops_gemm1(wl) -> int:
    return 2 * wl.T * wl.k * wl.d * 2 * wl.h


# ------------------------------------------------------------------ our arm
def rank_inputs(wl, rank: int, world: int, device):
    """The workload's tensors on ``device``; every rank past 0 draws its own batch x by
    the same recipe (skewed or long-context rows included) from its own seed, while the
    weights stay the same on every rank."""
    from dataclasses import replace

    from workloads import make_inputs
    inp = make_inputs(wl, device)
    if world > 1 and rank > 0:
        own = replace(wl, seed=wl.seed * 1000 + rank)
        inp["x"] = make_inputs(own, device, weights=False)["x"]
    return inp


ZERO_WEIGHTS_NOTE = ("all-zero expert weights: a diagnostic that keeps the data path and the "
                     "math but draws little power, so the SM clock stays near its maximum")


def zero_expert_weights(inp, args):
    """--zero-weights: W1, W3 and W2 set to zero (x and W_g, hence the routing, unchanged)."""
    if getattr(args, "zero_weights", False):
        for k in ("W1", "W3", "W2"):
            inp[k].zero_()


def regime_of(T: int) -> str:
    if T <= DECODE_MAX_TOKENS:
        return "decode"
    if T >= PAIR_MIN_TOKENS and os.environ.get("MOE_GEMM_PAIR", "1") != "0":
        return "pair"
    return "grouped"


def measure_forward(wl, inp, K: int, W: int, world: int, local: int, device):
    """Time K layer calls (after W warm-up calls) on the launching stream, with CUDA
    events around the expert FFN inside the timed region, then the same K steps end to
    end from pinned host buffers.  Returns the workload's result object (rank-local
    timings already maxed over ranks)."""
    import torch

    import sparse_mixture_experts_26_b200 as moe

    x, Wg, W1, W3, W2 = (inp[k] for k in ("x", "Wg", "W1", "W3", "W2"))
    T, d, h, E = wl.T, wl.d, wl.h, wl.E
    ws = moe.alloc_workspace(T, d, h, E, wl.k, x.dtype, device)
    y = torch.empty_like(x)
    stream = torch.cuda.current_stream(device)

    # Events around the expert FFN only (plus one between its two GEMMs for large
    # batches, where launches do not overlap anyway); the router, permutation and
    # combine run back to back, so small-batch launches keep overlapping their tails.
    fused = wl.T <= DECODE_MAX_TOKENS
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    for row in evs:  # create the underlying CUDA events before handing them over
        for e in row:
            e.record(stream)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    layer_call, events_call = moe.moe_layer_forward, moe.moe_layer_forward_events
    with ClockSampler(local) as clocks:
        for _ in range(W):
            layer_call(x, Wg, W1, W3, W2, y, ws)
        torch.cuda.synchronize()
        barrier(world, device)
        torch.cuda.synchronize()
        start.record(stream)
        for i in range(K):
            events_call(x, Wg, W1, W3, W2, y, ws,
                        [None, evs[i][0].cuda_event, None if fused else evs[i][1].cuda_event,
                         evs[i][2].cuda_event])
        end.record(stream)
        torch.cuda.synchronize()
        barrier(world, device)
    ms_local = start.elapsed_time(end) / K
    flags = moe.moe_device_status(ws)
    if flags:
        raise RuntimeError(f"device status flags {flags:#x} after the timed region")
    ms = max_over_ranks(ms_local, world, device)
    value = world * T / (ms * 1e-3)

    # expert-FFN times per step (same timed region, same stream)
    def span(a, b):
        return sum(evs[i][a].elapsed_time(evs[i][b]) for i in range(K)) / K
    t_ffn = span(0, 2)
    stages_ms = {"expert_ffn": t_ffn, "route+permute+combine": ms_local - t_ffn}
    if not fused:
        t_gemm1 = span(0, 1)
        stages_ms.update(gemm1_swiglu=t_gemm1, gemm2=span(1, 2))

    # routing statistics of this batch (for the algorithmic byte count)
    idx = torch.empty(T, 2, dtype=torch.int32, device=device)
    wts = torch.empty(T, 2, dtype=torch.float32, device=device)
    moe.moe_route(x, Wg, idx, wts)
    counts = torch.bincount(idx.flatten().long(), minlength=E).cpu().numpy()
    touched = int((counts > 0).sum())

    peaks, peak_src = load_peaks()
    regime = regime_of(wl.T)
    kname, tag, ksrc = DOMINANT[regime]
    if regime == "decode":  # weight streaming: HBM-bound, one fused FFN launch
        bound, unit = "hbm", "GB/s"
        ach = algorithmic_bytes_ffn_decode(wl, touched) / (t_ffn * 1e-3) / 1e9
        peak = float(peaks["hbm_gbs"])
        per_launch = {"bytes": algorithmic_bytes_ffn_decode(wl, touched)}
    else:  # grouped GEMM1 (+SwiGLU): tensor-bound
        bound, unit = "tensor", "TFLOP/s"
        ach = algorithmic_flops_gemm1(wl) / (t_gemm1 * 1e-3) / 1e12
        peak = float(peaks["bf16_tflops"])
        per_launch = {"flops": algorithmic_flops_gemm1(wl)}
    traffic = ncu_traffic(tag, wl.name, ksrc)
    roofline = {"bound": bound, "achieved": round(ach, 1), "peak": peak, "unit": unit,
                "frac": round(ach / peak, 4), "traffic": traffic, "kernel": kname,
                "peak_source": f"{peak_src} ({'burst' if bound == 'tensor' else 'copy'})",
                "algorithmic_per_launch": per_launch,
                "launch_ms": round(t_ffn if regime == "decode" else t_gemm1, 4)}
    if bound == "tensor" and "bf16_tflops_sustained" in peaks:
        roofline["frac_of_sustained"] = round(ach / float(peaks["bf16_tflops_sustained"]), 4)
    layer_bytes = touched * 3 * h * d * 2 + T * d * 2 * 2
    layer = {"ms": round(ms, 4), "tflops": round(wl.active_flops() / (ms * 1e-3) / 1e12, 1),
             "hbm_gbs": round(layer_bytes / (ms * 1e-3) / 1e9, 1),
             "experts_touched": touched, "rows_per_expert": [int(c) for c in counts],
             "stage_ms": {k: round(v, 4) for k, v in stages_ms.items()}}
    if regime != "decode":
        layer["frac_of_peak"] = round(wl.active_flops() / (ms * 1e-3) / 1e12 / peak, 4)

    # End to end through the public API with host buffers: every step copies its x
    # from pinned host memory, runs moe_layer_forward and reads y back to pinned host
    # memory.  Copies run on their own streams, double-buffered, so step i+1's input
    # copy and step i-1's output copy overlap step i's layer (as a serving loop would);
    # every step's copies are inside the timed region.
    x_host = x.cpu().pin_memory()
    y_host = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(x) for _ in range(2)]
    y_dev = [torch.empty_like(y) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_layer = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for e in ev_layer + ev_out:
        e.record(stream)

    def e2e_steps(n):
        for i in range(n):
            b = i & 1
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_layer[b])          # x_dev[b] no longer read
                x_dev[b].copy_(x_host, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])              # y_dev[b] already copied out
            layer_call(x_dev[b], Wg, W1, W3, W2, y_dev[b], ws)
            ev_layer[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_layer[b])
                y_host[b].copy_(y_dev[b], non_blocking=True)
                ev_out[b].record(s_out)

    e2e_steps(2)
    torch.cuda.synchronize()
    barrier(world, device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    e2e_steps(K)
    s_out.wait_stream(stream)
    e1.record(s_out)
    torch.cuda.synchronize()
    barrier(world, device)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / K, world, device)
    e2e = {"value": round(world * T / (e2e_ms * 1e-3), 1), "unit": UNIT,
           "h2d_bytes_per_step": x.numel() * x.element_size(),
           "d2h_bytes_per_step": y.numel() * y.element_size(),
           "pipeline": "double-buffered: H2D and D2H copies on their own streams"}
    launches = moe.launches_per_layer(T, d, E, wl.dtype == "bf16")
    return {"value": round(value, 1), "unit": UNIT, "steps": K, "warmup": W,
            "ms_per_step": round(ms, 4), "config": workload_config(wl),
            "roofline": roofline, "layer": layer, "e2e": e2e,
            "gpu_launches": launches * K, "clocks": clocks.summary()}


# Batches between the two measured serving regimes (the grouped-GEMM range, 129..511
# tokens), with plain and skewed routing: the layer alone, no events inside the timed
# region, against the copy bandwidth (the layer reads each touched expert's weights once).
SWEEP_TOKENS = (192, 256, 384)
SWEEP_ROUTINGS = ("prefill", "skew")


def measure_layer_only(wl, inp, K: int, W: int, world: int, local: int, device):
    import torch

    import sparse_mixture_experts_26_b200 as moe

    x, Wg, W1, W3, W2 = (inp[k] for k in ("x", "Wg", "W1", "W3", "W2"))
    T, d, h, E = wl.T, wl.d, wl.h, wl.E
    ws = moe.alloc_workspace(T, d, h, E, wl.k, x.dtype, device)
    y = torch.empty_like(x)
    stream = torch.cuda.current_stream(device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        for _ in range(W):
            moe.moe_layer_forward(x, Wg, W1, W3, W2, y, ws)
        torch.cuda.synchronize()
        barrier(world, device)
        start.record(stream)
        for _ in range(K):
            moe.moe_layer_forward(x, Wg, W1, W3, W2, y, ws)
        end.record(stream)
        torch.cuda.synchronize()
        barrier(world, device)
    if moe.moe_device_status(ws):
        raise RuntimeError("device status flags set after the timed region")
    ms = max_over_ranks(start.elapsed_time(end) / K, world, device)
    idx = torch.empty(T, 2, dtype=torch.int32, device=device)
    wts = torch.empty(T, 2, dtype=torch.float32, device=device)
    moe.moe_route(x, Wg, idx, wts)
    counts = torch.bincount(idx.flatten().long(), minlength=E).cpu().numpy()
    touched = int((counts > 0).sum())
    layer_bytes = touched * 3 * h * d * 2 + T * d * 2 * 2
    peaks, peak_src = load_peaks()
    gbs = layer_bytes / (ms * 1e-3) / 1e9
    return {"T": T, "routing": "skewed" if wl.kind == "skew" else "plain",
            "ms": round(ms, 4), "tokens_per_s": round(world * T / (ms * 1e-3), 1),
            "experts_touched": touched, "rows_per_expert": [int(c) for c in counts],
            "layer_bytes": int(layer_bytes), "hbm_gbs": round(gbs, 1),
            "frac_of_copy": round(gbs / float(peaks["hbm_gbs"]), 4),
            "peak_source": f"{peak_src} (copy)", "clocks": clocks.summary()}


def forward_cpu_baseline(inp, wl, args):
    n = min(wl.T, args.cpu_sample_tokens)
    tps, threads, reps, dt = oracle_tokens_per_s(cpu_copy(inp), n, args.cpu_budget_s)
    return {"value": round(tps, 3), "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"fp64 numpy oracle on the first {n} tokens of the {wl.name} batch "
                      f"(T={wl.T}), {reps} repeat(s) in {dt:.1f} s"}


def free_device_memory():
    import gc

    import torch
    gc.collect()
    torch.cuda.empty_cache()


# The default run: the prefill layer is the headline (its GEMM1 against the bf16
# tensor-core peak); the decode, skewed and long-context layers and the prefill
# backward are measured under the same timed-region rules and reported beside it.
SUITE_HEADLINE = "prefill"
SUITE_FORWARD = ("decode", "skew", "long")
SUITE_BACKWARD = ("prefill",)
DECODE_STEP_FACTOR = 10   # decode steps are ~0.4 ms: time 10x as many


def run_ours(args):
    import torch

    from workloads import WORKLOADS

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist("nccl")
    K, W = args.steps, args.warmup
    suite = args.workload is None
    name = SUITE_HEADLINE if suite else args.workload
    wl = with_tokens(WORKLOADS[name], args)
    inp = rank_inputs(wl, rank, world, device)
    zero_expert_weights(inp, args)
    head = measure_forward(wl, inp, K, W, world, local, device)
    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu_baseline = forward_cpu_baseline(inp, wl, args)
    del inp
    free_device_memory()

    sub = {}
    if suite and not args.headline_only:
        def forward_workload(other):
            owl = WORKLOADS[other]
            oinp = rank_inputs(owl, rank, world, device)
            k = K * DECODE_STEP_FACTOR if owl.T <= DECODE_MAX_TOKENS else K
            sub[other] = measure_forward(owl, oinp, k, W, world, local, device)
            del oinp
            free_device_memory()

        # the long-context layer runs for seconds at the power limit, so the
        # bandwidth-bound sweep goes before it
        for other in SUITE_FORWARD:
            if other != "long":
                forward_workload(other)
        sweep = []
        for T in SWEEP_TOKENS:
            for routing in SWEEP_ROUTINGS:
                owl = WORKLOADS[routing].with_tokens(T)
                oinp = rank_inputs(owl, rank, world, device)
                sweep.append(measure_layer_only(owl, oinp, K, W, world, local, device))
                del oinp
                free_device_memory()
        sub["batch_sweep"] = {
            "what": "layer time at batches between the small-batch and CTA-pair kernels "
                    "(grouped GEMMs), no events inside the timed region; bytes = touched "
                    "experts' weights + x + y",
            "steps": K, "warmup": W, "points": sweep}
        if "long" in SUITE_FORWARD:
            forward_workload("long")
        for other in SUITE_BACKWARD:
            owl = WORKLOADS[other]
            oinp = rank_inputs(owl, rank, world, device)
            sub[f"backward_{other}"] = measure_backward(owl, oinp, K, W, world, local, device)
            del oinp
            free_device_memory()

    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return None
    out = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype,
        "data": "synthetic (seeded normal draws of the Mixtral-8x7B layer shapes; "
                "random-init weights)",
        "config": workload_config(wl, {"parallelism": parallelism(world)}
                                  | ({"weights": ZERO_WEIGHTS_NOTE} if args.zero_weights else {})),
        "roofline": head["roofline"], "layer": head["layer"], "cpu_baseline": cpu_baseline,
        "e2e": head["e2e"], "gpu_launches": head["gpu_launches"], "clocks": head["clocks"],
    }
    if sub:
        out["workloads"] = sub
    return out


def with_tokens(wl, args):
    """The workload at --tokens tokens (same recipe and seed), if given."""
    if getattr(args, "tokens", None):
        if args.workload is None:
            raise SystemExit("--tokens needs --workload")
        return wl.with_tokens(args.tokens)
    return wl


def parallelism(world: int) -> str:
    return f"replicas x{world} (tokens sharded, weights replicated)"


# ------------------------------------------------------------------ our arm, backward
BWD_METRIC = "MoE-layer backward tokens/s (dx, dW1, dW3, dW2, dWg) and % of bf16 TC peak"
BWD_STAGES = ["prep (dY, dw, dlogits)", "dH = dY W2", "du, dv",
              "dX = [du dv][W1; W3]", "dx combine", "dW2", "dW1 + dW3", "dWg"]
BWD_KERNELS = (1, 2, 3, 5, 6)  # the tensor-core stages
BWD_PAIR_MIN_ROWS = 2048      # row GEMMs on CTA pairs from here (grouped rows)
BWD_WGRAD_SHORT_ROWS = 1024   # weight gradients on single SMs up to here


def backward_kernel(wl, stage: int):
    """(kernel name, profile tag) of a backward GEMM stage for this workload."""
    P = wl.T * wl.k
    if stage in (5, 6):
        single = P <= BWD_WGRAD_SHORT_ROWS
        name = ("bwd_wgrad_kernel<%s>" % ("kModeW2" if stage == 5 else "kModeW13") if single
                else "bwd_wgrad_pair_kernel")
        return name, "bwd_wgrad_w2" if stage == 5 else "bwd_wgrad_w13"
    pair = P >= BWD_PAIR_MIN_ROWS
    names = {1: ("grouped_gemm_pair_kernel<StoreF32, B MN-major>", "bwd_rows_kernel<kModeDH>"),
             2: ("grouped_gemm_pair_kernel<BwdSwiGLU>", "bwd_rows_kernel<kModeDUV>"),
             3: ("grouped_gemm_pair_kernel<StoreF32, B MN-major split>", "bwd_rows_kernel<kModeDX>")}
    return names[stage][0 if pair else 1], {1: "bwd_dh", 2: "bwd_duv", 3: "bwd_dx"}[stage]


def keeps_pre_activations(wl) -> bool:
    """The training forward keeps a and b at every batch size, and the backward's du/dv
    step is element-wise instead of a second GEMM1."""
    return wl.T > 0


def backward_stage_flops(wl):
    """Tensor-core flops of each GEMM stage (2*P*d*h units; P = 2T grouped rows); the
    du/dv step counts only where it recomputes a and b."""
    u = 2 * (wl.T * wl.k) * wl.d * wl.h
    f = {1: u, 2: 2 * u, 3: 2 * u, 5: u, 6: 2 * u}
    if keeps_pre_activations(wl):
        del f[2]
    return f


def wgrad_bytes(wl, stage: int) -> int:
    """Algorithmic bytes of a weight-gradient launch: fp32 outputs written once, the
    two grouped bf16 operands read once (stage 5: dW2 from dY and H; stage 6: dW1 and
    dW3 from [du dv] and x)."""
    P = wl.T * wl.k
    if stage == 5:
        return wl.E * wl.d * wl.h * 4 + P * (wl.d + wl.h) * 2
    return 2 * wl.E * wl.h * wl.d * 4 + P * (2 * wl.h + wl.d) * 2


def measure_backward(wl, inp, K: int, W: int, world: int, local: int, device):
    """Time K backward calls (after one training forward that fills the saved state --
    it keeps the pre-activations a, b, so the backward computes du, dv element by
    element -- and W warm-up calls), with events between the backward's
    stages inside the timed region, then K training and K plain forward calls (the
    training forward's cost), then the same backward steps end to end (dy in, dx out
    through pinned host buffers).  Returns the workload's result object."""
    import torch

    import sparse_mixture_experts_26_b200 as moe
    from workloads import WORKLOADS

    if wl.dtype != "bf16":
        raise SystemExit("the backward pass is built for bf16 layers")
    x, Wg, W1, W3, W2 = (inp[k] for k in ("x", "Wg", "W1", "W3", "W2"))
    T, d, h, E = wl.T, wl.d, wl.h, wl.E
    ws = moe.alloc_workspace(T, d, h, E, wl.k, x.dtype, device)
    bws = moe.alloc_backward_workspace(T, d, h, E, wl.k, x.dtype, device)
    y = torch.empty_like(x)
    moe.moe_layer_forward_train(x, Wg, W1, W3, W2, y, ws, bws)  # the state the backward reads
    dy = backward_dy(T, d).to(device)
    dx = torch.empty_like(x)
    f32 = dict(dtype=torch.float32, device=device)
    dWg, dW1 = torch.empty(Wg.shape, **f32), torch.empty(W1.shape, **f32)
    dW3, dW2 = torch.empty(W3.shape, **f32), torch.empty(W2.shape, **f32)
    stream = torch.cuda.current_stream(device)
    nst = len(BWD_STAGES) + 1
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nst)] for _ in range(K)]
    for row in evs:
        for e in row:
            e.record(stream)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def step(dy_, dx_, ev=None):
        if ev is None:
            moe.moe_layer_backward(x, Wg, W1, W3, W2, dy_, dx_, dWg, dW1, dW3, dW2, ws, bws)
        else:
            moe.moe_layer_backward_events(x, Wg, W1, W3, W2, dy_, dx_, dWg, dW1, dW3, dW2, ws,
                                          bws, [e.cuda_event for e in ev])

    with ClockSampler(local) as clocks:
        for _ in range(W):
            step(dy, dx)
        torch.cuda.synchronize()
        barrier(world, device)
        torch.cuda.synchronize()
        start.record(stream)
        for i in range(K):
            step(dy, dx, evs[i])
        end.record(stream)
        torch.cuda.synchronize()
        barrier(world, device)
    ms_local = start.elapsed_time(end) / K
    flags = moe.moe_device_status(bws)
    if flags:
        raise RuntimeError(f"device status flags {flags:#x} after the timed region")
    ms = max_over_ranks(ms_local, world, device)
    value = world * T / (ms * 1e-3)
    st_ms = [sum(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(K)) / K
             for j in range(nst - 1)]
    flops = backward_stage_flops(wl)
    dom = max((j for j in BWD_KERNELS if j in flops), key=lambda j: st_ms[j])
    kname, tag = backward_kernel(wl, dom)
    peaks, peak_src = load_peaks()
    if T <= DECODE_MAX_TOKENS and dom in (5, 6):
        # a few rows per expert: the weight-gradient GEMMs are bound by writing their
        # fp32 outputs, so their roofline is HBM bandwidth
        bound, unit, peak_kind = "hbm", "GB/s", "copy"
        ach = wgrad_bytes(wl, dom) / (st_ms[dom] * 1e-3) / 1e9
        peak = float(peaks["hbm_gbs"])
        per_launch = {"bytes": wgrad_bytes(wl, dom)}
    else:
        bound, unit, peak_kind = "tensor", "TFLOP/s", "burst"
        ach = flops[dom] / (st_ms[dom] * 1e-3) / 1e12
        peak = float(peaks["bf16_tflops"])
        per_launch = {"flops": flops[dom]}
    src = os.path.join(CSRC, "backward_pair_sm100.cu" if "pair" in kname else "backward_sm100.cu")
    if dom in (1, 2, 3) and "pair" in kname:
        src = os.path.join(CSRC, "grouped_gemm_pair_sm100.cu")
    traffic, traffic_note = ncu_traffic(tag, wl.name, src), None
    if traffic is None and wl.name == "prefill" and dom in (5, 6):
        # The full backward holds ~10 GB, too much for a --set full capture: scale the
        # half-width capture (same rows per expert) by the kernel's algorithmic bytes.
        t_half = ncu_traffic(tag, "prefill_half", src)
        if t_half is not None:
            half = WORKLOADS["prefill_half"]
            traffic = round(t_half * wgrad_bytes(wl, dom) / wgrad_bytes(half, dom))
            traffic_note = ("scaled from the prefill_half capture by algorithmic bytes "
                            f"({wgrad_bytes(wl, dom) / wgrad_bytes(half, dom):.2f}x)")
    roofline = {"bound": bound, "achieved": round(ach, 1), "peak": peak, "unit": unit,
                "frac": round(ach / peak, 4), "traffic": traffic,
                "kernel": f"{kname} (stage '{BWD_STAGES[dom]}')",
                "peak_source": f"{peak_src} ({peak_kind})",
                "algorithmic_per_launch": per_launch, "launch_ms": round(st_ms[dom], 4)}
    if traffic_note:
        roofline["traffic_note"] = traffic_note
    if bound == "tensor" and "bf16_tflops_sustained" in peaks:
        # the backward runs for seconds under the power limit: the sustained figure
        roofline["frac_of_sustained"] = round(ach / float(peaks["bf16_tflops_sustained"]), 4)
    total_flops = sum(flops.values())
    layer = {"ms": round(ms, 4), "tflops": round(total_flops / (ms * 1e-3) / 1e12, 1),
             "stage_ms": {n: round(v, 4) for n, v in zip(BWD_STAGES, st_ms)},
             "stage_tflops": {BWD_STAGES[j]: round(flops[j] / (st_ms[j] * 1e-3) / 1e12, 1)
                              for j in flops}}

    # The forward a training step pays: moe_layer_forward (nothing kept) and
    # moe_layer_forward_train (a and b kept), K calls each, in four alternating blocks
    # (the power limit slows whichever runs later), the training one last so that the
    # end-to-end backward steps below read the state it keeps.
    def time_block(call, n):
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        barrier(world, device)
        f0.record(stream)
        for _ in range(n):
            call()
        f1.record(stream)
        torch.cuda.synchronize()
        barrier(world, device)
        return f0.elapsed_time(f1)
    plain = lambda: moe.moe_layer_forward(x, Wg, W1, W3, W2, y, ws)  # noqa: E731
    train = lambda: moe.moe_layer_forward_train(x, Wg, W1, W3, W2, y, ws, bws)  # noqa: E731
    plain()
    train()
    blocks = [K // 4 + (1 if j < K % 4 else 0) for j in range(4)]
    tot = {"plain": 0.0, "train": 0.0}
    for j, n in enumerate(blocks):
        if n == 0:
            continue
        order = (("plain", plain), ("train", train)) if j % 2 == 0 else \
            (("train", train), ("plain", plain))
        for name, call in order:
            tot[name] += time_block(call, n)
    train()
    fwd_ms = max_over_ranks(tot["plain"] / K, world, device)
    fwd_train_ms = max_over_ranks(tot["train"] / K, world, device)
    layer["forward_ms"] = round(fwd_ms, 4)
    layer["forward_train_ms"] = round(fwd_train_ms, 4)
    layer["train_step_ms"] = round(fwd_train_ms + ms, 4)
    layer["pre_activations_kept"] = keeps_pre_activations(wl)

    # End to end through the public API with host buffers: dy in from pinned host memory,
    # dx back to pinned host memory, both on their own streams, double-buffered; the
    # weight gradients stay on the device for the optimizer.
    dy_host = dy.cpu().pin_memory()
    dx_host = [torch.empty(dx.shape, dtype=dx.dtype).pin_memory() for _ in range(2)]
    dy_dev = [torch.empty_like(dy) for _ in range(2)]
    dx_dev = [torch.empty_like(dx) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_step = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for e in ev_step + ev_out:
        e.record(stream)

    def e2e_steps(n):
        for i in range(n):
            b = i & 1
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_step[b])
                dy_dev[b].copy_(dy_host, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])
            step(dy_dev[b], dx_dev[b])
            ev_step[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_step[b])
                dx_host[b].copy_(dx_dev[b], non_blocking=True)
                ev_out[b].record(s_out)

    e2e_steps(2)
    torch.cuda.synchronize()
    barrier(world, device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    e2e_steps(K)
    s_out.wait_stream(stream)
    e1.record(s_out)
    torch.cuda.synchronize()
    barrier(world, device)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / K, world, device)
    e2e = {"value": round(world * T / (e2e_ms * 1e-3), 1), "unit": UNIT,
           "h2d_bytes_per_step": dy.numel() * dy.element_size(),
           "d2h_bytes_per_step": dx.numel() * dx.element_size(),
           "pipeline": "double-buffered: dy in and dx out on their own streams; weight "
                       "gradients stay on the device"}
    return {"metric": BWD_METRIC, "value": round(value, 1), "unit": UNIT, "steps": K,
            "warmup": W, "ms_per_step": round(ms, 4),
            "config": workload_config(wl, {"pass": "backward (after one forward that fills "
                                                   "the saved state)"}),
            "roofline": roofline, "layer": layer, "e2e": e2e,
            "gpu_launches": moe.launches_per_backward(T) * K, "clocks": clocks.summary()}


def run_ours_backward(args):
    import torch

    from workloads import WORKLOADS

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist("nccl")
    wl = with_tokens(WORKLOADS[args.workload or SUITE_HEADLINE], args)
    inp = rank_inputs(wl, rank, world, device)
    zero_expert_weights(inp, args)
    r = measure_backward(wl, inp, args.steps, args.warmup, world, local, device)
    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n = min(wl.T, args.cpu_sample_tokens_bwd)
        tps, threads, reps, dt = oracle_tokens_per_s(cpu_copy(inp), n, args.cpu_budget_s,
                                                     backward=True)
        cpu_baseline = {"value": round(tps, 3), "unit": UNIT, "cores": threads,
                        "kind": "oracle",
                        "sample": f"fp64 numpy oracle backward (with its forward) on the "
                                  f"first {n} tokens of the batch, {reps} repeat(s) in "
                                  f"{dt:.1f} s"}
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return None
    cfg = dict(r["config"], parallelism=parallelism(world))
    if args.zero_weights:
        cfg["weights"] = ZERO_WEIGHTS_NOTE
    return {
        "metric": BWD_METRIC, "value": r["value"], "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype,
        "data": "synthetic (seeded normal draws of the Mixtral-8x7B layer shapes and of dy; "
                "random-init weights)",
        "config": cfg, "roofline": r["roofline"], "layer": r["layer"],
        "cpu_baseline": cpu_baseline, "e2e": r["e2e"], "gpu_launches": r["gpu_launches"],
        "clocks": r["clocks"],
    }


# ------------------------------------------------------------------ reference arm
def run_reference(args):
    """The CPU oracle as it stands, on host cores, on a bounded sample per step."""
    import torch

    from workloads import WORKLOADS, make_inputs

    rank, world, _ = dist_env()
    if rank != 0:
        return None
    wl = with_tokens(WORKLOADS[args.workload or SUITE_HEADLINE], args)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp_cpu = cpu_copy(make_inputs(wl, dev))
    n = min(wl.T, args.cpu_sample_tokens)
    from oracle import moe_oracle as O
    if args.backward:
        n = min(wl.T, args.cpu_sample_tokens_bwd)
    x = inp_cpu["x"][:n]
    dy = backward_dy_cpu(x.shape)

    def one():
        if args.backward:
            O.moe_layer_backward(x, inp_cpu["Wg"], inp_cpu["W1"], inp_cpu["W3"], inp_cpu["W2"],
                                 dy)
        else:
            O.moe_layer(x, inp_cpu["Wg"], inp_cpu["W1"], inp_cpu["W3"], inp_cpu["W2"])

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    dt = time.perf_counter() - t0
    ms = dt / args.steps * 1e3
    value = n / (ms * 1e-3)
    try:
        from threadpoolctl import threadpool_info
        threads = max((p.get("num_threads", 1) for p in threadpool_info()
                       if p.get("user_api") == "blas"), default=1)
    except Exception:
        threads = os.cpu_count() or 1
    sample = (f"fp64 numpy oracle {'backward (with its forward) ' if args.backward else ''}"
              f"on the first {n} of the batch's {wl.T} tokens per step")
    return {
        "impl": "reference", "metric": BWD_METRIC if args.backward else METRIC, "value": round(value, 3), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, dict({"pass": "backward"} if args.backward else {},
                                           parallelism=parallelism(world))),
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": int(threads),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=None,
                    choices=["decode", "prefill", "skew", "long", "tiny_f32", "prefill_half"],
                    help="time one workload only (default: the prefill headline plus the "
                         "decode, skew and long layers and the prefill backward)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="with --workload: the same recipe at this many tokens")
    ap.add_argument("--zero-weights", action="store_true",
                    help="with --workload: all-zero expert weights (power diagnostic)")
    ap.add_argument("--headline-only", action="store_true",
                    help="default run without the other workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-tokens", type=int, default=16)
    ap.add_argument("--cpu-budget-s", type=float, default=10.0)
    ap.add_argument("--backward", action="store_true",
                    help="time the layer's backward pass instead of its forward")
    ap.add_argument("--cpu-sample-tokens-bwd", type=int, default=4)
    args = ap.parse_args(argv)
    ref = args.impl == "reference"
    if args.steps is None:
        args.steps = 3 if ref else (200 if args.workload == "decode" else 20)
    if args.warmup is None:
        args.warmup = 1 if ref else 10
    if not ref and args.warmup < 3:
        args.warmup = 3
    if args.zero_weights and (args.workload is None or ref):
        raise SystemExit("--zero-weights needs --workload (our arm)")
    if ref:
        out = run_reference(args)
    else:
        out = run_ours_backward(args) if args.backward else run_ours(args)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()

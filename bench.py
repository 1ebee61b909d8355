#!/usr/bin/env python
"""Benchmark of the MoE layer forward pass on B200 GPUs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--dtype bf16|f32] [--cf CF] [--impl ours|reference]

One step = one whole forward pass of the layer (router -> dispatch ->
grouped expert FFN -> combine -> statistics) over one batch of the
workload's synthetic tokens, inputs resident in HBM.  The default workload
is the largest single-GPU one, the large top-2 layer (T=8192, d=4096,
ff=14336, 8 experts, bf16, no capacity limit), where the expert FFN is
bound by the tensor cores.  L2 is flushed (a 256 MiB write) before every
step, outside the per-step device timing.

With N > 1 (torchrun, one process per GPU) every rank runs an independent
replica of the same layer: there is no data-path collective.  The timed
region is bracketed by a barrier and a device synchronisation on both
sides; its device time is reduced with MAX over ranks and the value is the
tokens processed by all ranks divided by that time.

Rank 0 prints one JSON line.  ``--impl reference`` times the float64 CPU
oracle (the correctness reference, a deliberately plain program) on a
bounded sample of the same workload on the host cores instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE layer tokens/s on 1 B200; expert-FFN TFLOP/s as % of bf16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
# dense bf16 tensor-core rate of one SM per cycle (tcgen05.mma kind::f16: a
# 128 x 256 x 16 MMA every 128 cycles; NVIDIA's nominal 2.25 PFLOP/s dense
# bf16 over 148 SMs at about 1.86 GHz)
TC_FLOP_PER_SM_CYCLE = 8192


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="large-top2")
    ap.add_argument("--dtype", default=None, help="bf16 or f32 (switch-top1 only; default bf16)")
    ap.add_argument("--cf", type=float, default=None, help="capacity factor (switch-top1: 1.0 or 1.5)")
    ap.add_argument("--shared", type=int, default=0, help="shared always-on experts added to the workload")
    ap.add_argument("--reroute", type=int, default=0,
                    help="rounds of overflow rerouting for assignments dropped at capacity (0: drop)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="budget for the oracle baseline")
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end leg (profiling runs: keeps device memory to one layer)")
    return ap.parse_args(argv)


def get_workload(args):
    from mixture_experts_layer_45_b200 import workloads as wl
    kw = {}
    if args.dtype is not None:
        kw["dtype"] = args.dtype
    if args.cf is not None:
        kw["cf"] = args.cf
    if args.shared:
        kw["shared"] = args.shared
    return wl.workload(args.workload, **kw)


def workload_label(w, reroute: int = 0) -> str:
    return (f"{w.name} T={w.T} d={w.d} ff={w.ff} E={w.E} k={w.k} {w.dtype} "
            f"cf={w.capacity_factor_label()}" + (f" shared={w.shared}" if w.shared else "")
            + (f" reroute={reroute}" if reroute else ""))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS if k in d}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# clocks sampled during the timed region (NVML, in-process)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {  # NVML clocks-event-reason bits
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, interval_s: float = 0.005):
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception as e:  # NVML unavailable: report it, do not guess
            self.error = str(e)
        self._interval = interval_s
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                util = nv.nvmlDeviceGetUtilizationRates(self._h).gpu
                self.samples.append((mhz, reasons, util))
            except Exception:
                pass
            time.sleep(self._interval)

    def start(self):
        if self._ok:
            self._t.start()
        return self

    def stop(self):
        if self._ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self._ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "error", "")}
        loaded = [s for s in self.samples if s[2] > 0] or self.samples
        reasons = set()
        for _, r, _ in loaded:
            for bit, name in self.REASONS.items():
                if r & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median([s[0] for s in loaded]) if loaded else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons), "samples": len(loaded)}


# ---------------------------------------------------------------------------
# the committed ncu traffic summary for the dominant kernel (null when the
# kernel sources changed since it was captured)
# ---------------------------------------------------------------------------
KERNEL_SOURCES = {
    "ffn1": ["ffn.cuh", "common.cuh"], "ffn2": ["ffn.cuh", "common.cuh"],
    "router": ["router.cuh", "common.cuh"], "combine": ["dispatch.cuh", "common.cuh"],
    "gather": ["dispatch.cuh", "common.cuh"], "permute": ["dispatch.cuh", "common.cuh"],
}
# fp32 layers run the grouped FFN in ffn_f32.cuh (which builds on ffn.cuh)
KERNEL_SOURCES_F32 = {"ffn1": ["ffn_f32.cuh", "ffn.cuh", "common.cuh"],
                      "ffn2": ["ffn_f32.cuh", "ffn.cuh", "common.cuh"]}


def kernel_source_hash(kernel: str, dtype: str = "bf16") -> str:
    """Hash of the sources of one kernel of the layer (for dtype's path)."""
    files = (KERNEL_SOURCES_F32 if dtype == "f32" else {}).get(kernel, KERNEL_SOURCES.get(kernel, []))
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "mixture_experts_layer_45_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def tag_dtype(workload_tag: str) -> str:
    """The dtype named in a workload tag (<name>-<dtype>-cf<..>)."""
    return "f32" if "-f32-" in workload_tag else "bf16"


def committed_traffic(kernel: str, workload_tag: str):
    """Per-launch DRAM bytes from profiles/<kernel>_<workload_tag>.md, or None."""
    p = os.path.join(ROOT, "profiles", f"{kernel}_{workload_tag}.md")
    if not os.path.exists(p):
        return None
    text = open(p).read()
    m = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    s = re.search(r"source_hash:\s*([0-9a-f]+)", text)
    if not m or not s or s.group(1) != kernel_source_hash(kernel, tag_dtype(workload_tag)):
        return None
    return float(m.group(1))


def workload_tag(w) -> str:
    return f"{w.name}-{w.dtype}-cf{w.capacity_factor_label()}" + (f"-shared{w.shared}" if w.shared else "")


# ---------------------------------------------------------------------------
# the oracle on the host cores (CPU baseline / reference arm)
# ---------------------------------------------------------------------------
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"), default=1)
    except Exception:
        return None


# float64 work of one oracle pass over a sample, kept near this many flops so
# a pass takes about a second on a host's cores whatever the workload
ORACLE_FLOPS_PER_PASS = 32e9


def oracle_sample_tokens(w, most: int) -> int:
    """Tokens of the oracle's sample: at most `most`, fewer where each token
    costs more (the expert FFN is 4*k*d*ff flops per token), at least 16;
    a power of two."""
    per_token = 4.0 * (w.k + w.shared) * w.d * w.ff
    n = max(16, min(most, w.T, int(ORACLE_FLOPS_PER_PASS // per_token)))
    return 1 << (n.bit_length() - 1)


def oracle_sample_inputs(w, sample_T, drawn=None):
    """A bounded sample of the workload: its first sample_T tokens (the same
    seeded draws), with the capacity recomputed for the sample's size.  The
    arrays are widened to float64 once here, outside any timing (the oracle
    computes in float64; bf16 and fp32 values are exact in it)."""
    import numpy as np
    from mixture_experts_layer_45_b200 import workloads as wl
    inp = dict(wl.draw_inputs(w) if drawn is None else drawn)
    inp["x"] = inp["x"][:sample_T]
    inp = {key: (None if v is None else np.asarray(v, np.float64)) for key, v in inp.items()}
    from oracle import moe_ref
    cap = moe_ref.capacity(sample_T, w.k, w.E, w.cf)
    return inp, cap


def time_oracle(w, seconds: float, sample_T: int, drawn=None):
    from oracle import moe_ref
    inp, cap = oracle_sample_inputs(w, sample_T, drawn)
    moe_ref.moe_layer(inp, w.k, cap)          # warm-up
    t0 = time.perf_counter()
    n = 0
    while True:
        moe_ref.moe_layer(inp, w.k, cap)
        n += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return n * sample_T / dt, n, dt


def cpu_baseline(w, seconds: float, drawn=None):
    sample_T = oracle_sample_tokens(w, 1024)
    tps, n, dt = time_oracle(w, seconds, sample_T, drawn)
    cores = len(os.sched_getaffinity(0))
    return {"value": tps, "unit": "tokens/s", "cores": cores, "blas_threads": blas_threads(),
            "kind": "oracle",
            "sample": f"{n} float64 oracle passes over the first {sample_T} tokens of {workload_label(w)} "
                      f"(capacity recomputed for the sample; inputs widened to float64 before timing), "
                      f"{dt:.1f} s wall"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = get_workload(args)
    from oracle import moe_ref
    sample_T = oracle_sample_tokens(w, 512)
    inp, cap = oracle_sample_inputs(w, sample_T)
    for _ in range(args.warmup):
        moe_ref.moe_layer(inp, w.k, cap)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        moe_ref.moe_layer(inp, w.k, cap)
    dt = time.perf_counter() - t0
    value = args.steps * sample_T / dt
    cores = len(os.sched_getaffinity(0))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * dt / max(args.steps, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded numpy draws)",
        "config": {"workload": workload_label(w), "sample_tokens_per_step": sample_T,
                   "parallelism": "host cores (rank 0 only)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "blas_threads": blas_threads(),
                         "kind": "oracle",
                         "sample": f"each step: float64 oracle over the first {sample_T} tokens"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# multi-rank timing aggregation (replicas: no data-path collective)
# ---------------------------------------------------------------------------
def reduce_max_ms(ms: float, device=None) -> float:
    """MAX of a per-rank device time over all ranks (identity on one rank)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(world: int, steps: int, tokens_per_step: int, max_ms: float) -> float:
    """Tokens processed by all ranks divided by the slowest rank's time."""
    return world * steps * tokens_per_step / (max_ms / 1000.0)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def algorithmic_bytes(kernel, w, R, E_active, es):
    """Bytes one launch must move at least: every operand read once, every
    result written once.  S shared experts add S weight panels and S*T rows
    to both FFN GEMMs (they read x once) and S*T rows to the combine."""
    d, ff, T, k, E, S = w.d, w.ff, w.T, w.k, w.E, w.shared
    if kernel == "ffn1":
        return ((E_active + S) * ff * d * es + (E + S) * ff * es + R * d * es + (T * d * es if S else 0)
                + (R + S * T) * ff * es)
    if kernel == "ffn2":
        return ((E_active + S) * d * ff * es + (E + S) * d * es + (R + S * T) * ff * es + (R + S * T) * d * es
                + R * 4)
    if kernel == "router":
        return T * d * es + E * d * es + T * k * 8 + E * 4
    if kernel == "permute":
        # the dispatch: x read once per token, xp written once per kept row,
        # the routing arrays (idx, gate, slot_of) and perm / row_gate; with a
        # direct top-1 output it also zeroes the dropped tokens' output rows
        direct = k == 1 and S == 0
        return T * d * es + R * d * es + T * k * 12 + R * 8 + ((T - R) * d * es if direct else 0)
    if kernel == "gather":
        return 2 * R * d * es + R * 4
    if kernel == "combine":
        return (R + S * T) * d * es + T * d * es + T * k * 4
    return None


def add_memory_rooflines(kernels, w, R, E_active, es, hbm_gbs):
    """GB/s and fraction of the HBM copy peak of the memory-bound kernels
    (router, dispatch, combine), from their algorithmic bytes per launch and
    their event-timed launch durations (launch gaps included)."""
    for name in ("router", "permute", "combine"):
        kn = kernels.get(name)
        nbytes = algorithmic_bytes(name, w, R, E_active, es)
        if kn is None or nbytes is None or not kn["ms_per_launch"]:
            continue
        gbs = nbytes / (kn["ms_per_launch"] / 1000.0) / 1e9
        kn.update({"algorithmic_bytes": nbytes, "gbs": gbs, "frac_of_hbm": gbs / hbm_gbs})
    return kernels


def copy_bandwidth(x_host, out_host, x_dev, out_dev, reps: int = 20):
    """Host<->device copy rates of one step's input and output (pinned, each
    direction alone, then both at once), GB/s: the ceiling of the end-to-end
    number."""
    import torch
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    res = {}
    for name, streams in (("h2d", [s_in]), ("d2h", [s_out]), ("both", [s_in, s_out])):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        for st in streams:
            st.wait_event(e0)
        for _ in range(reps):
            if s_in in streams:
                with torch.cuda.stream(s_in):
                    x_dev.copy_(x_host, non_blocking=True)
            if s_out in streams:
                with torch.cuda.stream(s_out):
                    out_host.copy_(out_dev, non_blocking=True)
        for st in streams:
            torch.cuda.current_stream().wait_stream(st)
        e1.record()
        torch.cuda.synchronize()
        nbytes = reps * x_host.numel() * x_host.element_size() * len(streams)
        res[name] = nbytes / (e0.elapsed_time(e1) / 1000.0) / 1e9
    return res


def run_e2e(args, layer, x, w, world, dev):
    """End to end through the public API: pinned host in, pinned host out,
    every step's input copied in and output copied back inside the timed
    region; consecutive steps overlap on three streams (HostPipeline, the
    library's native pipeline)."""
    import torch
    import torch.distributed as dist
    from mixture_experts_layer_45_b200.layer import HostPipeline
    # at least 50 steps: the pipeline's first input copy and last output
    # copy (no layer beside them) are then a small part of the timed region
    e2e_steps = args.e2e_steps or max(50, min(args.steps, 200))
    nbuf = 4
    x_hosts = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for _ in range(nbuf)]
    for xh in x_hosts:
        xh.copy_(x.cpu())
    out_hosts = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for _ in range(nbuf)]
    pipe = HostPipeline(layer, w.T)
    xs = [x_hosts[i % nbuf] for i in range(e2e_steps)]
    outs = [out_hosts[i % nbuf] for i in range(e2e_steps)]
    pipe.run(xs[:20], outs[:20])                              # warm-up (the first runs copy slower)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e2e_ms = reduce_max_ms(pipe.run(xs, outs), dev)
    if world > 1:
        dist.barrier()
    e2e_value = whole_job_tokens_per_s(world, e2e_steps, w.T, e2e_ms)
    io_bytes = x.numel() * x.element_size()
    pcie = copy_bandwidth(x_hosts[0], out_hosts[0], pipe.x_dev[0], pipe.out_dev[0])
    # the device result of the last step equals the device-only forward
    ref_out = layer.forward(x)
    torch.cuda.synchronize()
    if not torch.equal(outs[-1].to(dev).view(torch.int16) if x.dtype == torch.bfloat16 else outs[-1].to(dev),
                       ref_out.view(torch.int16) if x.dtype == torch.bfloat16 else ref_out):
        raise RuntimeError("end-to-end output differs from the device forward")
    return {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": io_bytes,
            "d2h_bytes_per_step": io_bytes, "steps": e2e_steps,
            "mode": "pinned host buffers; H2D, layer (a CUDA graph per lane) and D2H of consecutive steps "
                    "overlap on three streams, three lanes; native host loop (moe_pipeline_run)",
            "copy_gbs": pcie}


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"bench: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA GPU")
    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))

    from mixture_experts_layer_45_b200 import _lib
    from mixture_experts_layer_45_b200 import build as build_mod
    from mixture_experts_layer_45_b200.layer import MoELayer, MoEParams, dtype_code, read_stats, to_device
    from mixture_experts_layer_45_b200 import workloads as wl

    if rank == 0:
        build_mod.build()
    if world > 1:
        dist.barrier()
    _lib.load()

    w = get_workload(args)
    dt = dtype_code(w.dtype)
    es = 2 if w.dtype == "bf16" else 4
    inp = wl.draw_inputs(w)
    dev = torch.device("cuda", local_rank)
    params = MoEParams.from_arrays(inp, dt, dev)
    cap = _lib.moe_capacity(w.T, w.k, w.E, w.cf)
    layer = MoELayer(params, w.k, cap, reroute=args.reroute)
    x = to_device(inp["x"], dt, dev)
    out = torch.empty_like(x)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    # warm-up (W >= 3 enforced)
    warm = max(3, args.warmup)
    for _ in range(warm):
        layer.forward(x, out=out, stats=True)
    if _lib.moe_get_error() != 0:
        raise RuntimeError("device error during warm-up")
    st = read_stats(layer.stats_buf)
    R = int(st["rows_kept"])

    # experts with at least one grouped row (their weights are read), from
    # the dispatch's offsets after the warm-up forward
    offs = layer.workspace_view(w.T, "offsets", torch.int32, w.E + 1).cpu().numpy()
    E_active = int((offs[1:] > offs[:-1]).sum())

    # the grouped FFN's own record of the SM clock it runs at (one load and
    # four stores per CTA; read after the timed region: the last step's launches)
    _lib.moe_ffn_clock_enable(True)
    sampler = ClockSampler(local_rank).start() if rank == 0 else None
    time.sleep(0.05)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    # ---- the timed region: K steps, device-timed per step, nothing else in the stream
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    n0 = _lib.moe_launch_count()
    for i in range(args.steps):
        flush.zero_()
        starts[i].record(stream)
        layer.forward(x, out=out, stats=True)
        ends[i].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    launches = _lib.moe_launch_count() - n0
    if sampler:
        sampler.stop()
    ffn_clock = _lib.moe_ffn_clock_read()
    _lib.moe_ffn_clock_enable(False)
    err = _lib.moe_get_error()
    if err != 0:
        raise RuntimeError(f"device error in the timed region: {_lib.status_string(err)}")
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = reduce_max_ms(sum(step_ms), dev)
    value = whole_job_tokens_per_s(world, args.steps, w.T, total_ms)

    # ---- per-kernel durations: a second pass of the same K steps with CUDA
    # events recorded around every launch (they serialise the stream, so this
    # pass is not the one timed above)
    _lib.moe_timing_enable(True)
    _lib.moe_timing_read()
    for i in range(args.steps):
        flush.zero_()
        layer.forward(x, out=out, stats=True)
    torch.cuda.synchronize()
    kt = _lib.moe_timing_read()
    _lib.moe_timing_enable(False)

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, layer, x, w, world, dev)

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return 0

    peaks, peak_src = load_peaks()
    kernels = {}
    tot_k = sum(ms for ms, n in kt.values() if n)
    for name, (ms, n) in kt.items():
        if n:
            kernels[name] = {"launches": n, "ms_per_launch": ms / n, "share": ms / tot_k if tot_k else None}
    add_memory_rooflines(kernels, w, R, E_active, es, peaks["hbm_gbs"])
    modelled = [kn for kn in kernels if algorithmic_bytes(kn, w, R, E_active, es) is not None]
    dom = max(modelled, key=lambda k: kernels[k]["ms_per_launch"] * kernels[k]["launches"])
    ffn_ms = sum(kernels[k]["ms_per_launch"] for k in ("ffn1", "ffn2") if k in kernels)
    ffn_rows = R + w.shared * w.T                 # routed rows kept + shared-expert rows
    ffn_flops = 4.0 * ffn_rows * w.d * w.ff
    ffn_tflops = ffn_flops / (ffn_ms / 1000.0) / 1e12 if ffn_ms else None
    dom_bytes = algorithmic_bytes(dom, w, R, E_active, es)
    dom_s = kernels[dom]["ms_per_launch"] / 1000.0
    # The tensor peak: the burst figure (a GEMM timed alone, before the power
    # cap acts) unless the clocks record shows the power cap during the timed
    # region or the region is seconds long; then the sustained figure, which
    # was itself measured under the cap.
    clocks = sampler.summary() if sampler else None
    capped = bool(clocks and "sw_power_cap" in (clocks.get("reasons") or []))
    sustained = capped or total_ms >= 2000
    tensor_peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    flops_dom = 2.0 * ffn_rows * w.d * w.ff
    ridge = tensor_peak * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if dom in ("ffn1", "ffn2") and w.dtype == "bf16" and flops_dom / max(dom_bytes, 1) > ridge:
        achieved = flops_dom / dom_s / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tensor_peak, "unit": "TFLOP/s",
                "frac": achieved / tensor_peak,
                "peak_kind": ("sustained (sw_power_cap during the timed region)" if capped else
                              "sustained (timed region >= 2 s)" if sustained else "burst"),
                "frac_of_burst": achieved / peaks["bf16_tflops"],
                "algorithmic_flops_per_launch": flops_dom}
    else:
        achieved = dom_bytes / dom_s / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"]}
    roof.update({"kernel": dom, "peak_source": peak_src, "algorithmic_bytes_per_launch": dom_bytes,
                 "traffic": committed_traffic(dom, workload_tag(w))})
    # the FFN launches at the clock they ran at: tcgen05 kind::f16 retires
    # TC_FLOP_PER_SM_CYCLE dense bf16 flop per SM per cycle
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    ffn_clock_rec = {}
    for k in ("ffn1", "ffn2"):
        mhz, span_us = ffn_clock[k]
        if mhz > 0 and span_us > 0:
            rec = {"sm_mhz": mhz, "span_us": span_us}
            if w.dtype == "bf16":
                rec["tensor_frac_at_clock"] = flops_dom / (sms * TC_FLOP_PER_SM_CYCLE * mhz * 1e6 * span_us * 1e-6)
            ffn_clock_rec[k] = rec
    if dom in ffn_clock_rec:
        roof["sm_mhz_in_kernel"] = ffn_clock_rec[dom]["sm_mhz"]
        if "tensor_frac_at_clock" in ffn_clock_rec[dom]:
            roof["tensor_frac_at_clock"] = ffn_clock_rec[dom]["tensor_frac_at_clock"]

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": warm, "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded numpy draws of the workload's distributions; random-init weights)",
        "config": {"workload": workload_label(w, args.reroute), "T": w.T, "d": w.d, "ff": w.ff, "E": w.E, "k": w.k,
                   "shared_experts": w.shared, "reroute_rounds": args.reroute, "capacity": cap, "rows_kept": R,
                   "l2": "flushed before every step (256 MiB write), outside the step timing",
                   "kernel_timing": "second pass of the same steps with CUDA events around each launch",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": roof,
        "ffn": {"tflops": ffn_tflops, "frac_of_bf16_peak": (ffn_tflops / tensor_peak) if ffn_tflops else None,
                "frac_of_burst": (ffn_tflops / peaks["bf16_tflops"]) if ffn_tflops else None,
                "flops_per_step": ffn_flops, "ms_per_step": ffn_ms},
        "kernels": kernels,
        "ffn_clock": dict(ffn_clock_rec, note="SM cycles / ns inside the last timed step's fc1 and fc2 launches "
                          "(median over CTAs); tensor_frac_at_clock = FLOPs / (SMs x 8192 x cycles)"),
        "e2e": e2e,
        "clocks": clocks,
        "gpu_launches": launches,
        "stats": {k: st[k] for k in ("aux_loss", "imbalance", "drop_rate", "rerouted")},
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds, drawn=inp)
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())

#!/usr/bin/env python
"""Throughput of the sparse MoE feed-forward layer on B200: tokens/s of whole layer calls.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl ours|reference]

The default workload is the largest one, the 8x22B-shape prefill layer
(T=16384, d=6144, ffn=16384, E=8, k=2, bf16); --config 2 is the Mixtral-shape
decode layer (T=16), --config 3 / 4 the Mixtral-shape prefill and skewed ones.

A step is one call of the whole layer (route, dispatch, gather, expert GEMMs,
combine) over one batch of T tokens of the chosen workload, with inputs and
weights already resident in HBM.  The timed region is K steps bracketed by a
barrier and a device synchronise; times come from CUDA events on the stream
the kernels run on, max over ranks.  With N > 1 (torchrun, one process per
GPU) every rank runs an independent replica of the layer on its own batch:
tokens are independent and the layer needs no exchange, so there is no
collective on the data path ("replicas", weak scaling).

One JSON line is printed by rank 0.  Besides the base keys it carries:
  stages_ms     mean device time of each stage (events recorded between launches)
  roofline      the dominant kernel: algorithmic bytes or FLOPs per launch over its
                measured mean duration, against MEASURED_PEAKS.json
  layer_roofline  the whole layer against max(FLOPs / tensor peak, bytes / HBM)
  e2e           the same metric through moe_forward_host: x copied from pinned host
                memory and out copied back inside every timed step (wall clock)
  cpu_baseline  the fp64 CPU oracle on the host cores, on a bounded token sample
  clocks        NVML samples taken during the timed region
--impl reference times the fp64 CPU oracle (there is no other implementation
of this layer to run) on the same workload and prints the same line.
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
from datetime import timedelta

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import moe_inputs  # noqa: E402

METRIC = "MoE-layer tokens/sec at 1 B200; achieved % of roofline (tensor TFLOPS or HBM GB/s)"
BLOCK_METRIC = ("MoE sub-layer (RMSNorm + MoE + residual, load-balance statistics) tokens/sec at 1 B200; "
                "achieved % of roofline")
BLOCK_ALPHA = 0.01
TRAIN_METRIC = "MoE-layer training step (forward + backward) tokens/sec at 1 B200; achieved % of roofline"
BLOCK_TRAIN_METRIC = ("MoE sub-layer (RMSNorm + MoE + residual) training step (forward + backward) tokens/sec "
                      "at 1 B200; achieved % of roofline")
L2_BYTES = 126 * 1000 * 1000
# the largest workload: the 8x22B-shape prefill layer (T=16384, d=6144, ffn=16384, E=8, k=2)
DEFAULT_CONFIG = 5
# timed steps when --steps is not given: about half a second of layer calls per workload
DEFAULT_STEPS = {1: 200, 2: 200, 3: 60, 4: 40, 5: 30}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None, help="timed steps (default: by workload, ~0.5 s)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=DEFAULT_CONFIG, choices=sorted(moe_inputs.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target length of the CPU-oracle sample")
    ap.add_argument("--ref-seconds", type=float, default=150.0,
                    help="target length of the whole --impl reference run (warm-up + timed steps)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--block", action="store_true",
                    help="time the block form out = h + MoE(RMSNorm(h)) with load-balance statistics")
    ap.add_argument("--shape", default=None,
                    help="T,d,ffn: run the workload's recipe (E, k, dtype, seed, routing) at other sizes, "
                         "for profiler captures small enough to stay within a few GB")
    ap.add_argument("--train", action="store_true",
                    help="time a training step: forward (grouped-GEMM path) + backward with all gradients")
    ap.add_argument("--bf16-wgrad", action="store_true",
                    help="with --train: weight gradients rounded to bf16 in the GEMM epilogue (fp32 otherwise)")
    ap.add_argument("--ep", action="store_true",
                    help="expert parallelism: each of the N ranks holds E/N experts and its own batch; route, "
                         "dispatch, NCCL all-to-all of the rows, this rank's experts, all-to-all back, combine")
    ap.add_argument("--seed", type=int, default=None,
                    help="the workload's recipe with another seed (inputs, weights and routing change with it)")
    ap.add_argument("--stage-every", type=int, default=8,
                    help="record per-stage events on every n-th timed step (events between launches "
                         "break the overlap of dependent launches, so most steps run without them)")
    args = ap.parse_args()
    if args.ep and (args.train or args.block or args.impl == "reference"):
        ap.error("--ep times the plain layer's forward on our kernels")
    if args.steps is None:
        args.steps = 8 if args.train else DEFAULT_STEPS[args.config]
    return args


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            doc = json.load(f)
        return {k: float(doc[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks

REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
           0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting", 0x10: "sync_boost",
           0x1: "gpu_idle"}


class ClockSampler:
    """NVML samples of SM clock, throttle reasons and power every 10 ms while running."""

    def __init__(self, device_index):
        self.samples = []
        self._stop = threading.Event()
        self._thread = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            handle = None
            try:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                handle = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
            except Exception:
                handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.h = handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report no clocks rather than guess
            self.err = str(e)

    def _sample(self):
        nv = self.nv
        sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
        try:
            reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            reasons = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        power = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
        self.samples.append((sm, reasons, power))

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(0.01)

    def start(self):
        if self.ok:
            self._sample()
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if not self.ok:
            return None
        self._sample()
        self._stop.set()
        self._thread.join()
        sms = [s[0] for s in self.samples]
        mask = 0
        for s in self.samples:
            mask |= int(s[1])
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": self.max_mhz,
                "reasons": [n for b, n in sorted(REASONS.items()) if mask & b and n != "gpu_idle"],
                "samples": len(sms), "power_w_max": round(max(s[2] for s in self.samples), 1)}


class nvtx_range:
    """An NVTX range around a harness phase (warm-up, timed steps, e2e); the library adds its own
    ranges per layer stage.  A no-op without a profiler attached."""

    def __init__(self, name):
        self.name = name

    def __enter__(self):
        torch.cuda.nvtx.range_push(self.name)

    def __exit__(self, *exc):
        torch.cuda.nvtx.range_pop()
        return False


# ------------------------------------------------------------------ work accounting


def accounting(inp, counts, block=False):
    """Algorithmic FLOPs and bytes of the layer and of each expert GEMM (padding rows excluded).

    The block form adds the norm (square, sum, two products per element), the
    residual add and the gain vector; h is read once and out written once, as x is.
    """
    T, d, F, E, k = inp.T, inp.d, inp.F, inp.E, inp.k
    es = 2 if inp.dtype == "bf16" else 4
    touched = int((np.asarray(counts) > 0).sum())
    kT = k * T
    extra_flops = 5.0 * T * d if block else 0.0
    extra_bytes = d * es if block else 0.0
    return {
        "touched": touched,
        "layer_flops": 2.0 * T * d * E + 6.0 * kT * d * F + extra_flops,
        "layer_bytes": touched * 3.0 * d * F * es + 2.0 * T * d * es + E * d * es + extra_bytes,
        "expert1_flops": 4.0 * kT * d * F,
        "expert1_bytes": touched * 2.0 * F * d * es + kT * d * es + kT * F * es,
        "expert2_flops": 2.0 * kT * d * F,
        "expert2_bytes": touched * 1.0 * d * F * es + kT * F * es + kT * d * 4.0,
    }


def source_sha(files):
    h = hashlib.sha1()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:12]


def recorded_traffic(kernel, workload):
    """dram read+write bytes per launch from a committed ncu capture, if the kernel source is unchanged since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        doc = json.load(f)
    ent = doc.get(f"{kernel}@{workload}")
    if not ent:
        return None
    if ent.get("source_sha") != source_sha(ent.get("sources", [])):
        return None
    return ent.get("bytes_per_launch")


# ------------------------------------------------------------------ CPU oracle


def oracle_fn(inp, block):
    """The oracle call the CPU legs time: fn(tokens, nthreads) for the layer or the block form."""
    import oracle
    if block:
        return lambda toks, nt: oracle.block(inp.x, inp.gamma, moe_inputs.BLOCK_EPS, inp.Wg, inp.W1, inp.W3, inp.W2,
                                             k=inp.k, dtype=inp.dtype, tokens=toks, nthreads=nt)
    return lambda toks, nt: oracle.moe(*inp.arrays(), k=inp.k, dtype=inp.dtype, tokens=toks, nthreads=nt)


def oracle_train_run(inp, dout, target_s, block=False):
    """Time the oracle's forward + backward (all gradients) on an evenly spaced token sample of about
    target_s seconds (the oracle's backward runs on one thread); returns (tokens/s, sample text, seconds).
    block: the block form's backward (RMSNorm and residual around the layer, dh and dgamma included)."""
    import oracle

    def run(toks):
        x, d_s = np.ascontiguousarray(inp.x[toks]), np.ascontiguousarray(dout[toks])
        if block:
            return oracle.block_backward(x, inp.gamma, moe_inputs.BLOCK_EPS, inp.Wg, inp.W1, inp.W3, inp.W2, d_s,
                                         inp.k, inp.dtype, alpha=BLOCK_ALPHA)
        return oracle.backward(x, inp.Wg, inp.W1, inp.W3, inp.W2, d_s, inp.k, inp.dtype, alpha=BLOCK_ALPHA)

    t0 = time.perf_counter()
    run([0])
    per_tok = max(time.perf_counter() - t0, 1e-5)
    n = int(max(1, min(inp.T, round(target_s / per_tok))))
    toks = np.unique(np.linspace(0, inp.T - 1, n).astype(np.int64))
    t0 = time.perf_counter()
    run(toks)
    dt = time.perf_counter() - t0
    what = "dh, dgamma, dWg, dW1, dW3, dW2" if block else "dx, dWg, dW1, dW3, dW2"
    sample = (f"{len(toks)} of {inp.T} tokens (evenly spaced): forward and every gradient ({what}, "
              f"load-balance loss included) of those tokens in fp64, one thread")
    return len(toks) / dt, sample, dt


def make_workload(cfg, block, shape=None, seed=None):
    if shape or seed is not None:
        c = moe_inputs.WORKLOADS[cfg]
        T, d, F = (int(v) for v in shape.split(",")) if shape else (c["T"], c["d"], c["F"])
        inp = moe_inputs.make_inputs(T, d, F, c["E"], c["k"], c["dtype"], c["seed"] if seed is None else seed,
                                     c["skew"])
    else:
        inp = moe_inputs.make_config(cfg)
    return moe_inputs.make_block(inp) if block else inp


def workload_name(cfg, shape=None, seed=None):
    c = moe_inputs.WORKLOADS[cfg]
    return c["name"] + (f"@shape={shape}" if shape else "") + (f"@seed={seed}" if seed is not None else "")


def cpu_oracle_run(inp, target_s, threads, block=False):
    """Time the fp64 oracle on a token sample sized for about target_s seconds; returns (tokens/s, sample text)."""
    run = oracle_fn(inp, block)
    t0 = time.perf_counter()
    run([0], 1)
    per_tok = max(time.perf_counter() - t0, 1e-5)
    n = int(max(1, min(inp.T, round(target_s * threads / per_tok))))
    toks = np.unique(np.linspace(0, inp.T - 1, n).astype(np.int32))
    reps = max(1, int(target_s * threads / (per_tok * len(toks)))) if len(toks) == inp.T else 1
    reps = min(reps, 50)
    t0 = time.perf_counter()
    for _ in range(reps):
        run(toks, threads)
    dt = time.perf_counter() - t0
    what = "RMSNorm, routing over all E, k SwiGLU experts, weighted sum, residual" if block else \
        "routing over all E, k SwiGLU experts, weighted sum"
    sample = f"{len(toks)} of {inp.T} tokens (evenly spaced), x{reps}, full {'block' if block else 'layer'} " \
             f"per token ({what}) in fp64"
    return reps * len(toks) / dt, sample, dt


# ------------------------------------------------------------------ reference arm


def run_reference(args, rank):
    if rank != 0:
        return
    c = moe_inputs.WORKLOADS[args.config]
    inp = make_workload(args.config, args.block, args.shape, args.seed)
    if args.train:
        dout = moe_inputs.make_dout(inp.T, inp.d, inp.dtype, seed=inp.seed)
        per_step = max(0.05, min(30.0, args.ref_seconds / max(args.steps + args.warmup, 1)))
        for _ in range(args.warmup):
            oracle_train_run(inp, dout, per_step, args.block)
        total_tok, total_t = 0.0, 0.0
        for _ in range(args.steps):
            v, sample, dt = oracle_train_run(inp, dout, per_step, args.block)
            total_tok += v * dt
            total_t += dt
        value = total_tok / total_t
        line = {
            "impl": "reference", "metric": BLOCK_TRAIN_METRIC if args.block else TRAIN_METRIC, "value": value,
            "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * total_t / max(args.steps, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_name(args.config, args.shape, args.seed) + ("+block" if args.block else "") + "+train",
                       "T": inp.T, "d": inp.d,
                       "ffn": inp.F, "E": inp.E,
                       "k": inp.k, "seed": inp.seed},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line), flush=True)
        return
    run = oracle_fn(inp, args.block)
    threads = len(os.sched_getaffinity(0))
    total_steps = args.steps + args.warmup
    per_step = max(0.05, min(30.0, args.ref_seconds / max(total_steps, 1)))
    t0 = time.perf_counter()
    run([0], 1)
    per_tok = max(time.perf_counter() - t0, 1e-5)
    n = int(max(1, min(inp.T, round(per_step * threads / per_tok))))
    toks = np.unique(np.linspace(0, inp.T - 1, n).astype(np.int32))
    for _ in range(args.warmup):
        run(toks, threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run(toks, threads)
    dt = time.perf_counter() - t0
    value = args.steps * len(toks) / dt
    sample = f"{len(toks)} of {inp.T} tokens per step (evenly spaced), fp64 oracle, {threads} threads"
    line = {
        "impl": "reference", "metric": BLOCK_METRIC if args.block else METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * dt / max(args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(args.config, args.shape, args.seed) + ("+block" if args.block else ""),
                   "T": inp.T, "d": inp.d,
                   "ffn": inp.F, "E": inp.E, "k": inp.k, "seed": inp.seed,
                   "sample_tokens_per_step": int(len(toks))},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm


def reduce_max(value: float, world: int, device=None) -> float:
    """Max of a per-rank number over all ranks (the job's time is its slowest rank's)."""
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(tokens_per_rank_step: int, steps: int, world: int, max_ms: float) -> float:
    """Tokens per second of the whole job: every rank processes its own batch each step."""
    return world * tokens_per_rank_step * steps / (max_ms / 1000.0)


def to_dev(a, dtype, device):
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def run_ours(args, rank, world, local):
    import sparse_mixture_experts_14_b200 as moe
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    c = moe_inputs.WORKLOADS[args.config]
    block = args.block
    inp = make_workload(args.config, block, args.shape, args.seed)
    dev = [to_dev(a, inp.dtype, device) for a in inp.arrays()]
    tdt = dev[0].dtype
    T, d, F, E, k = inp.T, inp.d, inp.F, inp.E, inp.k
    code = moe.MOE_DTYPE_BF16 if inp.dtype == "bf16" else moe.MOE_DTYPE_F32
    wsize = moe.moe_block_workspace_size if block else moe.moe_workspace_size
    ws = torch.empty(wsize(T, d, F, E, k, code), dtype=torch.uint8, device=device)
    out = torch.empty((T, d), dtype=tdt, device=device)
    if block:
        gamma = to_dev(inp.gamma, inp.dtype, device)
        stats = torch.empty(2 * E + 1, dtype=torch.float32, device=device)

    def step(events=None):
        if block:
            return moe.moe_block_forward_ws(dev[0], gamma, moe_inputs.BLOCK_EPS, *dev[1:], k, ws, out,
                                            alpha=BLOCK_ALPHA, stats=stats, events=events)
        return moe.moe_forward_profiled(*dev, k, ws, out, events=events)

    if block:
        # the block routes the normalised rows: take its counts from its own statistics (f = count / T)
        step()
        counts = np.rint(stats[:E].double().cpu().numpy() * T).astype(np.int64)
    else:
        idx, _ = moe.moe_route(dev[0], dev[1], k)
        counts = moe.moe_dispatch(idx, E)[0].cpu().numpy()
    acc = accounting(inp, counts, block)
    flush = acc["layer_bytes"] < 3 * L2_BYTES
    flush_buf = torch.empty(512 * 2 ** 20, dtype=torch.uint8, device=device) if flush else None

    ns = moe.MOE_NUM_STAGES
    K, W = args.steps, args.warmup
    # stage events on every `every`-th step (all steps when L2 is flushed between steps)
    every = 1 if flush else max(1, args.stage_every)
    staged = [i for i in range(K) if i % every == 0]
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(ns + 1)] for _ in range(K)]
    stream = torch.cuda.current_stream()
    for row in events:          # create the CUDA events before the library records them
        for e in row:
            e.record(stream)
    with nvtx_range("bench.warmup"):
        for _ in range(W):
            step()
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    launches = 0
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with nvtx_range("bench.timed"):
        start.record(stream)
        for i in range(K):
            if flush:
                flush_buf.zero_()
                events[i][0].record(stream)
            launches += step(events=events[i] if i % every == 0 else None)
        end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    status = moe.moe_get_device_status()
    if status != moe.MOE_OK:
        raise RuntimeError(f"device fault during the timed region: {moe.moe_status_string(status)}")

    if flush:
        total_ms = sum(events[i][0].elapsed_time(events[i][ns]) for i in range(K))
    else:
        total_ms = start.elapsed_time(end)
    stage_ms = [statistics.mean(events[i][s].elapsed_time(events[i][s + 1]) for i in staged) for s in range(ns)]
    total_ms = reduce_max(total_ms, world, device)
    value = weak_scaling_value(T, K, world, total_ms)

    # e2e: host buffers, copies inside every step
    e2e = None
    if not args.no_e2e and not block:
        x_host = dev[0].cpu().pin_memory() if inp.dtype == "bf16" else None
        if x_host is not None:
            out_host = torch.empty((T, d), dtype=tdt, pin_memory=True)
            for _ in range(max(1, min(W, 3))):
                moe.moe_forward_host(x_host, *dev[1:], k, out_host)
            if world > 1:
                torch.distributed.barrier()
            with nvtx_range("bench.e2e"):
                t0 = time.perf_counter()
                for _ in range(K):
                    moe.moe_forward_host(x_host, *dev[1:], k, out_host)
                wall = time.perf_counter() - t0
            wall = reduce_max(wall, world, device)
            e2e = {"value": weak_scaling_value(T, K, world, wall * 1000.0), "unit": "tokens/s",
                   "h2d_bytes_per_step": T * d * 2, "d2h_bytes_per_step": T * d * 2,
                   "timing": "host wall clock around moe_forward_host (synchronises every step)"}

    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    long_run = total_ms > 1000.0
    tflops_peak = peaks["bf16_tflops_sustained"] if long_run else peaks["bf16_tflops"]
    hbm = peaks["hbm_gbs"]
    stages = dict(zip(moe.STAGE_NAMES, stage_ms))

    layer_t_tensor = acc["layer_flops"] / (tflops_peak * 1e12)
    layer_t_hbm = acc["layer_bytes"] / (hbm * 1e9)
    layer_bound = "tensor" if layer_t_tensor >= layer_t_hbm else "hbm"
    roof_tps = T / max(layer_t_tensor, layer_t_hbm)
    layer_roof = {"bound": layer_bound, "roofline_tokens_per_s": roof_tps, "frac": (value / world) / roof_tps,
                  "flops": acc["layer_flops"], "bytes": acc["layer_bytes"], "touched_experts": acc["touched"]}
    if layer_bound == "tensor":
        # the same fraction against the other dense bf16 denominators: the measured burst and
        # sustained (power-capped) rates, and the 2.25 PFLOP/s datasheet figure
        achieved = acc["layer_flops"] * (value / world) / T / 1e12
        layer_roof["frac_vs"] = {"burst": achieved / peaks["bf16_tflops"],
                                 "sustained": achieved / peaks["bf16_tflops_sustained"],
                                 "datasheet": achieved / 2250.0}

    dom = max(("expert1", "expert2"), key=lambda s: stages[s])
    fl, by = acc[f"{dom}_flops"], acc[f"{dom}_bytes"]
    sec = stages[dom] / 1000.0
    if inp.dtype == "bf16" and fl / (tflops_peak * 1e12) >= by / (hbm * 1e9):
        roof = {"bound": "tensor", "achieved": fl / sec / 1e12, "peak": tflops_peak, "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": by / sec / 1e9, "peak": hbm, "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    if inp.dtype != "bf16":
        kname = {"expert1": "simt_gemm_kernel<true>", "expert2": "simt_gemm_kernel<false>"}[dom]
    elif T <= moe.moe_decode_max_tokens():
        kname = {"expert1": "decode_kernel<true>", "expert2": "decode_kernel<false>"}[dom]
    else:
        # the forward GEMMs run on 256 x 512 tiles when their reduction is 5120 or longer
        kname = {"expert1": "tc_gemm_kernel<kFwd1W>" if d >= 5120 else "tc_gemm_kernel<kFwd1>",
                 "expert2": "tc_gemm_kernel<kFwd2W>" if F >= 5120 else "tc_gemm_kernel<kFwd2>"}[dom]
    roof["traffic"] = recorded_traffic(kname, workload_name(args.config, args.shape, args.seed))
    roof["kernel"] = kname
    roof["per_launch"] = {"flops": fl, "bytes": by, "ms": stages[dom]}
    roof["peak_source"] = f"{peak_src} ({'sustained' if long_run and roof['unit'] == 'TFLOP/s' else 'burst'})"

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        threads = len(os.sched_getaffinity(0))
        v, sample, _ = cpu_oracle_run(inp, args.cpu_seconds, threads, block)
        cpu = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample}

    line = {
        "metric": BLOCK_METRIC if block else METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": W,
        "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": inp.dtype, "data": "synthetic",
        "config": {"workload": workload_name(args.config, args.shape, args.seed) + ("+block" if block else ""), "T": T, "d": d,
                   "ffn": F, "E": E, "k": k,
                   "seed": inp.seed,
                   "routing": "zipf1.2-skewed" if c["skew"] else "near-uniform",
                   "l2": "L2 flushed between steps" if flush else "touched weights larger than L2 (no flush)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "roofline": roof,
        "layer_roofline": layer_roof,
        "stages_ms": stages,
        "stage_events": f"recorded on {len(staged)} of {K} timed steps (every {every})",
        "expert_counts": [int(v) for v in counts],
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def run_train(args, rank, world, local):
    """One step = moe_forward_profiled (training path) + moe_backward_ws with the load-balance loss
    (alpha = 0.01) over one batch, inputs resident.  With --block: the block form, moe_block_forward_ws
    (training path, statistics on) + moe_block_backward_ws (dh, dgamma and the layer's gradients)."""
    import sparse_mixture_experts_14_b200 as moe
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    c = moe_inputs.WORKLOADS[args.config]
    block = args.block
    inp = make_workload(args.config, block, args.shape, args.seed)
    dev = [to_dev(a, inp.dtype, device) for a in inp.arrays()]
    dout_np = moe_inputs.make_dout(inp.T, inp.d, inp.dtype, seed=inp.seed)
    dout = to_dev(dout_np, inp.dtype, device)
    T, d, F, E, k = inp.T, inp.d, inp.F, inp.E, inp.k
    code = moe.MOE_DTYPE_BF16 if inp.dtype == "bf16" else moe.MOE_DTYPE_F32
    if block:
        gamma = to_dev(inp.gamma, inp.dtype, device)
        stats = torch.empty(2 * E + 1, dtype=torch.float32, device=device)
        fws = torch.empty(moe.moe_block_train_workspace_size(T, d, F, E, k, code), dtype=torch.uint8, device=device)
        bws = torch.empty(moe.moe_block_backward_workspace_size(T, d, F, E, k, code), dtype=torch.uint8,
                          device=device)
    else:
        fws = torch.empty(moe.moe_train_workspace_size(T, d, F, E, k, code), dtype=torch.uint8, device=device)
        bws = torch.empty(moe.moe_backward_workspace_size(T, d, F, E, k, code), dtype=torch.uint8, device=device)
    out = torch.empty((T, d), dtype=dev[0].dtype, device=device)
    f32 = torch.float32
    wd = torch.bfloat16 if (args.bf16_wgrad and inp.dtype == "bf16") else f32
    grads = dict(dx=torch.empty((T, d), dtype=dev[0].dtype, device=device),
                 dWg=torch.empty((E, d), dtype=f32, device=device), dW1=torch.empty((E, F, d), dtype=wd, device=device),
                 dW3=torch.empty((E, F, d), dtype=wd, device=device),
                 dW2=torch.empty((E, d, F), dtype=wd, device=device))
    if block:
        grads["dh"] = grads.pop("dx")
        grads["dgamma"] = torch.empty(d, dtype=f32, device=device)
        moe.moe_block_forward_ws(dev[0], gamma, moe_inputs.BLOCK_EPS, *dev[1:], k, fws, out, alpha=BLOCK_ALPHA,
                                 stats=stats, path=moe.MOE_PATH_TRAIN)
        counts = np.rint(stats[:E].double().cpu().numpy() * T).astype(np.int64)
    else:
        idx, _ = moe.moe_route(dev[0], dev[1], k)
        counts = moe.moe_dispatch(idx, E)[0].cpu().numpy()
    acc = accounting(inp, counts, block)
    kT = k * T
    # executed FLOPs of each backward GEMM stage (bf16: the SwiGLU backward is fused into dgrad_h and
    # reads GEMM1's kept pre-activations; fp32 recomputes GEMM1 in the swiglu_bwd stage)
    bwd_flops = {"dgrad_h": 2.0 * kT * d * F, "dgrad_x": 4.0 * kT * d * F, "wgrad2": 2.0 * kT * d * F,
                 "wgrad13": 4.0 * kT * d * F}
    if inp.dtype != "bf16":
        bwd_flops["swiglu_bwd"] = 4.0 * kT * d * F
    # algorithmic work of a training step: the forward, then 12 kT d F of expert gradients and
    # 4 T d E for the router's two gradients
    step_flops = acc["layer_flops"] + 12.0 * kT * d * F + 4.0 * T * d * E

    ns, nb = moe.MOE_NUM_STAGES, moe.MOE_BWD_NUM_STAGES
    K, W = args.steps, args.warmup
    every = max(1, args.stage_every)
    staged = [i for i in range(K) if i % every == 0]
    fev = [[torch.cuda.Event(enable_timing=True) for _ in range(ns + 1)] for _ in range(K)]
    bev = [[torch.cuda.Event(enable_timing=True) for _ in range(nb + 1)] for _ in range(K)]
    stream = torch.cuda.current_stream()
    for row in fev + bev:
        for e in row:
            e.record(stream)

    def step(i=None):
        on = i is not None and i % every == 0
        if block:
            n = moe.moe_block_forward_ws(dev[0], gamma, moe_inputs.BLOCK_EPS, *dev[1:], k, fws, out,
                                         alpha=BLOCK_ALPHA, stats=stats, path=moe.MOE_PATH_TRAIN,
                                         events=fev[i] if on else None)
            _, m = moe.moe_block_backward_ws(dev[0], gamma, *dev[1:], dout, k, fws, workspace=bws, grads=grads,
                                             alpha=BLOCK_ALPHA, events=bev[i] if on else None)
            return n + m
        n = moe.moe_forward_profiled(*dev, k, fws, out, events=fev[i] if on else None, path=moe.MOE_PATH_TRAIN)
        _, m = moe.moe_backward_ws(*dev, dout, k, fws, workspace=bws, grads=grads, alpha=BLOCK_ALPHA,
                                   events=bev[i] if on else None)
        return n + m

    with nvtx_range("bench.warmup"):
        for _ in range(W):
            step()
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    launches = 0
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with nvtx_range("bench.timed"):
        start.record(stream)
        for i in range(K):
            launches += step(i)
        end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    status = moe.moe_get_device_status()
    if status != moe.MOE_OK:
        raise RuntimeError(f"device fault during the timed region: {moe.moe_status_string(status)}")
    total_ms = reduce_max(start.elapsed_time(end), world, device)
    value = weak_scaling_value(T, K, world, total_ms)
    if rank != 0:
        return
    fst = {n: statistics.mean(fev[i][s].elapsed_time(fev[i][s + 1]) for i in staged)
           for s, n in enumerate(moe.STAGE_NAMES)}
    bst = {n: statistics.mean(bev[i][s].elapsed_time(bev[i][s + 1]) for i in staged)
           for s, n in enumerate(moe.BWD_STAGE_NAMES)}
    peaks, peak_src = load_peaks()
    long_run = total_ms > 1000.0
    tflops_peak = peaks["bf16_tflops_sustained"] if long_run else peaks["bf16_tflops"]
    dom = max(bwd_flops, key=lambda n: bst[n])
    sec = bst[dom] / 1000.0
    roof = {"bound": "tensor", "achieved": bwd_flops[dom] / sec / 1e12, "peak": tflops_peak, "unit": "TFLOP/s",
            "traffic": recorded_traffic(f"tc_gemm_kernel ({dom})", workload_name(args.config, args.shape, args.seed)),
            "kernel": f"tc_gemm_kernel ({dom})",
            "per_launch": {"flops": bwd_flops[dom], "ms": bst[dom]},
            "peak_source": f"{peak_src} ({'sustained' if long_run else 'burst'})"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof_tps = T / (step_flops / (tflops_peak * 1e12))
    step_roof = {"bound": "tensor", "roofline_tokens_per_s": roof_tps, "frac": (value / world) / roof_tps,
                 "flops": step_flops}
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        v, sample, _ = oracle_train_run(inp, dout_np, args.cpu_seconds, block)
        cpu = {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample}
    line = {
        "metric": BLOCK_TRAIN_METRIC if block else TRAIN_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": inp.dtype, "data": "synthetic",
        "config": {"workload": workload_name(args.config, args.shape, args.seed) + ("+block" if block else "") + "+train",
                   "T": T, "d": d, "ffn": F, "E": E,
                   "k": k, "seed": inp.seed, "weight_grads": "bf16" if wd == torch.bfloat16 else "fp32",
                   "l2": "touched weights larger than L2 (no flush)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "roofline": roof,
        "step_roofline": step_roof,
        "stages_ms": {"forward": fst, "backward": bst},
        "stage_events": f"recorded on {len(staged)} of {K} timed steps (every {every})",
        "cpu_baseline": cpu,
        "e2e": None,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


EP_METRIC = ("MoE-layer tokens/sec, expert parallel over the job's GPUs (experts split across ranks, "
             "all-to-all dispatch and combine)")


def run_ep(args, rank, world, local):
    """One expert-parallel forward per step (sparse_mixture_experts_14_b200.ep.moe_forward_ep): the
    route, dispatch, expert and combine kernels of the library around torch.distributed's NCCL
    all-to-alls.  Every rank holds the experts expert_range(E, world, rank) and its own batch of
    the workload's T tokens; the first step's output is checked against the single-GPU layer on
    the same tokens, bit for bit.  The plan needs the counts on the host, so each step
    synchronises twice: the timing is device time between events around whole steps."""
    import sparse_mixture_experts_14_b200 as moe
    from sparse_mixture_experts_14_b200.ep import expert_range, moe_forward_ep
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    c = moe_inputs.WORKLOADS[args.config]
    inp = make_workload(args.config, False, args.shape, args.seed)
    if inp.dtype != "bf16":
        raise SystemExit("--ep runs the bf16 workloads")
    x, Wg, W1, W3, W2 = [to_dev(a, inp.dtype, device) for a in inp.arrays()]
    T, d, F, E, k = inp.T, inp.d, inp.F, inp.E, inp.k
    lo, hi = expert_range(E, world, rank)
    W1l, W3l, W2l = W1[lo:hi].contiguous(), W3[lo:hi].contiguous(), W2[lo:hi].contiguous()
    # the single-GPU check needs the full weights; the timed steps touch only this rank's experts
    ref = moe.moe_forward(x, Wg, W1, W3, W2, k)
    got = moe_forward_ep(x, Wg, W1l, W3l, W2l, k)
    torch.cuda.synchronize()
    if not torch.equal(got, ref):
        raise RuntimeError("expert-parallel output differs from the single-GPU layer")
    del ref, got, W1, W3, W2
    torch.cuda.empty_cache()
    K, W = args.steps, args.warmup
    for _ in range(W):
        moe_forward_ep(x, Wg, W1l, W3l, W2l, k)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    stream = torch.cuda.current_stream(device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with nvtx_range("bench.timed"):
        start.record(stream)
        for _ in range(K):
            moe_forward_ep(x, Wg, W1l, W3l, W2l, k)
        end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if moe.moe_get_device_status() != moe.MOE_OK:
        raise RuntimeError("device fault during the timed region")
    total_ms = reduce_max(start.elapsed_time(end), world, device)
    value = weak_scaling_value(T, K, world, total_ms)
    if rank != 0:
        return
    line = {
        "metric": EP_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": inp.dtype, "data": "synthetic",
        "config": {"workload": workload_name(args.config, args.shape, args.seed) + "+ep", "T": T, "d": d, "ffn": F, "E": E,
                   "k": k, "seed": inp.seed, "experts_per_rank": hi - lo,
                   "parallelism": f"expert parallel x{world}" if world > 1 else "expert parallel x1 (one-rank group)",
                   "check": "first step equal to the single-GPU layer bit for bit"},
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    dist = world > 1 or args.ep
    if dist:
        torch.cuda.set_device(local)
        if world == 1:
            # a one-rank NCCL group for the expert-parallel data plane on one GPU
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("MASTER_PORT", str(29500 + os.getpid() % 1000))
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        torch.distributed.init_process_group("nccl", timeout=timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    try:
        if args.ep:
            run_ep(args, rank, world, local)
        else:
            (run_train if args.train else run_ours)(args, rank, world, local)
    finally:
        if dist:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

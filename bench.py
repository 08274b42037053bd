#!/usr/bin/env python
"""Throughput of the TokenMixer-Large forward on B200 (one JSON line on rank 0).

A step is one tm_stack_forward over one batch of a workload with synthetic inputs and random
weights already resident in HBM.  The default workload is the large Sparse-Pertoken MoE stack
(B=16384 samples, T=48 tokens, D=768, H=48 heads, L=4 blocks with the inter-residual every 2,
per token E=16 SwiGLU experts of hidden 512, top-4, alpha=4, a shared expert of hidden 768,
~8e9 expert parameters resident): the largest workload that fits one GPU.  Each timed step is
bracketed by CUDA events on the launching stream; a 256 MB write between steps flushes the
126 MB L2 (the workload's inputs and weights are far larger than the L2 as well).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]
                  [--batch B] [--layers L] [--e2e-chunks C] [--fp8 | --backward]

Without --steps the step count is chosen from the warm-up steps' time so that the timed region
lasts about two seconds.  N > 1 (under torchrun): every rank runs its own batch (weak scaling,
no data-path collective); the step time is the max over ranks.  --impl reference times the CPU
float64 oracle on the host cores (rank 0 only) on a bounded sample of the workload.  The
end-to-end leg runs a stream of steps through the public API, each copying its batch from pinned
host memory and its result back, the copies overlapping the neighbouring steps' compute
(--e2e-mode step: each step alone, its copies overlapping its own compute in C sample chunks); the
result is checked bit for bit against the full-batch device run.  --batch and --layers run a smaller case of the same kernels (profiler
captures).  --fp8 and --backward print their own lines (the FP8 serving path, the dense block
backward).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import tm_synth as S  # noqa: E402

METRIC = "samples/sec & TFLOP/s of TokenMixer-Large fwd, % of B200 bf16 TC roofline"
METRIC_BWD = "samples/sec & TFLOP/s of TokenMixer-Large dense block backward, % of B200 bf16 TC roofline"
DEFAULT_WORKLOAD = "large_moe_stack_bf16"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = ["tm_gemm.cuh", "tm_fused.cuh", "tm_fused128.cuh", "tm_device.cuh", "tm_gemm.cu", "tm_kernels.cu", "tm_api.cu"]


def describe(cfg) -> str:
    def ffn(s):
        if s.is_moe:
            return f"MoE E={s.E} k={s.k} Fe={s.hidden_e} Fs={s.hidden_s} alpha={s.alpha:g}"
        return f"SwiGLU F={s.hidden}"
    return (f"{cfg.name}: B={cfg.B} T={cfg.T} D={cfg.D} H={cfg.H} L={cfg.L} gap={cfg.gap} {cfg.dtype}; "
            f"mix {ffn(cfg.mix)}; rev {ffn(cfg.rev)}")


def sublayer_flops_per_sample(cfg, sub) -> float:
    """Algorithmic flops of one sub-layer per sample: only the work the method performs
    (the k chosen experts, the shared expert, the router); Mix/Revert 0, RMSNorm not counted."""
    s, W, banks = cfg.ffn(sub), cfg.width(sub), cfg.banks(sub)
    if s.is_moe:
        return banks * (s.k * 6.0 * W * s.hidden_e + 6.0 * W * s.hidden_s + 2.0 * W * s.E)
    return banks * 6.0 * W * s.hidden


def flops_per_sample(cfg) -> float:
    return cfg.L * (sublayer_flops_per_sample(cfg, 0) + sublayer_flops_per_sample(cfg, 1))


def kernel_flops(cfg, B) -> dict:
    """Algorithmic flops of one step attributed to each kernel family the library launches
    (the dispatch: dense bf16 sub-layers of row width 128/256 run as one fused kernel; other
    dense sub-layers as GEMM1+SwiGLU and GEMM2+residual; MoE as routed and shared GEMMs)."""
    out = {}

    def add(k, v):
        out[k] = out.get(k, 0.0) + v
    for _ in range(cfg.L):
        for sub in (0, 1):
            s, W, banks = cfg.ffn(sub), cfg.width(sub), cfg.banks(sub)
            if s.is_moe:
                add("gemm_swiglu", B * banks * 4.0 * W * (s.k * s.hidden_e + s.hidden_s))
                add("gemm_slot", B * banks * s.k * 2.0 * W * s.hidden_e)
                add("gemm_combine", B * banks * 2.0 * W * s.hidden_s)
                add("router", B * banks * 2.0 * W * s.E)
            elif cfg.dtype == "bf16" and W in (128, 256) and s.hidden % 64 == 0:
                add("fused_swiglu", B * banks * 6.0 * W * s.hidden)
            else:
                add("gemm_swiglu", B * banks * 4.0 * W * s.hidden)
                # bf16 rows readable through a tensor map (row layout, or mixed with 16-column head
                # pieces) take the combine kernel (residual by identity MMAs); others the residual epilogue
                tmap = cfg.dtype == "bf16" and (sub == 1 or (cfg.D // cfg.H) % 16 == 0)
                add("gemm_combine" if tmap else "gemm_resid", B * banks * 2.0 * W * s.hidden)
    return out


def kernel_flops_fp8(cfg, B) -> dict:
    """The FP8 path: dense sub-layers run the fused kernel in its FP8 mode; MoE sub-layers run every
    expert's GEMM1 (routed and shared) as the E4M3 grouped GEMM and the rest as on the bf16 path."""
    out = {}

    def add(k, v):
        out[k] = out.get(k, 0.0) + v
    for _ in range(cfg.L):
        for sub in (0, 1):
            s, W, banks = cfg.ffn(sub), cfg.width(sub), cfg.banks(sub)
            if s.is_moe:
                add("gemm_swiglu_fp8", B * banks * 4.0 * W * (s.k * s.hidden_e + s.hidden_s))
                add("gemm_slot", B * banks * s.k * 2.0 * W * s.hidden_e)
                add("gemm_combine", B * banks * 2.0 * W * s.hidden_s)
                add("router", B * banks * 2.0 * W * s.E)
            else:
                add("fused_swiglu_fp8", B * banks * 6.0 * W * s.hidden)
    return out


def backward_flops_per_sample(cfg) -> float:
    """Algorithmic flops of the dense block backward per sample: per row and bank of each sub-layer
    the derivative's own contractions, dH (2 W F), dWd (2 W F), dWg and dWu (4 W F) and the gradient
    at the normalised row (4 W F), i.e. twice the forward's 6 W F.  The recomputation the step also
    performs (the gate / up projections, 4 W F, and the mixing sub-layer's forward) is not counted."""
    return cfg.L * sum(cfg.banks(sub) * 12.0 * cfg.width(sub) * cfg.ffn(sub).hidden for sub in (0, 1))


def kernel_flops_backward(cfg, B) -> dict:
    """Flops of one backward step per kernel family: every contraction of the two sub-layer
    backward passes (recomputed projections included, 16 W F per row and bank) runs on the grouped
    GEMM's plain store epilogue ("gemm_slot"); the mixing sub-layer's forward (X_rev recomputed)
    takes the forward's dispatch."""
    out = {"gemm_slot": sum(B * cfg.banks(sub) * 16.0 * cfg.width(sub) * cfg.ffn(sub).hidden for sub in (0, 1))}
    W, F, H = cfg.W, cfg.mix.hidden, cfg.H
    if W in (128, 256) and F % 64 == 0:
        out["fused_swiglu"] = B * H * 6.0 * W * F
    else:
        out["gemm_swiglu"] = B * H * 4.0 * W * F
        out["gemm_combine" if (cfg.D // H) % 16 == 0 else "gemm_resid"] = B * H * 2.0 * W * F
    return out


def fp8_effective_peak(bf16_peak: float) -> float:
    """Tensor peak of the FP8 kernel's mix of work: GEMM1 (4 W F flops per row) at the E4M3 rate,
    taken as the measured bf16 peak x 2 (the nominal 4.5 / 2.25 PFLOP/s ratio), GEMM2 (2 W F) at
    the bf16 rate: 6 / (4 / 2P + 2 / P) = 1.5 P."""
    return 6.0 / (4.0 / (2.0 * bf16_peak) + 2.0 / bf16_peak)


def kernel_peak_factor(kernel: str) -> float:
    """The kernel's tensor peak in units of the measured bf16 peak: the fused FP8 sub-layer 1.5
    (fp8_effective_peak), the E4M3 grouped GEMM1 2 (all of its flops at the E4M3 rate), bf16 kernels 1."""
    return {"fused_swiglu_fp8": 1.5, "gemm_swiglu_fp8": 2.0}.get(kernel, 1.0)


def step_peak_factor(cfg, fp8: bool) -> float:
    """The whole step's tensor peak in units of the bf16 peak: its flops over the time they take at
    each kernel's own peak."""
    if not fp8:
        return 1.0
    kf = kernel_flops_fp8(cfg, 1)
    return sum(kf.values()) / sum(v / kernel_peak_factor(k) for k, v in kf.items())


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# The sources each profiled kernel family is compiled from (its own code and the device helpers it
# uses); a DRAM figure in profiles/traffic.json counts only while these are unchanged.
KERNEL_SOURCES_OF = {
    "fused_swiglu": ["tm_fused128.cuh", "tm_fused.cuh", "tm_device.cuh"],
    "gemm_swiglu": ["tm_gemm.cuh", "tm_device.cuh"],
    "gemm_slot": ["tm_gemm.cuh", "tm_device.cuh"],
    "gemm_combine": ["tm_gemm.cuh", "tm_device.cuh"],
    "router": ["tm_gemm.cuh", "tm_device.cuh"],
}


def kernel_hash(kernel: str = None) -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES_OF.get(kernel, KERNEL_SOURCES):
        with open(os.path.join(ROOT, "token_sparse_moe_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on these kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(workload, {}).get(kernel)
    if not e or e.get("kernel_hash") != kernel_hash(kernel):
        return None
    return float(e["dram_bytes_per_launch"])


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.f = None

    def __enter__(self):
        try:
            self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.f is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.f.flush()
        with open(self.f.name) as g:
            rows = [l.strip().split(", ") for l in g if l.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle timing
def oracle_param_bytes(cfg) -> float:
    """float64 bytes of every weight of the workload (what the oracle would hold to run it whole)."""
    n = 0
    for sub in (0, 1):
        s, W, banks = cfg.ffn(sub), cfg.width(sub), cfg.banks(sub)
        per = 3 * W * s.hidden if not s.is_moe else s.E * (W + 3 * W * s.hidden_e) + 3 * W * s.hidden_s
        n += banks * per
    return 8.0 * cfg.L * n


def oracle_probe(cfg, n: int, max_banks: int = 2):
    """The oracle as it stands, on a bounded sample of the workload: a function that runs it once and
    returns the host seconds that the whole stack would take on n samples, plus a description.

    Workloads whose weights fit the host in float64 (up to 4 GB): stack_forward on samples
    0..n-1, weights drawn beforehand.  Larger ones: the oracle's sub-layer (sublayer(): RMSNorm,
    routing, experts) on samples 0..n-1 and the first nb banks of both sub-layers of block 1,
    scaled by banks / nb and by the L blocks (every bank and block has the same shapes and the
    routing is near uniform); the token rows stand in for the reverting sub-layer's input (the
    same shape and distribution as X_revert)."""
    import oracle
    from oracle import tokenmixer as O
    n = min(n, cfg.B)
    X = S.to_f64(S.make_x(cfg, np.arange(n)))
    if oracle_param_bytes(cfg) <= 4e9:
        get = oracle.synth_banks(cfg)
        for l in range(cfg.L):
            for sub in (0, 1):
                for j in range(cfg.banks(sub)):
                    get(l, sub, j)

        def step():
            t0 = time.perf_counter()
            oracle.stack_forward(X, cfg, get)
            return time.perf_counter() - t0
        return step, f"oracle stack_forward on samples 0..{n - 1} of {cfg.name}"
    nb = min(max_banks, cfg.H, cfg.T)
    get = oracle.synth_banks(cfg)
    for sub in (0, 1):
        for j in range(nb):
            get(0, sub, j)
    rows_mix = O.mix(X, cfg.H)[:, :nb]
    rows_rev = X[:, :nb]

    def step():
        t0 = time.perf_counter()
        O.sublayer(rows_mix, lambda j: get(0, 0, j), cfg.mix, cfg.eps)
        t1 = time.perf_counter()
        O.sublayer(rows_rev, lambda j: get(0, 1, j), cfg.rev, cfg.eps)
        t2 = time.perf_counter()
        return cfg.L * ((t1 - t0) * cfg.H / nb + (t2 - t1) * cfg.T / nb)
    return step, (f"oracle sublayer() on samples 0..{n - 1} x banks 0..{nb - 1} of both sub-layers of block 1 "
                  f"of {cfg.name}, scaled to all {cfg.H}+{cfg.T} banks and {cfg.L} blocks")


def oracle_threads() -> int:
    from threadpoolctl import threadpool_info
    return int(max([i.get("num_threads", 1) for i in threadpool_info()] or [1]))


def time_oracle(cfg, budget_s: float, max_samples: int):
    """Oracle samples/s on the host cores over a bounded sample (weights drawn beforehand)."""
    step, desc = oracle_probe(cfg, max_samples)
    n = min(max_samples, cfg.B)
    done, equiv, t0 = 0, 0.0, time.perf_counter()
    while True:
        equiv += step()
        done += n
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return done / equiv, {"cores": oracle_threads(), "samples": done, "seconds": dt, "per_call": n, "desc": desc}


def time_oracle_fp8(cfg, budget_s: float, max_samples: int):
    """The FP8 oracle's samples/s on the host cores (weights quantized beforehand, as served).  MoE
    workloads: the FP8 MoE sub-layer on the first banks of block 1, scaled as oracle_probe scales."""
    import oracle
    from oracle import fp8 as F
    from threadpoolctl import threadpool_info
    if any(cfg.ffn(s).is_moe for s in (0, 1)):
        return time_oracle_fp8_moe(cfg, budget_s, max_samples)
    get = oracle.synth_banks(cfg)
    q = {(l, sub, j): F.quantize_bank(get(l, sub, j)) for l in range(cfg.L) for sub in (0, 1)
         for j in range(cfg.banks(sub))}
    n = min(max_samples, cfg.B)
    X = S.to_f64(S.make_x(cfg, np.arange(n)))
    done, t0 = 0, time.perf_counter()
    while True:
        Y = X
        for l in range(cfg.L):
            Y = F.block_forward_fp8(Y, cfg, lambda sub, j: q[(l, sub, j)])["Y"]
        done += n
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return done / dt, {"cores": int(threads), "samples": done, "seconds": dt, "per_call": n}


def time_oracle_backward(cfg, budget_s: float, max_samples: int):
    """The backward oracle's samples/s on the host cores over a bounded sample (one dense block)."""
    import oracle
    from oracle import backward as BW
    from threadpoolctl import threadpool_info
    get = oracle.synth_banks(cfg)
    for sub in (0, 1):
        for j in range(cfg.banks(sub)):
            get(0, sub, j)
    n = min(max_samples, cfg.B)
    X = S.to_f64(S.make_x(cfg, np.arange(n)))
    dY = S.to_f64(S.make_x(cfg.with_(seed=cfg.seed + 17), np.arange(n)))
    done, t0 = 0, time.perf_counter()
    while True:
        BW.block_backward(X, cfg, 0, get, dY, storage=cfg.dtype)
        done += n
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return done / dt, {"cores": int(threads), "samples": done, "seconds": dt, "per_call": n}


def run_reference(args, cfg, rank):
    if rank != 0:
        return
    steps, warm = args.steps_ref, min(args.warmup, 3)
    n = min(args.ref_samples, cfg.B)
    step, desc = oracle_probe(cfg, n)
    for _ in range(warm):
        step()
    t = [step() for _ in range(steps)]
    sec = sum(t)
    value = n * steps / sec
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "samples/s", "n_gpus": args.gpus,
        "steps": steps, "warmup": warm, "ms_per_step": 1e3 * sec / steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": describe(cfg), "global_batch": n, "parallelism": "host cores",
                   "step": f"{desc}; ms_per_step is the whole stack's time on those {n} samples"},
        "tflops": flops_per_sample(cfg) * value / 1e12,
        "cpu_baseline": {"value": value, "unit": "samples/s", "cores": oracle_threads(), "kind": "oracle",
                         "sample": f"{steps} steps: {desc}"},
        "e2e": {"value": value, "unit": "samples/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ multi-rank bookkeeping
def max_over_ranks(value: float, world: int, device) -> float:
    """The largest of every rank's value (the job is as slow as its slowest rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(samples_per_rank: int, world: int, step_ms: float) -> float:
    """Samples all ranks processed per second: each rank runs its own batch (weak scaling)."""
    return samples_per_rank * world / (step_ms / 1e3)


def time_oracle_fp8_moe(cfg, budget_s: float, max_samples: int, max_banks: int = 2):
    import oracle
    from oracle import fp8 as F
    from oracle import tokenmixer as O
    n = min(max_samples, cfg.B)
    nb = min(max_banks, cfg.H, cfg.T)
    get = oracle.synth_banks(cfg)
    q = {(s, j): F.quantize_moe_bank(get(0, s, j)) for s in (0, 1) for j in range(nb)}
    X = S.to_f64(S.make_x(cfg, np.arange(n)))
    rows = {0: O.mix(X, cfg.H)[:, :nb], 1: X[:, :nb]}
    done, equiv, t0 = 0, 0.0, time.perf_counter()
    while True:
        for s, banks in ((0, cfg.H), (1, cfg.T)):
            t1 = time.perf_counter()
            F.sublayer_moe_fp8(rows[s], lambda j: q[(s, j)], cfg.ffn(s), cfg.eps)
            equiv += cfg.L * (time.perf_counter() - t1) * banks / nb
        done += n
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return done / equiv, {"cores": oracle_threads(), "samples": done, "seconds": dt, "per_call": n,
                          "desc": f"oracle fp8.sublayer_moe_fp8 on samples 0..{n - 1} x banks 0..{nb - 1} of both "
                                  f"sub-layers of block 1, scaled to all {cfg.H}+{cfg.T} banks and {cfg.L} blocks"}


def rank_config(cfg, rank: int):
    """Each rank draws its own input batch (seed offset by the rank); weights are shared."""
    return cfg.with_(seed=cfg.seed + rank)


# ------------------------------------------------------------------ GPU arm
def run_ours(args, cfg, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from token_sparse_moe_b200 import api

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    blocks = api.blocks_from_synth(cfg, dev, workers=min(16, os.cpu_count() or 1))
    sh = api.config_shape(cfg)
    dY = None
    moe = any(cfg.ffn(sub).is_moe for sub in (0, 1))
    if args.backward and (cfg.gap or cfg.dtype != "bf16" or moe):
        raise SystemExit("--backward covers bf16 dense blocks without the inter-residual")
    if args.fp8 and cfg.dtype != "bf16":
        raise SystemExit("--fp8 covers bf16 workloads")
    if args.backward:
        if cfg.L != 1:
            raise SystemExit("--backward times one dense block")
        dY = api.to_device(S.make_x(rank_config(cfg, rank).with_(seed=cfg.seed + rank + 17)), dev)
        run = api.BlockBackwardRunner(blocks[0], sh, dY, dev)
    elif args.fp8 and (moe or cfg.gap):
        run = api.Fp8StackRunner([(api.sublayer8_from_bf16(b.mix), api.sublayer8_from_bf16(b.rev)) for b in blocks],
                                 sh, cfg.gap, dev)
        del blocks
        torch.cuda.empty_cache()
    elif args.fp8:
        run = api.Fp8BlockRunner([api.Block8.from_bf16(b) for b in blocks], sh, dev)
    else:
        run = api.StackRunner(blocks, sh, cfg.gap, dev)
    X = api.to_device(S.make_x(rank_config(cfg, rank)), dev)
    Y = torch.empty_like(X)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    K, W = args.steps, args.warmup

    with torch.cuda.stream(stream):
        t_warm = time.perf_counter()
        for _ in range(W):
            flush.zero_()
            run(X, Y, stream)
        stream.synchronize()
        t_warm = (time.perf_counter() - t_warm) / max(W, 1)
        api.get_device_error(stream)
        if K is None:
            # about two seconds of timed steps (the same count on every rank)
            K = int(min(5000, max(10, round(2.0 / max(t_warm, 1e-5)))))
            if world > 1:
                K = int(max_over_ranks(float(K), world, dev))
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        n0 = api.launch_count()
        api.profile_start()
        with ClockSampler(local_rank) as clk:
            t_wall = time.perf_counter()
            for i in range(K):
                flush.zero_()
                ev[i][0].record(stream)
                run(X, Y, stream)
                ev[i][1].record(stream)
            stream.synchronize()
            t_wall = time.perf_counter() - t_wall
        kern = api.profile_stop()
        launches = api.launch_count() - n0
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        api.get_device_error(stream)
        step_ms = [a.elapsed_time(b) for a, b in ev]

    mean_ms = max_over_ranks(sum(step_ms) / K, world, dev)

    # end to end through the public API: pinned host X -> device -> forward -> pinned host Y
    Ke = min(K, args.e2e_steps)
    Xh = X.cpu().pin_memory()
    Yh = torch.empty_like(Xh).pin_memory()
    Xd = torch.empty_like(X)
    # the backward step's inputs are X and dY (both copied in), its result dX (copied back)
    dYh = dY.cpu().pin_memory() if args.backward else None
    chunks = (api.RAMP_CHUNKS if args.e2e_chunks == "ramp" else int(args.e2e_chunks)) \
        if not args.backward and isinstance(run, (api.StackRunner, api.Fp8StackRunner)) else 1
    if args.backward:
        host = lambda: run.run_host(Xh, Yh, Xd, Y, dYh, stream)
    elif chunks != 1:
        host = lambda: run.run_host(Xh, Yh, Xd, Y, stream, chunks=chunks)
    else:
        host = lambda: run.run_host(Xh, Yh, Xd, Y, stream)
    # the whole batch on the device once more, for the bit-exact check of the end-to-end result
    Yref = torch.empty_like(Y)
    with torch.cuda.stream(stream):
        run(X, Yref, stream)
    stream.synchronize()
    streamed = args.e2e_mode == "stream" and not args.backward and hasattr(run, "run_host_steps")
    if streamed:
        # a stream of Ke steps as a serving loop runs it: every step copies its batch in and its result
        # out, each step's copies overlapping the neighbouring steps' compute (run_host_steps)
        Xb, Yb = [Xd, torch.empty_like(X)], [torch.empty_like(X), torch.empty_like(X)]
        with torch.cuda.stream(stream):
            run.run_host_steps(Xh, Yh, Xb, Yb, 2, stream)
            stream.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            run.run_host_steps(Xh, Yh, Xb, Yb, Ke, stream)
            e1.record(stream)
            stream.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / Ke, world, dev)
    else:
        with torch.cuda.stream(stream):
            for _ in range(3):
                host()
            stream.synchronize()
            eve = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(Ke)]
            for i in range(Ke):
                flush.zero_()
                eve[i][0].record(stream)
                host()
                eve[i][1].record(stream)
            stream.synchronize()
        e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in eve) / Ke, world, dev)
    e2e_exact = bool(torch.equal(Yh, Yref.cpu()))
    io_bytes = X.numel() * X.element_size()
    h2d_bytes = io_bytes * (2 if args.backward else 1)

    if rank != 0:
        return
    pk, pk_src = peaks()
    total_samples = cfg.B * world
    value = job_throughput(cfg.B, world, mean_ms)
    tflops = (backward_flops_per_sample(cfg) if args.backward else flops_per_sample(cfg)) * value / 1e12
    # dominant kernel: largest share of device time in the timed region
    dom = max(kern.items(), key=lambda kv: kv[1]["total_ms"]) if kern else (None, None)
    roof = None
    kf = (kernel_flops_fp8(cfg, cfg.B) if args.fp8 else
          kernel_flops_backward(cfg, cfg.B) if args.backward else kernel_flops(cfg, cfg.B))
    if dom[0] in kf:
        per_launch = kf[dom[0]] / (dom[1]["launches"] / K)
        avg_ms = dom[1]["total_ms"] / dom[1]["launches"]
        ach = per_launch / (avg_ms / 1e3) / 1e12
        tr = traffic_for(dom[0], cfg.name)
        # a step of 10 ms or more keeps the GPU at its power limit for the whole timed region: the
        # sustained figure (a seconds-long cuBLAS loop); shorter steps: the burst figure
        long_step = mean_ms >= 10.0
        key = "bf16_tflops_sustained" if long_step else "bf16_tflops"
        src = (f"measured bf16 {'sustained' if long_step else 'burst'} (MEASURED_PEAKS.json {key})"
               if pk_src == "measured" else f"fallback {'1.40' if long_step else '1.59'} PFLOP/s")
        fac = kernel_peak_factor(dom[0])
        peak = pk[key] * fac
        if fac == 1.5:
            src = ("GEMM1 at 2 x, GEMM2 at 1 x the " + src + ": 1.5 x the bf16 peak for the kernel's "
                   "2:1 split of flops")
        elif fac == 2.0:
            src = "2 x the " + src + " (E4M3 operands: the nominal 4.5 / 2.25 PFLOP/s ratio)"
        roof = {"kernel": dom[0], "bound": "tensor", "achieved": ach, "peak": peak,
                "unit": "TFLOP/s", "frac": ach / peak, "traffic": tr, "peak_source": src,
                "frac_of_burst": ach / (pk["bf16_tflops"] * fac),
                "flops_per_launch": per_launch, "avg_launch_ms": avg_ms}
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        timer = time_oracle_fp8 if args.fp8 else time_oracle_backward if args.backward else time_oracle
        v, info = timer(cfg, args.cpu_seconds, args.cpu_samples)
        cpu = {"value": v, "unit": "samples/s", "cores": info["cores"], "kind": "oracle",
               "sample": (f"{info['desc']}; " if "desc" in info else "") +
                         f"{info['samples']} samples ({info['per_call']} per oracle call) of {cfg.name}, "
                         f"{info['seconds']:.1f} s of host time"}
    line = {
        "metric": METRIC_BWD if args.backward else METRIC, "value": value, "unit": "samples/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": mean_ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3+bf16" if args.fp8 else "bf16",
        "data": "synthetic (seeded normal inputs, random-init weights of the workload's shapes)",
        "config": {"workload": describe(cfg), "global_batch": total_samples, "seq_len": cfg.T,
                   "parallelism": f"dp{world} (independent batches, no data-path collective)",
                   "l2": "flushed by a 256 MB write between timed steps (outside the step events)",
                   **({"precision": "FP8 serving path: GEMM1 (gate, up) on E4M3 operands, one power-of-two scale "
                                    "per bank weight matrix and per activation row; GEMM2 and residual bf16"}
                      if args.fp8 and not moe else {}),
                   **({"precision": "FP8 serving path: every expert's GEMM1 (routed and shared gate, up) on E4M3 "
                                    "operands, one power-of-two scale per (bank, expert) weight matrix and per "
                                    "activation row; fp32 router, bf16 GEMM2, combine and residuals"}
                      if args.fp8 and moe else {}),
                   **({"step": "tm_block_backward: the mixing sub-layer's forward recomputed (X_rev), then the "
                               "reverting and mixing sub-layer backward passes (dX and all six weight gradients); "
                               "tflops counts the backward's own 12 W F per row and bank, not the recomputation"}
                      if args.backward else {})},
        "tflops": tflops,
        "tc_roofline_frac": tflops / (pk["bf16_tflops"] * step_peak_factor(cfg, args.fp8)),
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": {"value": job_throughput(cfg.B, world, e2e_ms), "unit": "samples/s", "h2d_bytes_per_step": h2d_bytes,
                "d2h_bytes_per_step": io_bytes, "ms_per_step": e2e_ms, "steps": Ke,
                "mode": ("stream: Ke consecutive steps, each copying its batch in and its result out, the copies "
                         "overlapping the neighbouring steps' compute (two device buffers each); one pair of "
                         "events around the whole stream") if streamed else
                        "one step at a time, its copies overlapping its own compute in sample chunks",
                "chunks": None if streamed else (list(chunks) if not isinstance(chunks, int) else chunks),
                "matches_device_result": e2e_exact},
        "gpu_launches": int(launches),
        "launches_per_step": launches / K,
        "kernels": {k: {"launches": v["launches"], "avg_ms": v["total_ms"] / v["launches"],
                        "share": v["total_ms"] / sum(x["total_ms"] for x in kern.values())}
                    for k, v in sorted(kern.items(), key=lambda kv: -kv[1]["total_ms"])},
        "clocks": clk.summary(),
        "wall_s_timed": t_wall,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: about two seconds' worth, from the warm-up steps' time)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(S.CONFIGS))
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--cpu-samples", type=int, default=256)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-samples", type=int, default=128)
    ap.add_argument("--steps-ref", type=int, default=None)
    ap.add_argument("--batch", type=int, default=None,
                    help="run the workload with this many samples instead of its own B (small cases for "
                         "profiler captures; the line's workload string carries the B used)")
    ap.add_argument("--layers", type=int, default=None,
                    help="run the workload with this many blocks (small cases for profiler captures)")
    ap.add_argument("--e2e-mode", choices=["stream", "step"], default="stream",
                    help="end-to-end leg: a stream of steps whose copies overlap the neighbouring steps' compute "
                         "(stream), or each step alone with its copies overlapping its own compute in chunks (step)")
    ap.add_argument("--e2e-chunks", default="ramp",
                    help="end-to-end leg: split the batch into this many equal chunks whose host copies overlap "
                         "the compute, or 'ramp' (chunk sizes 1:3:8:3:1, small at both ends; forward only)")
    ap.add_argument("--backward", action="store_true",
                    help="the dense block backward (training): its own line, not the forward metric's")
    ap.add_argument("--fp8", action="store_true",
                    help="the FP8 E4M3 serving path (GEMM1 of dense banks and of every MoE expert): its own "
                         "line, not the bf16 metric's")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    cfg = S.CONFIGS[args.workload]
    if args.batch is not None:
        if args.batch < 1:
            raise SystemExit("--batch must be positive")
        cfg = cfg.with_(B=args.batch)
    if args.layers is not None:
        if args.layers < 1:
            raise SystemExit("--layers must be positive")
        cfg = cfg.with_(L=args.layers)
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.impl == "reference":
        args.steps_ref = args.steps_ref or min(args.steps or 10, 10)
        run_reference(args, cfg, rank)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, cfg, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

"""Seeded synthetic inputs for the TokenMixer-Large block forward.

This module only prepares inputs: the five workload shapes, the seeds, the
normal draws, and the rounding of each draw to its storage dtype. It computes
no step of the method. The CPU oracle and the CUDA path both receive the very
same stored bits from here, so a parity test compares two computations on one
input.

Recipe (one rule for every workload):
  * X ~ N(0, 1); gate/up weights ~ N(0, 1/fan_in) with fan_in = the sub-layer
    row width; down weights ~ N(0, 1/F) * down_scale (down_scale = 0.01, the
    "down-matrix small init" of the TokenMixer-Large digest, §2.4.4); router
    weights ~ N(0, 1/width) kept in fp32.  No bias.  RMSNorm gain = 1 (None).
  * Each tensor is drawn from its own PCG64 stream, keyed by
    (layer, sub-layer, tensor id, bank) below seed 0, so any one bank can be
    regenerated on its own (the oracle streams large workloads bank by bank).
  * Draws are float32 normals times a float32 std; bf16 storage rounds that
    float32 value to nearest-even.  fp32 storage keeps it as is.
"""
from __future__ import annotations

import os
from dataclasses import dataclass, replace
from typing import Dict, Optional

import numpy as np

# tensor ids inside the seed key
T_X, T_GATE, T_UP, T_DOWN, T_ROUTER, T_SGATE, T_SUP, T_SDOWN, T_GAIN = range(9)
SUB_MIX, SUB_REV = 0, 1
X_CHUNK = 1024  # samples per X seed stream


@dataclass(frozen=True)
class FFNSpec:
    """Feed-forward bank of one sub-layer: a per-token SwiGLU or a sparse per-token MoE."""
    kind: str              # "dense" or "moe"
    hidden: int = 0        # dense: SwiGLU hidden width F
    E: int = 0             # moe: routed experts per bank
    k: int = 0             # moe: experts chosen per row
    hidden_e: int = 0      # moe: hidden width of one routed expert
    hidden_s: int = 0      # moe: hidden width of the shared expert (0 = none)
    alpha: float = 0.0     # moe: gate-value scale

    @property
    def is_moe(self) -> bool:
        return self.kind == "moe"


@dataclass(frozen=True)
class Config:
    name: str
    B: int
    T: int
    D: int
    H: int
    L: int
    dtype: str             # "f32" or "bf16"
    mix: FFNSpec
    rev: FFNSpec
    gap: int = 0           # inter-residual gap (0 = off)
    eps: float = 1e-6
    down_scale: float = 0.01
    seed: int = 0

    @property
    def dh(self) -> int:
        return self.D // self.H

    @property
    def W(self) -> int:
        """Row width of the mixing sub-layer, T*D/H."""
        return self.T * self.D // self.H

    def banks(self, sub: int) -> int:
        return self.H if sub == SUB_MIX else self.T

    def width(self, sub: int) -> int:
        return self.W if sub == SUB_MIX else self.D

    def ffn(self, sub: int) -> FFNSpec:
        return self.mix if sub == SUB_MIX else self.rev

    def with_(self, **kw) -> "Config":
        return replace(self, **kw)


CONFIGS: Dict[str, Config] = {
    # fp32 tiny dense stack: B=64, T=8, D=64, H=8, L=2, F=128
    "tiny_f32_dense": Config("tiny_f32_dense", B=64, T=8, D=64, H=8, L=2, dtype="f32",
                             mix=FFNSpec("dense", hidden=128), rev=FFNSpec("dense", hidden=128)),
    # one dense bf16 block: B=4096, T=16, D=256, H=16, F=1024
    "dense_block_bf16": Config("dense_block_bf16", B=4096, T=16, D=256, H=16, L=1, dtype="bf16",
                               mix=FFNSpec("dense", hidden=1024), rev=FFNSpec("dense", hidden=1024)),
    # non-square mixing: H=8 != T=16, mixing rows of width 768
    "nonsquare_dense_bf16": Config("nonsquare_dense_bf16", B=4096, T=16, D=384, H=8, L=2, dtype="bf16",
                                   mix=FFNSpec("dense", hidden=1536), rev=FFNSpec("dense", hidden=768)),
    # sparse per-token MoE stack: E=8, k=2, alpha=4, shared expert, inter-residual gap 2
    "moe_stack_bf16": Config("moe_stack_bf16", B=8192, T=32, D=512, H=32, L=4, dtype="bf16", gap=2,
                             mix=FFNSpec("moe", E=8, k=2, hidden_e=256, hidden_s=256, alpha=4.0),
                             rev=FFNSpec("moe", E=8, k=2, hidden_e=256, hidden_s=256, alpha=4.0)),
    # large sparse stack: E=16, k=4, alpha=4, shared hidden 768, ~8e9 expert parameters
    "large_moe_stack_bf16": Config("large_moe_stack_bf16", B=16384, T=48, D=768, H=48, L=4, dtype="bf16", gap=2,
                                   mix=FFNSpec("moe", E=16, k=4, hidden_e=512, hidden_s=768, alpha=4.0),
                                   rev=FFNSpec("moe", E=16, k=4, hidden_e=512, hidden_s=768, alpha=4.0)),
}
CONFIG_ORDER = ["tiny_f32_dense", "dense_block_bf16", "nonsquare_dense_bf16",
                "moe_stack_bf16", "large_moe_stack_bf16"]


# ---------------------------------------------------------------- rounding
def bf16_bits(a32: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(a32, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_storage(a32: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return bf16_bits(a32)
    if dtype == "f32":
        return np.ascontiguousarray(a32, dtype=np.float32)
    raise ValueError(dtype)


def to_f64(stored: np.ndarray, dtype: Optional[str] = None) -> np.ndarray:
    """Exact float64 value of a stored array (uint16 = bf16 bits, float32 as is)."""
    if stored.dtype == np.uint16:
        return bf16_to_f32(stored).astype(np.float64)
    return stored.astype(np.float64)


# ---------------------------------------------------------------- draws
def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=tuple(int(k) for k in key))))


def _normal(seed: int, key, shape, std: float) -> np.ndarray:
    out = _rng(seed, *key).standard_normal(shape, dtype=np.float32)
    out *= np.float32(std)
    return out


def make_x(cfg: Config, samples: Optional[np.ndarray] = None) -> np.ndarray:
    """X [B, T, D] (or only the listed samples) in the storage dtype."""
    T, D = cfg.T, cfg.D
    if samples is None:
        samples = np.arange(cfg.B)
    samples = np.asarray(samples)
    out = np.empty((len(samples), T, D), dtype=np.uint16 if cfg.dtype == "bf16" else np.float32)
    chunks = np.unique(samples // X_CHUNK)
    for c in chunks:
        n = min(X_CHUNK, cfg.B - c * X_CHUNK)
        block = _normal(cfg.seed, (0, 0, T_X, c), (n, T, D), 1.0)
        sel = np.nonzero(samples // X_CHUNK == c)[0]
        out[sel] = to_storage(block[samples[sel] - c * X_CHUNK], cfg.dtype)
    return out


def bank_weights(cfg: Config, layer: int, sub: int, bank: int,
                 down_scale: Optional[float] = None) -> Dict[str, np.ndarray]:
    """All weights of one bank of one sub-layer, in storage dtype ([out, in] layout).

    dense: w_gate [F, W], w_up [F, W], w_down [W, F]
    moe:   w_router [E, W] (fp32), we_gate/we_up [E, Fe, W], we_down [E, W, Fe],
           ws_gate/ws_up [Fs, W], ws_down [W, Fs]
    """
    spec, W = cfg.ffn(sub), cfg.width(sub)
    ds = cfg.down_scale if down_scale is None else down_scale
    s, dt = cfg.seed, cfg.dtype
    key = lambda t: (layer, sub, t, bank)
    if not spec.is_moe:
        F = spec.hidden
        return {
            "w_gate": to_storage(_normal(s, key(T_GATE), (F, W), W ** -0.5), dt),
            "w_up": to_storage(_normal(s, key(T_UP), (F, W), W ** -0.5), dt),
            "w_down": to_storage(_normal(s, key(T_DOWN), (W, F), ds * F ** -0.5), dt),
        }
    E, Fe, Fs = spec.E, spec.hidden_e, spec.hidden_s
    out = {
        "w_router": _normal(s, key(T_ROUTER), (E, W), W ** -0.5),
        "we_gate": to_storage(_normal(s, key(T_GATE), (E, Fe, W), W ** -0.5), dt),
        "we_up": to_storage(_normal(s, key(T_UP), (E, Fe, W), W ** -0.5), dt),
        "we_down": to_storage(_normal(s, key(T_DOWN), (E, W, Fe), ds * Fe ** -0.5), dt),
    }
    if Fs > 0:
        out["ws_gate"] = to_storage(_normal(s, key(T_SGATE), (Fs, W), W ** -0.5), dt)
        out["ws_up"] = to_storage(_normal(s, key(T_SUP), (Fs, W), W ** -0.5), dt)
        out["ws_down"] = to_storage(_normal(s, key(T_SDOWN), (W, Fs), ds * Fs ** -0.5), dt)
    return out


def _bank_job(args):
    cfg, layer, sub, bank, ds = args
    return bank_weights(cfg, layer, sub, bank, ds)


def sublayer_weights(cfg: Config, layer: int, sub: int, down_scale: Optional[float] = None,
                     workers: Optional[int] = None) -> Dict[str, np.ndarray]:
    """All banks of one sub-layer stacked on a leading bank axis.

    With workers > 1 the banks are drawn in a spawn-started process pool (spawn, so that it is
    safe after a CUDA context exists in the parent; the caller's main module must be guarded).
    """
    banks = cfg.banks(sub)
    if workers is None:
        # a process pool only on request (TM_SYNTH_WORKERS or the argument): spawn-started workers
        # re-import the caller's main module, which a script without a main guard cannot survive
        workers = int(os.environ.get("TM_SYNTH_WORKERS", "1"))
    workers = max(1, min(workers, banks))
    jobs = [(cfg, layer, sub, b, down_scale) for b in range(banks)]
    if workers <= 1:
        parts = [_bank_job(j) for j in jobs]
    else:
        import multiprocessing as mp
        with mp.get_context("spawn").Pool(workers) as pool:
            parts = pool.map(_bank_job, jobs, chunksize=1)
    return {k: np.stack([p[k] for p in parts]) for k in parts[0]}


def gain(cfg: Config, layer: int, sub: int) -> np.ndarray:
    """An optional non-unit RMSNorm gain (storage dtype), used only by tests of the gain path."""
    g = 1.0 + 0.25 * _normal(cfg.seed, (layer, sub, T_GAIN, 0), (cfg.width(sub),), 1.0)
    return to_storage(g.astype(np.float32), cfg.dtype)


def subsample(B: int, n: int) -> np.ndarray:
    """Deterministic sample subset of size n containing the first and last sample."""
    if n >= B:
        return np.arange(B)
    inner = _rng(12345, B, n).choice(np.arange(1, B - 1), n - 2, replace=False)
    return np.sort(np.concatenate([[0, B - 1], inner])).astype(np.int64)

"""CPU oracle of the TokenMixer-Large block / stack forward (float64).

TEST INFRASTRUCTURE ONLY: imported by tests, by the graft smoke check and by
the CPU-baseline leg of the benchmark, never by the library.
"""
from __future__ import annotations

from functools import lru_cache

import numpy as np

import tm_synth
from . import tokenmixer
from .tokenmixer import (block_forward, mix, revert, rmsnorm, round_bf16, route, silu, softmax, sp_moe,
                         sp_moe_dense_masked, stack_forward, storage_round, sublayer, swiglu, topk)


def synth_banks(cfg, down_scale=None, cache=True):
    """A (layer, sub, bank) -> float64 weight dict getter over the seeded synthetic weights.

    Banks are drawn on demand, so workloads too large to hold in float64 are streamed.
    """
    def get(layer, sub, bank):
        w = tm_synth.bank_weights(cfg, layer, sub, bank, down_scale)
        return {k: tm_synth.to_f64(v) for k, v in w.items()}
    return lru_cache(maxsize=None)(get) if cache else get


def run_stack(cfg, samples=None, down_scale=None, gains=None, cache=True, keep=False, storage=None):
    """Oracle stack forward of a synthetic workload on the given samples (default: all)."""
    X = tm_synth.to_f64(tm_synth.make_x(cfg, samples))
    return stack_forward(X, cfg, synth_banks(cfg, down_scale, cache), gains=gains, keep=keep, storage=storage)

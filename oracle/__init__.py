"""CPU oracle of the TokenMixer-Large block / stack forward (float64).

TEST INFRASTRUCTURE ONLY: imported by tests, by the graft smoke check and by
the CPU-baseline leg of the benchmark, never by the library.
"""
from __future__ import annotations

from functools import lru_cache


import tm_synth
from . import tokenmixer
from .tokenmixer import (block_forward, mix, revert, rmsnorm, round_bf16, route, silu, softmax, sp_moe,
                         sp_moe_dense_masked, stack_forward, storage_round, sublayer, swiglu, topk)


def synth_banks(cfg, down_scale=None, cache=True, workers=None):
    """A (layer, sub, bank) -> float64 weight dict getter over the seeded synthetic weights.

    cache=True keeps every bank once drawn (float64); cache=False draws a bank on every request, so
    workloads too large to hold in float64 are streamed; cache="layer" draws all banks of a layer's
    two sub-layers together (in a spawn-started pool of `workers` processes), keeps them in their
    storage dtype until another layer is requested, and converts a bank to float64 on request --
    for streaming the largest workload layer by layer when the oracle visits each bank more than once.
    """
    def get(layer, sub, bank):
        w = tm_synth.bank_weights(cfg, layer, sub, bank, down_scale)
        return {k: tm_synth.to_f64(v) for k, v in w.items()}
    if cache == "layer":
        held = {}

        def get_layer(layer, sub, bank):
            if held.get("layer") != layer:
                held.clear()
                held["layer"] = layer
                for s in (0, 1):
                    held[s] = tm_synth.sublayer_weights(cfg, layer, s, down_scale, workers)
            return {k: tm_synth.to_f64(v[bank]) for k, v in held[sub].items()}
        return get_layer
    return lru_cache(maxsize=None)(get) if cache else get


def run_stack(cfg, samples=None, down_scale=None, gains=None, cache=True, keep=False, storage=None):
    """Oracle stack forward of a synthetic workload on the given samples (default: all)."""
    X = tm_synth.to_f64(tm_synth.make_x(cfg, samples))
    return stack_forward(X, cfg, synth_banks(cfg, down_scale, cache), gains=gains, keep=keep, storage=storage)

"""GPU parity of the scoring head and of end-to-end scoring (tokenizer -> stack -> head) through
the C ABI, against the float64 oracle (oracle/tokenmixer.py: head, model_forward)."""
import numpy as np
import pytest
import torch

import oracle
import tm_synth as S
from oracle import tokenmixer as O
from tm_synth import FFNSpec
from token_sparse_moe_b200 import api

from parity_util import rms, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _dev(a, dtype):
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16 if dtype == "bf16" else torch.float32).to(DEV)


def _store(a, dtype):
    return O.round_bf16(a) if dtype == "bf16" else a.astype(np.float32).astype(np.float64)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_head_matches_oracle(dtype):
    rng = np.random.default_rng(7)
    B, T, D = 1000, 16, 256                        # 8 KB of bf16 per sample, a ragged last block of warps
    X = _store(rng.standard_normal((B, T, D)), dtype)
    w = _store(rng.standard_normal(D) / np.sqrt(D), dtype)
    sh = api.shape(B, T, D, 16, dtype)
    got = to_np(api.head_forward(_dev(X, dtype), sh, _dev(w, dtype)))
    want = O.head(X, w)
    # fp32 accumulation of T*D products: bounded by a few ulps of the sum of |terms| / T
    scale = np.abs(X).mean(axis=1) @ np.abs(w)
    assert np.all(np.abs(got - want) <= 1e-5 * scale + 1e-7)


@pytest.mark.parametrize("cfg", [
    S.Config("score_dense", B=300, T=16, D=256, H=16, L=3, gap=2, dtype="bf16",
             mix=FFNSpec("dense", hidden=256), rev=FFNSpec("dense", hidden=384)),
    S.Config("score_f32", B=130, T=8, D=64, H=8, L=2, gap=0, dtype="f32",
             mix=FFNSpec("dense", hidden=128), rev=FFNSpec("dense", hidden=96)),
], ids=lambda c: c.name)
def test_model_forward_matches_oracle(cfg):
    # dense stacks: the chaining of tokenizer, stack (with the inter-residual) and head is under
    # test; routing near-ties of MoE stacks are the stack tests' business
    rng = np.random.default_rng(11)
    G, dg = cfg.T - 1, 24
    groups = _store(rng.standard_normal((cfg.B, G, dg)), cfg.dtype)
    w_group = _store(rng.standard_normal((G, cfg.D, dg)) / np.sqrt(dg), cfg.dtype)
    w_global = _store(rng.standard_normal((cfg.D, G * dg)) / np.sqrt(G * dg), cfg.dtype)
    w_head = _store(rng.standard_normal(cfg.D) / np.sqrt(cfg.D), cfg.dtype)
    blocks = api.blocks_from_synth(cfg, DEV)
    logits = to_np(api.model_forward(_dev(groups, cfg.dtype), _dev(w_group, cfg.dtype), _dev(w_global, cfg.dtype),
                                     blocks, cfg.gap, _dev(w_head, cfg.dtype), api.config_shape(cfg)))
    api.get_device_error()
    o = O.model_forward(groups, w_group, w_global, cfg, oracle.synth_banks(cfg), w_head, storage=cfg.dtype)
    e = float(np.max(np.abs(logits - o["logits"])) / rms(o["logits"]))
    # the logits average the stored stack output, so they inherit its bf16 storage error averaged
    # over T*D terms: the same 2e-2 (bf16) / 1e-4 (fp32) bars as the stack, relative to rms
    assert e <= (2e-2 if cfg.dtype == "bf16" else 1e-4), e

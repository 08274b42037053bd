"""GPU parity of the dense backward (tm_pertoken_swiglu_backward, tm_block_backward) through the
C ABI against the float64 backward oracle, element by element on the same seeded inputs.

Bar, per gradient tensor (dx and each weight gradient, all banks together), derived from the
arithmetic of a bf16 path (the workloads give a bar for the forward only):
  * rms(g - o) / rms(o) <= 1e-2: every tensor the path stores between its contractions (the
    normalised rows, the recomputed projections, the hidden gradients, the gradient at the
    normalised row, the result) is rounded to bf16, a relative error of at most 2^-9 each, about
    1.1e-3 in rms; the chain has a handful of them, and a float64 model of exactly these
    roundings lands at 4.3e-3 on every case here;
  * max(0, |g - o| - ulp(o)) / rms(o) <= 5e-2: gradients are products of several normal
    factors, so their largest elements reach 8-12 times their rms, where one bf16 ulp is already
    3-6 % of the rms.  The result's own storage rounding therefore gets one ulp; what remains is
    the propagated rounding of the intermediates, up to 3.0e-2 in the same float64 model (the
    forward's 2e-2 of the plain max error cannot hold here: rounding the exact gradient to bf16
    alone, with nothing else rounded, reaches 1.4e-2 to 2.2e-2).
The oracle is exact: it rounds only X_rev, the tensor the block's forward stores between its
sub-layers.
"""
import numpy as np
import pytest
import torch

import oracle
import tm_synth as S
from oracle import backward as BW
from oracle import tokenmixer as O
from tm_synth import FFNSpec
from token_sparse_moe_b200 import TMError, api
from token_sparse_moe_b200 import _abi as A

from parity_util import rms, to_np, ulp

RMS_TOL = 1e-2
MAX_TOL = 5e-2

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def small(name, B, T, D, H, mix, rev, L=1, gap=0):
    return S.Config(name, B=B, T=T, D=D, H=H, L=L, dtype="bf16", mix=FFNSpec("dense", hidden=mix),
                    rev=FFNSpec("dense", hidden=rev), gap=gap)


CASES = [
    # head width 16, mixing and reverting rows of width 256; 300 samples = 2 full row tiles + 44
    small("bwd_sq", 300, 16, 256, 16, 384, 256),
    # head width 48 (mixed rows of width 768 through the Mix view), reverting width 384 (192-wide
    # output tiles); 200 samples: the sample dimension of the weight gradients padded to 256
    small("bwd_ns", 200, 16, 384, 8, 256, 128),
    # T != H: mixing rows of width 256 over 4 heads, reverting rows of width 128; 600 samples
    small("bwd_w128", 600, 8, 128, 4, 128, 256),
]


def dev(arr):
    return api.to_device(arr, DEV)


def grads_np(g):
    return {k: to_np(v) for k, v in g.items()}


def check(name, got, want):
    den = rms(want)
    e_rms = rms(got - want) / den
    e_max = float(np.max(np.maximum(np.abs(got - want) - ulp(want, "bf16"), 0.0)) / den)
    assert e_rms <= RMS_TOL and e_max <= MAX_TOL, f"{name}: rms {e_rms:.3e}, max beyond one ulp {e_max:.3e}"
    return e_rms, e_max


def check_bank_grads(g, o, tag):
    for key in ("dw_gate", "dw_up", "dw_down"):
        check(f"{tag}.{key}", g[key], np.stack(o[key]))


def seeded(cfg):
    return S.make_x(cfg), S.make_x(cfg.with_(seed=cfg.seed + 17))


@pytest.mark.parametrize("down_scale", [None, 1.0])
@pytest.mark.parametrize("sub", [0, 1])
@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_sublayer_backward(cfg, sub, down_scale):
    X, dY = seeded(cfg)
    sw = api.sublayer_from_synth(cfg, 0, sub, DEV, down_scale)
    sh = api.config_shape(cfg)
    layout = A.TM_LAYOUT_MIXED if sub == 0 else A.TM_LAYOUT_ROWS
    dx, g = api.pertoken_swiglu_backward(dev(X), dev(dY), layout, sh, sw)
    api.get_device_error()
    X64, dY64 = S.to_f64(X), S.to_f64(dY)
    rows, drows = (O.mix(X64, cfg.H), O.mix(dY64, cfg.H)) if sub == 0 else (X64, dY64)
    get = oracle.synth_banks(cfg, down_scale)
    o = BW.sublayer_backward(rows, drows, lambda j: get(0, sub, j), cfg.ffn(sub), cfg.eps)
    odx = O.revert(o["dx"], cfg.T) if sub == 0 else o["dx"]
    check("dx", to_np(dx), odx)
    check_bank_grads(grads_np(g), o, f"sub{sub}")


@pytest.mark.parametrize("sub", [0, 1])
def test_sublayer_backward_residual_addend(sub):
    """dx_add = dy: the sub-layer that adds its own input as the residual passes dy straight on."""
    cfg = CASES[0]
    X, dY = seeded(cfg)
    sw = api.sublayer_from_synth(cfg, 0, sub, DEV)
    sh = api.config_shape(cfg)
    layout = A.TM_LAYOUT_MIXED if sub == 0 else A.TM_LAYOUT_ROWS
    dyt = dev(dY)
    dx0, _ = api.pertoken_swiglu_backward(dev(X), dyt, layout, sh, sw)
    dx1, _ = api.pertoken_swiglu_backward(dev(X), dyt, layout, sh, sw, dx_add=dyt)
    api.get_device_error()
    X64, dY64 = S.to_f64(X), S.to_f64(dY)
    rows, drows = (O.mix(X64, cfg.H), O.mix(dY64, cfg.H)) if sub == 0 else (X64, dY64)
    get = oracle.synth_banks(cfg)
    o = BW.sublayer_backward(rows, drows, lambda j: get(0, sub, j), cfg.ffn(sub), cfg.eps)
    odx = (O.revert(o["dx"], cfg.T) if sub == 0 else o["dx"]) + dY64
    check("dx+dy", to_np(dx1), odx)
    # the addend enters in fp32 before the one bf16 rounding of dx
    ref = (to_np(dx0) + dY64).astype(np.float32)
    assert np.max(np.abs(to_np(dx1) - ref)) <= 2.0 ** -7 * np.max(np.abs(ref))


def _block_parity(cfg, down_scale=None):
    X, dY = seeded(cfg)
    blk = api.Block(api.sublayer_from_synth(cfg, 0, 0, DEV, down_scale),
                    api.sublayer_from_synth(cfg, 0, 1, DEV, down_scale))
    sh = api.config_shape(cfg)
    dX, g = api.block_backward(dev(X), dev(dY), blk, sh)
    api.get_device_error()
    get = oracle.synth_banks(cfg, down_scale)
    o = BW.block_backward(S.to_f64(X), cfg, 0, get, S.to_f64(dY), storage="bf16")
    errs = {"dX": check("dX", to_np(dX), o["dX"])}
    check_bank_grads(grads_np(g["mix"]), o["mix"], "mix")
    check_bank_grads(grads_np(g["rev"]), o["rev"], "rev")
    return errs


@pytest.mark.parametrize("down_scale", [None, 1.0])
@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_block_backward(cfg, down_scale):
    _block_parity(cfg, down_scale)


def test_block_backward_full_size_dense_block():
    """The dense block workload (B=4096, T=16, D=256, H=16, F=1024) in full: the weight gradients
    sum over every sample, so the oracle runs the whole batch (float64, ~25 s of host time)."""
    _block_parity(S.CONFIGS["dense_block_bf16"])


def test_backward_deterministic_bits():
    cfg = CASES[0]
    X, dY = seeded(cfg)
    blk = api.Block(api.sublayer_from_synth(cfg, 0, 0, DEV), api.sublayer_from_synth(cfg, 0, 1, DEV))
    sh = api.config_shape(cfg)
    a, ga = api.block_backward(dev(X), dev(dY), blk, sh)
    b, gb = api.block_backward(dev(X), dev(dY), blk, sh)
    api.get_device_error()
    assert torch.equal(a, b)
    for s in ("mix", "rev"):
        for k in ga[s]:
            assert torch.equal(ga[s][k], gb[s][k]), (s, k)


def test_backward_rejects_a_norm_gain():
    """The GPU backward supports gain 1 only; a gain is refused before any launch (MoE blocks are
    refused the same way, checked on the CPU in test_abi)."""
    cfg = CASES[0]
    X, dY = seeded(cfg)
    sw = api.sublayer_from_synth(cfg, 0, 1, DEV, with_gain=True)
    with pytest.raises(TMError):
        api.pertoken_swiglu_backward(dev(X), dev(dY), A.TM_LAYOUT_ROWS, api.config_shape(cfg), sw)


STACKS = [
    # four blocks, inter-residual after block 2 (X_2 += X_0; none after the last block)
    small("bwd_stack_gap2", 300, 16, 256, 16, 256, 384, L=4, gap=2),
    # three blocks with gap 1 (X_1 += X_0, X_2 += X_1) on the width-128 geometry
    small("bwd_stack_gap1", 200, 8, 128, 4, 128, 256, L=3, gap=1),
]


@pytest.mark.parametrize("cfg", STACKS, ids=lambda c: c.name)
def test_stack_backward(cfg):
    """tm_stack_backward against the oracle's stack backward (the forward recomputed with the bf16
    storage of X_rev and of every block output, the inter-residual's gradient handed back)."""
    X, dY = seeded(cfg)
    blocks = api.blocks_from_synth(cfg, DEV)
    sh = api.config_shape(cfg)
    dX, grads = api.stack_backward(dev(X), dev(dY), blocks, cfg.gap, sh)
    api.get_device_error()
    o = BW.stack_backward(S.to_f64(X), cfg, oracle.synth_banks(cfg), S.to_f64(dY), storage="bf16")
    check("dX", to_np(dX), o["dX"])
    for l in range(cfg.L):
        check_bank_grads(grads_np(grads[l]["mix"]), o["blocks"][l]["mix"], f"block{l}.mix")
        check_bank_grads(grads_np(grads[l]["rev"]), o["blocks"][l]["rev"], f"block{l}.rev")


def test_stack_backward_one_block_is_block_backward():
    """L = 1: the stack backward is the block backward, bit for bit."""
    cfg = CASES[0]
    X, dY = seeded(cfg)
    blk = api.Block(api.sublayer_from_synth(cfg, 0, 0, DEV), api.sublayer_from_synth(cfg, 0, 1, DEV))
    sh = api.config_shape(cfg)
    a, ga = api.block_backward(dev(X), dev(dY), blk, sh)
    b, gb = api.stack_backward(dev(X), dev(dY), [blk], 0, sh)
    api.get_device_error()
    assert torch.equal(a, b)
    for s in ("mix", "rev"):
        for k in ga[s]:
            assert torch.equal(ga[s][k], gb[0][s][k]), (s, k)

"""GPU parity: the CUDA path through the C ABI against the float64 oracle, element by
element on the same seeded inputs.

Small cases span several 128-row tiles with a ragged tail and every kernel path
(TMA Mix map, 3-D row map, cp.async gather, each output tile width, fp32 CUDA-core
path).  The full-size workloads run the whole batch on the GPU and compare a
deterministic sample subset (first and last sample included) with the oracle;
samples are independent, so the subset's rows are exact oracle outputs.
"""
import numpy as np
import pytest
import torch

import oracle
import tm_synth as S
from oracle import tokenmixer as O
from tm_synth import FFNSpec
from token_sparse_moe_b200 import TMError, api
from token_sparse_moe_b200 import _abi as A

from parity_util import (BF16_TOL, F32_TOL, GAP_TOL, check_buckets, check_routing, check_stack, err, err_bf16,
                         err_delta, err_f32, err_moe_delta, oracle_sublayer, rms, routed_abs_contrib, to_np, tol)

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def small(name, B, T, D, H, dtype, mix, rev, L=1, gap=0):
    return S.Config(name, B=B, T=T, D=D, H=H, L=L, dtype=dtype, mix=mix, rev=rev, gap=gap)


def moe(E, k, Fe, Fs, alpha=None):
    return FFNSpec("moe", E=E, k=k, hidden_e=Fe, hidden_s=Fs, alpha=float(E) / k if alpha is None else alpha)


DENSE_SMALL = [
    # dh = 16: Mix read through the 4-D tensor map; rows through the 3-D map; 300 rows = 2 full tiles + 44
    small("dense_sq", 300, 16, 256, 16, "bf16", FFNSpec("dense", hidden=384), FFNSpec("dense", hidden=256)),
    # dh = 48: three 16-column Mix boxes per head; hidden 192/320 -> 64-wide hidden tiles; rev width 384 -> 192-wide
    small("dense_ns", 200, 16, 384, 8, "bf16", FFNSpec("dense", hidden=192), FFNSpec("dense", hidden=320)),
    # fp32 CUDA-core path
    small("dense_f32", 150, 8, 64, 8, "f32", FFNSpec("dense", hidden=128), FFNSpec("dense", hidden=96)),
    # one 128-row tile per bank, width 128; mixing hidden 192 takes the 64-wide-chunk fused kernel
    small("dense_one_tile", 100, 16, 128, 16, "bf16", FFNSpec("dense", hidden=192), FFNSpec("dense", hidden=128)),
    # width 128 and 256 with 5 row tiles (an odd count on CTA pairs: the last pair's second tile is empty)
    small("dense_w128", 600, 8, 128, 4, "bf16", FFNSpec("dense", hidden=128), FFNSpec("dense", hidden=256)),
    # 160 tiles on 148 SMs: a last wave of 12 tiles
    small("dense_split", 1280, 16, 256, 16, "bf16", FFNSpec("dense", hidden=384), FFNSpec("dense", hidden=256)),
    # width 128: 8 banks x 19 tiles (the last one ragged) = 152 tiles, a last wave of 4
    small("dense_split_w128", 2400, 8, 128, 4, "bf16", FFNSpec("dense", hidden=256), FFNSpec("dense", hidden=512)),
]
MOE_SMALL = [
    # tensor-core router; routed rows copied into bucket order, then read by GEMM1 through a 2-D map
    small("moe_sq", 300, 16, 256, 16, "bf16", moe(8, 2, 128, 128, 4.0), moe(4, 1, 64, 192, 4.0)),
    small("moe_ns", 260, 8, 384, 4, "bf16", moe(16, 4, 128, 256), moe(6, 3, 64, 64)),
    # 24 experts: the CUDA-core router; mixed rows then reach GEMM1 through the bucket-order copy
    small("moe_e24", 170, 8, 256, 8, "bf16", moe(24, 3, 64, 64), moe(24, 2, 64, 128)),
    # head width 64: four 16-column pieces per token in the Mix geometry
    small("moe_dh64", 150, 8, 256, 4, "bf16", moe(8, 2, 128, 128), moe(4, 2, 64, 128)),
    small("moe_f32", 150, 8, 64, 8, "f32", moe(4, 2, 64, 32), moe(8, 3, 32, 64)),
]


def dev(arr):
    return api.to_device(arr, DEV)


def inputs(cfg):
    X = S.make_x(cfg)
    R = S.make_x(cfg.with_(seed=cfg.seed + 17))
    return X, R


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("T,D,H", [(16, 256, 16), (16, 384, 8), (8, 64, 8), (32, 512, 32), (48, 768, 48), (5, 40, 10)])
def test_mix_revert_bit_exact(dtype, T, D, H):
    cfg = small("m", 37, T, D, H, dtype, FFNSpec("dense", hidden=64), FFNSpec("dense", hidden=64))
    X = S.make_x(cfg)
    Hm = api.mix(dev(X), H)
    ref = O.mix(S.to_f64(X), H)
    assert np.array_equal(to_np(Hm), ref)
    back = api.revert(Hm, T)
    assert np.array_equal(to_np(back), S.to_f64(X))


def check_outputs(cfg, y, o, x, down_scale):
    """Small-init workloads: the stated measure (fp32: max relative error, bf16: max abs / rms).
    Down weights at std x 1 (the FFN term is as large as the residual, so outputs cancel to
    near zero in places and reach |y| ~ 8 in others): the FFN's own error beyond one ulp of
    the stored output, relative to rms(o - x), at the dtype's tolerance."""
    if down_scale is None:
        assert err(cfg.dtype, y, o) <= tol(cfg.dtype), err(cfg.dtype, y, o)
    else:
        assert err_delta(y, o, x, cfg.dtype) <= tol(cfg.dtype), err_delta(y, o, x, cfg.dtype)


def _run_sub(cfg, sub, X, R, down_scale=None, with_gain=False):
    sw = api.sublayer_from_synth(cfg, 0, sub, DEV, down_scale, with_gain)
    sh = api.config_shape(cfg)
    layout = A.TM_LAYOUT_MIXED if sub == 0 else A.TM_LAYOUT_ROWS
    fn = api.sparse_pertoken_moe if sw.is_moe else api.pertoken_swiglu
    y = fn(dev(X), dev(R), layout, sh, sw)
    api.get_device_error()
    return to_np(y), sw


def _oracle_sub(cfg, sub, X, R, down_scale=None, with_gain=False):
    X64, R64 = S.to_f64(X), S.to_f64(R)
    g = S.to_f64(S.gain(cfg, 0, sub)) if with_gain else None
    if sub == 0:
        rows = O.mix(X64, cfg.H)
        r = oracle_sublayer(cfg, 0, 0, rows, down_scale, g)
        return O.revert(r["out"] + O.mix(R64, cfg.H), cfg.T), r, rows
    r = oracle_sublayer(cfg, 0, 1, X64, down_scale, g)
    return r["out"] + R64, r, X64


@pytest.mark.parametrize("down_scale", [None, 1.0])
@pytest.mark.parametrize("sub", [0, 1])
@pytest.mark.parametrize("cfg", DENSE_SMALL, ids=lambda c: c.name)
def test_dense_sublayer(cfg, sub, down_scale):
    X, R = inputs(cfg)
    y, _ = _run_sub(cfg, sub, X, R, down_scale)
    o, _, _ = _oracle_sub(cfg, sub, X, R, down_scale)
    R64 = S.to_f64(R)
    check_outputs(cfg, y, o, R64, down_scale)


@pytest.mark.parametrize("resid", ["input", "none"])
@pytest.mark.parametrize("sub", [0, 1])
@pytest.mark.parametrize("cfg", [DENSE_SMALL[0], DENSE_SMALL[4]], ids=lambda c: c.name)
def test_dense_sublayer_residual_forms(cfg, sub, resid):
    """The residual is the sub-layer input itself (the tensor core adds it from the resident input
    tile) or absent; both against the oracle with R = X and R = 0."""
    X, _ = inputs(cfg)
    sw = api.sublayer_from_synth(cfg, 0, sub, DEV)
    sh = api.config_shape(cfg)
    layout = A.TM_LAYOUT_MIXED if sub == 0 else A.TM_LAYOUT_ROWS
    Xd = dev(X)
    y = api.pertoken_swiglu(Xd, Xd if resid == "input" else None, layout, sh, sw)
    api.get_device_error()
    R = X if resid == "input" else np.zeros_like(X)
    o, _, _ = _oracle_sub(cfg, sub, X, R)
    if resid == "input":
        check_outputs(cfg, to_np(y), o, S.to_f64(R), None)
    else:
        # no residual: y is the FFN term alone, whose bf16 storage rounding reaches 2^-9 |y| at the
        # tails (|y| ~ 10 rms), so one ulp of the stored value is allowed first
        assert err_delta(to_np(y), o, 0.0, cfg.dtype) <= tol(cfg.dtype)


@pytest.mark.parametrize("sub", [0, 1])
@pytest.mark.parametrize("cfg", MOE_SMALL, ids=lambda c: c.name)
def test_route_topk(cfg, sub):
    X, _ = inputs(cfg)
    sw = api.sublayer_from_synth(cfg, 0, sub, DEV)
    layout = A.TM_LAYOUT_MIXED if sub == 0 else A.TM_LAYOUT_ROWS
    r = api.route_topk(dev(X), layout, api.config_shape(cfg), sw)
    api.get_device_error()
    X64 = S.to_f64(X)
    rows = O.mix(X64, cfg.H) if sub == 0 else X64
    info = oracle_sublayer(cfg, 0, sub, rows)
    spec = cfg.ffn(sub)
    idx = r["idx"].cpu().numpy()
    bad, near = check_routing(idx, r["gate"].cpu().numpy(), info, spec.alpha, spec.E)
    assert bad == 0, f"{bad} rows routed differently outside near ties ({near} near-tie rows)"
    inv = 1.0 / np.sqrt(np.mean(rows * rows, axis=-1) + cfg.eps)
    assert np.allclose(r["inv_rms"].cpu().numpy(), inv, rtol=1e-5)
    # logit_gap_opt: z_(k) - z_(k+1) of the GPU's fp32 logits against the oracle's (+inf when k == E)
    gg = r["gap"].cpu().numpy().astype(np.float64)
    og = info["gap"]
    assert np.array_equal(np.isfinite(gg), np.isfinite(og))
    fin = np.isfinite(og)
    assert np.all(gg[fin] >= 0.0)
    assert np.max(np.abs(gg[fin] - og[fin]), initial=0.0) <= 1e-4, np.max(np.abs(gg[fin] - og[fin]))
    check_buckets(idx, r["offsets"].cpu().numpy(), r["rows"].cpu().numpy(), r["slot_of"].cpu().numpy(), spec.E)


@pytest.mark.parametrize("down_scale", [None, 1.0])
@pytest.mark.parametrize("sub", [0, 1])
@pytest.mark.parametrize("cfg", MOE_SMALL, ids=lambda c: c.name)
def test_moe_sublayer(cfg, sub, down_scale):
    X, R = inputs(cfg)
    y, sw = _run_sub(cfg, sub, X, R, down_scale)
    o, info, rows = _oracle_sub(cfg, sub, X, R, down_scale)
    layout = A.TM_LAYOUT_MIXED if sub == 0 else A.TM_LAYOUT_ROWS
    gi = api.route_topk(dev(X), layout, api.config_shape(cfg), sw)["idx"].cpu().numpy()
    flip = np.any(np.sort(gi, -1) != np.sort(info["idx"], -1), axis=-1)            # [B, banks]
    assert np.all(info["gap"][flip] < GAP_TOL), "routing differs outside a near tie"
    if down_scale is None:
        assert err(cfg.dtype, y, o) <= tol(cfg.dtype), err(cfg.dtype, y, o)
        return
    # FFN term as large as the residual: per element, the FFN's error beyond the output's own
    # ulp and the bf16 rounding of the routed expert rows must stay within tol * rms(o - x).
    # Samples where a near tie flipped an expert carry a different (valid) expert: left out.
    keep = ~np.any(flip, axis=1)
    c = routed_abs_contrib(cfg, 0, sub, rows, down_scale)
    if sub == 0:
        c = O.revert(c, cfg.T)
    R64 = S.to_f64(R)
    e = err_moe_delta(y[keep], o[keep], R64[keep], c[keep], cfg.dtype)
    assert e <= tol(cfg.dtype), e


@pytest.mark.parametrize("tied", [False, True], ids=["generic", "tied_router"])
@pytest.mark.parametrize("sub", [0, 1])
@pytest.mark.parametrize("cfg", MOE_SMALL, ids=lambda c: c.name)
def test_moe_sublayer_teacher_forced(cfg, sub, tied):
    """Every row of an MoE sub-layer against the oracle routed by the GPU's own expert choices
    (the oracle's teacher-forced mode), near ties included.  With tied routers, experts 0 and 1
    of every bank share one router row, so their logits are equal for every row and the top-k
    at the tie is decided by each side's own tie-breaking: the forced oracle follows the GPU."""
    X, R = inputs(cfg)
    sw = api.sublayer_from_synth(cfg, 0, sub, DEV, 1.0)
    base = oracle.synth_banks(cfg, 1.0)
    get = base
    if tied:
        sw.tensors["w_router"][:, 1].copy_(sw.tensors["w_router"][:, 0])

        def get(layer, s, j):
            w = dict(base(layer, s, j))
            w["w_router"] = w["w_router"].copy()
            w["w_router"][1] = w["w_router"][0]
            return w
    sh = api.config_shape(cfg)
    layout = A.TM_LAYOUT_MIXED if sub == 0 else A.TM_LAYOUT_ROWS
    gi = api.route_topk(dev(X), layout, sh, sw)["idx"].cpu().numpy().astype(np.int64)
    y = to_np(api.sparse_pertoken_moe(dev(X), dev(R), layout, sh, sw))
    api.get_device_error()
    X64, R64 = S.to_f64(X), S.to_f64(R)
    rows = O.mix(X64, cfg.H) if sub == 0 else X64
    res = R64 if sub == 1 else O.mix(R64, cfg.H)
    r = oracle_sublayer(cfg, 0, sub, rows, forced_idx=gi, get=get)
    o = r["out"] + res
    c = routed_abs_contrib(cfg, 0, sub, rows, forced_idx=gi, get=get)
    if sub == 0:
        o, c = O.revert(o, cfg.T), O.revert(c, cfg.T)
    e = err_moe_delta(y, o, R64, c, cfg.dtype)
    assert e <= tol(cfg.dtype), e
    # the GPU's choices differ from the oracle's own only inside near ties (exact ones included)
    own = oracle_sublayer(cfg, 0, sub, rows, get=get)
    flip = np.any(np.sort(gi, -1) != np.sort(own["idx"], -1), axis=-1)
    assert np.all(own["gap"][flip] < GAP_TOL)


@pytest.mark.parametrize("cfg", [DENSE_SMALL[0], MOE_SMALL[0], DENSE_SMALL[2]], ids=lambda c: c.name)
def test_norm_gain(cfg):
    X, R = inputs(cfg)
    for sub in (0, 1):
        y, _ = _run_sub(cfg, sub, X, R, 1.0, with_gain=True)
        o, _, rows = _oracle_sub(cfg, sub, X, R, 1.0, with_gain=True)
        if cfg.ffn(sub).is_moe:
            # the gain is folded into the bf16 gate and up weights: two more roundings of at
            # most 2^-8 each on every expert's output, routed and shared, on top of the slot one
            g = S.to_f64(S.gain(cfg, 0, sub))
            c = routed_abs_contrib(cfg, 0, sub, rows, 1.0, g)
            call = routed_abs_contrib(cfg, 0, sub, rows, 1.0, g, include_shared=True)
            if sub == 0:
                c, call = O.revert(c, cfg.T), O.revert(call, cfg.T)
            e = err_moe_delta(y, o, S.to_f64(R), c, cfg.dtype, extra=2 * 2.0 ** -8 * call)
            assert e <= tol(cfg.dtype), e
        else:
            check_outputs(cfg, y, o, S.to_f64(R), 1.0)


def _stack_gpu(cfg, down_scale=None, samples=None, blocks=None):
    """The stack over the whole batch; returns (float64 copy of the rows `samples` (all when None),
    the device blocks)."""
    import os
    big = cfg.B * cfg.T * cfg.D > 1e8
    if blocks is None:
        blocks = api.blocks_from_synth(cfg, DEV, down_scale, workers=min(16, os.cpu_count() or 1) if big else 1)
    sh = api.config_shape(cfg)
    X = S.make_x(cfg)
    Y = api.stack_forward(dev(X), blocks, cfg.gap, sh)
    api.get_device_error()
    Y = to_np(Y)
    return (Y if samples is None else Y[samples]), blocks


@pytest.mark.parametrize("cfg", [
    small("stack_moe", 200, 16, 256, 16, "bf16", moe(8, 2, 128, 128), moe(8, 2, 128, 128), L=4, gap=2),
    small("stack_dense", 200, 16, 256, 16, "bf16", FFNSpec("dense", hidden=256), FFNSpec("dense", hidden=256), L=5, gap=2),
    small("stack_f32_moe", 130, 8, 64, 8, "f32", moe(4, 2, 64, 64), moe(4, 1, 32, 32), L=3, gap=2),
], ids=lambda c: c.name)
def test_small_stack_with_inter_residual(cfg):
    y, blocks = _stack_gpu(cfg)
    check_stack(cfg, blocks, y)


def test_fp32_stack_tiny_config_full():
    cfg = S.CONFIGS["tiny_f32_dense"]
    y, blocks = _stack_gpu(cfg)
    _, res = check_stack(cfg, blocks, y)
    o = res["Y"][-1]
    assert err_f32(y, o) <= F32_TOL
    assert err_delta(y, o, S.to_f64(S.make_x(cfg)), "f32") <= 1e-3


@pytest.mark.parametrize("name,n", [("dense_block_bf16", 256), ("nonsquare_dense_bf16", 128), ("moe_stack_bf16", 64),
                                    ("large_moe_stack_bf16", 32)])
def test_full_size_config(name, n):
    """The whole batch of each workload on the GPU; a deterministic sample subset (first and last
    included) against the oracle, every block, every sampled row at the stated tolerance, the top-k
    of every MoE sub-layer compared with the oracle's own (near ties counted)."""
    cfg = S.CONFIGS[name]
    samples = S.subsample(cfg.B, n)
    y, blocks = _stack_gpu(cfg, samples=samples)
    check_stack(cfg, blocks, y, samples)


def test_block_forward_matches_stack_and_returns_revert():
    cfg = DENSE_SMALL[0]
    X, _ = inputs(cfg)
    blocks = api.blocks_from_synth(cfg, DEV)
    sh = api.config_shape(cfg)
    Xd = dev(X)
    Xr = torch.empty_like(Xd)
    Y = api.block_forward(Xd, blocks[0], sh, X_revert=Xr)
    api.get_device_error()
    b = O.block_forward(S.to_f64(X), cfg, 0, oracle.synth_banks(cfg), storage="bf16")
    assert err_bf16(to_np(Y), b["Y"]) <= BF16_TOL
    assert err_bf16(to_np(Xr), b["Xr"]) <= BF16_TOL
    assert np.array_equal(to_np(api.stack_forward(Xd, blocks, 0, sh)), to_np(Y))


BLOCK_FUSED = [
    # 3 row tiles x 16 banks: all 96 tiles in one wave, reverting tiles wait on mixing tiles beside them
    DENSE_SMALL[0],
    # 9 row tiles x 16 banks = 144 mixing tiles on 148 SMs: the second item of CTA c is a reverting tile of
    # the row block of its own first (mixing) tile, whose output and count go out before that A load waits
    small("block_selfdep", 1100, 16, 256, 16, "bf16", FFNSpec("dense", hidden=256), FFNSpec("dense", hidden=384)),
    # width 128 (T = H = 8, dh = 16): 20 row tiles x 8 banks = 160 + 160 tiles, waves straddle the sub-layers
    small("block_w128", 2500, 8, 128, 8, "bf16", FFNSpec("dense", hidden=256), FFNSpec("dense", hidden=128)),
]


def _fused_launches(fn):
    api.profile_start()
    out = fn()
    api.get_device_error()
    return out, api.profile_stop().get("fused_swiglu", {}).get("launches", 0)


@pytest.mark.parametrize("cfg", BLOCK_FUSED, ids=lambda c: c.name)
@pytest.mark.parametrize("with_gain", [False, True], ids=["gain1", "gain"])
def test_fused_block_one_launch(cfg, with_gain, monkeypatch):
    """Both dense sub-layers of a block in one launch (mixing tiles, then reverting tiles that wait
    for their row block): the same bits as one launch per sub-layer, since every tile does the same
    arithmetic, X_revert included; within tolerance of the oracle."""
    X, _ = inputs(cfg)
    blk = api.Block(api.sublayer_from_synth(cfg, 0, 0, DEV, None, with_gain),
                    api.sublayer_from_synth(cfg, 0, 1, DEV, None, with_gain))
    sh = api.config_shape(cfg)
    Xd = dev(X)

    def run():
        Xr = torch.empty_like(Xd)
        return api.block_forward(Xd, blk, sh, X_revert=Xr), Xr
    (Y1, Xr1), n1 = _fused_launches(run)
    monkeypatch.setenv("TM_FUSED_BLOCK", "0")
    (Y0, Xr0), n0 = _fused_launches(run)
    monkeypatch.delenv("TM_FUSED_BLOCK")
    assert (n1, n0) == (1, 2)
    assert torch.equal(Y1.view(torch.int16), Y0.view(torch.int16))
    assert torch.equal(Xr1.view(torch.int16), Xr0.view(torch.int16))
    gains = tuple(S.to_f64(S.gain(cfg, 0, sub)) for sub in (0, 1)) if with_gain else (None, None)
    b = O.block_forward(S.to_f64(X), cfg, 0, oracle.synth_banks(cfg), gains=gains, storage="bf16")
    assert err_bf16(to_np(Y1), b["Y"]) <= BF16_TOL
    assert err_bf16(to_np(Xr1), b["Xr"]) <= BF16_TOL


def test_fused_block_stack_with_inter_residual(monkeypatch):
    """A dense stack with the inter-residual (gap 2) through one launch per block: the same bits as
    one launch per sub-layer, and the oracle's stack within tolerance."""
    cfg = small("stack_blk", 700, 16, 256, 16, "bf16", FFNSpec("dense", hidden=256), FFNSpec("dense", hidden=512),
                L=3, gap=2)
    (y1, blocks), n1 = _fused_launches(lambda: _stack_gpu(cfg))
    monkeypatch.setenv("TM_FUSED_BLOCK", "0")
    (y0, _), n0 = _fused_launches(lambda: _stack_gpu(cfg, blocks=blocks))
    monkeypatch.delenv("TM_FUSED_BLOCK")
    assert (n1, n0) == (3, 6)
    assert np.array_equal(y1, y0)       # float64 copies of the bf16 outputs
    check_stack(cfg, blocks, y1)


def test_deterministic_bits():
    cfg = MOE_SMALL[0].with_(L=2, gap=2)
    blocks = api.blocks_from_synth(cfg, DEV)
    sh = api.config_shape(cfg)
    X = dev(S.make_x(cfg))
    run = api.StackRunner(blocks, sh, cfg.gap, DEV)
    Y1 = run(X, torch.empty_like(X)).clone()
    Y2 = run(X, torch.empty_like(X))
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))


@pytest.mark.parametrize("cfg", [DENSE_SMALL[0], DENSE_SMALL[3], MOE_SMALL[0], MOE_SMALL[1]], ids=lambda c: c.name)
def test_rows_give_the_same_bits_wherever_they_sit(cfg):
    """Samples are independent, so each sample's output bits must not depend on where it sits in
    the batch (its row within a 128-row tile, its bucket position): the batch in reverse order and
    a shuffled half of it give the same rows as the batch in order."""
    c = cfg.with_(L=2, gap=0)
    blocks = api.blocks_from_synth(c, DEV)
    X = dev(S.make_x(c))
    Y = api.stack_forward(X, blocks, 0, api.config_shape(c))
    rev = torch.arange(c.B - 1, -1, -1, device=DEV)
    Yr = api.stack_forward(X[rev].contiguous(), blocks, 0, api.config_shape(c))
    assert torch.equal(Yr.view(torch.int16), Y[rev].view(torch.int16))
    sub = torch.from_numpy(np.random.default_rng(5).permutation(c.B)[: c.B // 2].copy()).to(DEV)
    Ys = api.stack_forward(X[sub].contiguous(), blocks, 0, api.config_shape(c.with_(B=c.B // 2)))
    api.get_device_error()
    assert torch.equal(Ys.view(torch.int16), Y[sub].view(torch.int16))


@pytest.mark.parametrize("cfg", [MOE_SMALL[0], MOE_SMALL[1], DENSE_SMALL[1]], ids=lambda c: c.name)
def test_cta_pair_gemms_match_single_cta_gemms(cfg, monkeypatch):
    """The grouped GEMMs on CTA pairs (M = 256 per tile, each SM streaming half of the weight rows)
    against the one-CTA form (TM_PAIR=0): the same bits, a stack of two blocks with the gain."""
    c = cfg.with_(L=2, gap=0)
    blocks = [api.Block(api.sublayer_from_synth(c, l, 0, DEV, None, True), api.sublayer_from_synth(c, l, 1, DEV, None, True))
              for l in range(c.L)]
    X = dev(S.make_x(c))
    sh = api.config_shape(c)
    Y1 = api.stack_forward(X, blocks, 0, sh)
    monkeypatch.setenv("TM_PAIR", "0")
    Y0 = api.stack_forward(X, blocks, 0, sh)
    monkeypatch.delenv("TM_PAIR")
    api.get_device_error()
    assert torch.equal(Y1.view(torch.int16), Y0.view(torch.int16))


def test_tokenize_stub():
    rng = np.random.default_rng(3)
    B, G, dg, D = 33, 5, 24, 64
    g = rng.standard_normal((B, G, dg)).astype(np.float32)
    wg = rng.standard_normal((G, D, dg)).astype(np.float32)
    wG = rng.standard_normal((D, G * dg)).astype(np.float32)
    X = api.tokenize_stub(dev(g), dev(wg), dev(wG), D, 8)
    ref = O.tokenize(g.astype(np.float64), wg.astype(np.float64), wG.astype(np.float64))
    # unit-scale random weights: outputs are sums of 120 terms that cancel near zero in places,
    # so the fp32 accumulation error is measured against the output rms
    assert err_bf16(to_np(X), ref) <= 1e-5, err_bf16(to_np(X), ref)


def test_workspace_too_small_is_reported():
    cfg = DENSE_SMALL[0]
    X, R = inputs(cfg)
    sw = api.sublayer_from_synth(cfg, 0, 0, DEV)
    small_ws = torch.empty(1024, dtype=torch.uint8, device=DEV)
    with pytest.raises(TMError) as e:
        lib = api.lib()
        import ctypes
        sh = api.config_shape(cfg)
        w = sw.dense_c()
        y = torch.empty((cfg.B, cfg.T, cfg.D), dtype=torch.bfloat16, device=DEV)
        A.check(lib.tm_pertoken_swiglu(api._p(dev(X)), None, A.TM_LAYOUT_MIXED, ctypes.byref(sh), None,
                                       ctypes.byref(w), api._p(y), api._p(small_ws), 1024, api._s(None)), "call")
    assert e.value.status == A.TM_ERR_WORKSPACE
    api.get_device_error()


@pytest.mark.parametrize("cfg", [MOE_SMALL[0], DENSE_SMALL[0]], ids=lambda c: c.name)
def test_end_to_end_host_calls_give_the_device_bits(cfg):
    """The end-to-end calls through pinned host memory: the chunked single step (equal chunks and
    the ramp) and the stream of steps with double-buffered copies give the bits of the plain device
    call on the same batch."""
    c = cfg.with_(L=2, gap=1)
    blocks = api.blocks_from_synth(c, DEV)
    sh = api.config_shape(c)
    run = api.StackRunner(blocks, sh, c.gap, DEV)
    X = dev(S.make_x(c))
    Y = torch.empty_like(X)
    run(X, Y)
    Xh = X.cpu().pin_memory()
    s = torch.cuda.Stream()
    for chunks in (1, 4, api.RAMP_CHUNKS):
        Yh = torch.zeros_like(Xh).pin_memory()
        with torch.cuda.stream(s):
            run.run_host(Xh, Yh, torch.empty_like(X), torch.empty_like(X), s, chunks=chunks)
        s.synchronize()
        assert torch.equal(Yh.view(torch.int16), Y.cpu().view(torch.int16)), chunks
    Yh = torch.zeros_like(Xh).pin_memory()
    with torch.cuda.stream(s):
        run.run_host_steps(Xh, Yh, [torch.empty_like(X), torch.empty_like(X)],
                           [torch.empty_like(X), torch.empty_like(X)], 5, s)
    s.synchronize()
    api.get_device_error()
    assert torch.equal(Yh.view(torch.int16), Y.cpu().view(torch.int16))


MOE_DEGENERATE = [
    # k = E: every row reaches every expert (the dense softmax mixture of [digest] Eq. 19 with alpha = 1)
    small("moe_k_eq_E", 200, 8, 256, 8, "bf16", moe(4, 4, 128, 128, 1.0), moe(3, 3, 64, 128, 1.0)),
    # one expert, top-1: softmax over one logit is 1, so the gate is alpha for every row
    small("moe_E1", 170, 8, 256, 8, "bf16", moe(1, 1, 128, 128, 2.0), moe(1, 1, 128, 64, 2.0)),
]


@pytest.mark.parametrize("sub", [0, 1])
@pytest.mark.parametrize("cfg", MOE_DEGENERATE, ids=lambda c: c.name)
def test_moe_degenerate_routing(cfg, sub):
    """The routing's degenerate cases, every row of the sub-layer against the oracle: k = E (no
    choice is made, every bucket holds all rows) and E = 1; the GPU's expert sets equal the oracle's
    (no near tie can change a set that contains every expert)."""
    X, R = inputs(cfg)
    sw = api.sublayer_from_synth(cfg, 0, sub, DEV, 1.0)
    sh = api.config_shape(cfg)
    layout = A.TM_LAYOUT_MIXED if sub == 0 else A.TM_LAYOUT_ROWS
    r = api.route_topk(dev(X), layout, sh, sw)
    y = to_np(api.sparse_pertoken_moe(dev(X), dev(R), layout, sh, sw))
    api.get_device_error()
    spec = cfg.ffn(sub)
    assert spec.k == spec.E
    gi = np.sort(r["idx"].cpu().numpy(), -1)
    assert np.array_equal(gi, np.broadcast_to(np.arange(spec.E), gi.shape))     # every expert, every row
    assert np.all(np.isinf(r["gap"].cpu().numpy()))                            # no expert left out
    X64, R64 = S.to_f64(X), S.to_f64(R)
    rows = O.mix(X64, cfg.H) if sub == 0 else X64
    res = R64 if sub == 1 else O.mix(R64, cfg.H)
    o = oracle_sublayer(cfg, 0, sub, rows, 1.0)["out"] + res
    c = routed_abs_contrib(cfg, 0, sub, rows, 1.0)
    if sub == 0:
        o, c = O.revert(o, cfg.T), O.revert(c, cfg.T)
    e = err_moe_delta(y, o, R64, c, cfg.dtype)
    assert e <= tol(cfg.dtype), e

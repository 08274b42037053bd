"""Shared helpers of the GPU parity tests: error measures and the oracle-side runs.

Tolerances (from the workload descriptions):
  * fp32 tensors: max relative error <= 1e-4, relative to max(|o|, 1e-3 * rms(o));
  * bf16 tensors: max |y - o| / rms(o) <= 2e-2;
  * routing: top-k sets equal wherever the oracle's logit gap z_(k) - z_(k+1) >= 1e-3;
    rows below that gap are counted and reported, and only their validity is checked.
"""
import numpy as np

import oracle
import tm_synth as S
from oracle import tokenmixer as O

F32_TOL = 1e-4
BF16_TOL = 2e-2
GAP_TOL = 1e-3


def rms(a):
    return float(np.sqrt(np.mean(np.square(a))))


def err_bf16(y, o):
    return float(np.max(np.abs(y - o)) / rms(o))


def err_f32(y, o):
    den = np.maximum(np.abs(o), 1e-3 * rms(o))
    return float(np.max(np.abs(y - o) / den))


def ulp(o, dtype):
    """One unit in the last place of the storage dtype at |o| (bf16: 8 significant bits)."""
    mant = 7 if dtype == "bf16" else 23
    e = np.floor(np.log2(np.maximum(np.abs(o), 1e-30)))
    return np.exp2(e - mant)


def err_delta(y, o, x, dtype="bf16"):
    """Error of the sub-layer's own contribution d = y - x, relative to rms(o - x).

    The stored output y carries its storage rounding (up to one ulp of |y|, which at
    |y| ~ 4 is already 3% of a unit-scale d), so that one ulp is allowed before the
    FFN's error is measured: max(0, |y - o| - ulp(o)) / rms(o - x)."""
    excess = np.maximum(np.abs(y - o) - ulp(o, dtype), 0.0)
    return float(np.max(excess) / rms(o - x))


def routed_abs_contrib(cfg, layer, sub, rows, down_scale=None, gain=None, include_shared=False, forced_idx=None,
                       get=None):
    """Per element of each row: sum over the row's chosen experts of |alpha * p_e * Expert_e(n)|
    (plus |Shared(n)| when include_shared).

    The GPU stores each routed expert's output row in bf16 before the combine weights it by
    alpha * p_e, so its rounding error there is at most 2^-8 of this sum.  forced_idx
    [R, banks, k]: the chosen experts, instead of the oracle's own top-k; get: a (layer, sub,
    bank) weight getter in place of the synthetic weights."""
    get = get or oracle.synth_banks(cfg, down_scale)
    spec = cfg.ffn(sub)
    R, banks, W = rows.shape
    out = np.zeros_like(rows)
    for j in range(banks):
        bw = get(layer, sub, j)
        n = O.rmsnorm(rows[:, j, :], cfg.eps, gain)
        r = O.route(n, bw["w_router"], spec.k)
        chosen = r["idx"] if forced_idx is None else forced_idx[:, j, :]
        for e in range(spec.E):
            sel = np.nonzero(np.any(chosen == e, axis=1))[0]
            if sel.size:
                ye = O.swiglu(n[sel], bw["we_gate"][e], bw["we_up"][e], bw["we_down"][e])
                out[sel, j, :] += np.abs(spec.alpha * r["p"][sel, e][:, None] * ye)
        if include_shared and "ws_gate" in bw:
            out[:, j, :] += np.abs(O.swiglu(n, bw["ws_gate"], bw["ws_up"], bw["ws_down"]))
    return out


def err_moe_delta(y, o, x, contrib, dtype="bf16", extra=None):
    """err_delta with the bf16 slot rounding of the routed experts allowed as well:
    max(0, |y - o| - ulp(o) - 2^-8 * contrib - extra) / rms(o - x)."""
    allow = ulp(o, dtype) + (2.0 ** -8 if dtype == "bf16" else 0.0) * contrib
    if extra is not None:
        allow = allow + extra
    excess = np.maximum(np.abs(y - o) - allow, 0.0)
    return float(np.max(excess) / rms(o - x))


def tol(dtype):
    return F32_TOL if dtype == "f32" else BF16_TOL


def err(dtype, y, o):
    return err_f32(y, o) if dtype == "f32" else err_bf16(y, o)


def to_np(t):
    import torch
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy().astype(np.float64)


def oracle_sublayer(cfg, layer, sub, rows, down_scale=None, gain=None, forced_idx=None, get=None):
    """Oracle FFN(Norm(rows)) for one sub-layer of a synthetic workload (no residual); MoE
    sub-layers routed by forced_idx [R, banks, k] when given (teacher forcing)."""
    get = get or oracle.synth_banks(cfg, down_scale)
    return O.sublayer(rows, lambda j: get(layer, sub, j), cfg.ffn(sub), cfg.eps, gain, forced_idx)


def check_routing(gpu_idx, gpu_gate, info, alpha, E):
    """Compare GPU top-k with the oracle's; returns (mismatch rows, near-tie rows)."""
    R, banks, k = gpu_idx.shape
    o_idx, gap, p = info["idx"], info["gap"], info["p"]          # [R, banks, k], [R, banks], [R, banks, E]
    gs = np.sort(gpu_idx, axis=-1)
    os_ = np.sort(o_idx, axis=-1)
    differ = np.any(gs != os_, axis=-1)
    near = gap < GAP_TOL
    bad = differ & ~near
    # the gate of every chosen expert is alpha * p (fp32 softmax vs fp64), descending
    pg = alpha * np.take_along_axis(p, gpu_idx.astype(np.int64), axis=-1)
    assert np.allclose(gpu_gate, pg, rtol=2e-5, atol=1e-6), np.max(np.abs(gpu_gate - pg))
    assert np.all(np.diff(gpu_gate, axis=-1) <= 1e-6)
    # a row routed differently inside a near tie must still pick a valid top-k under the oracle's logits
    z = info["logits"]
    for r, b in zip(*np.nonzero(differ & near)):
        zk = np.sort(z[r, b])[::-1][k - 1]
        assert np.all(z[r, b][gpu_idx[r, b]] >= zk - GAP_TOL)
    return int(bad.sum()), int((differ & near).sum())


def check_buckets(idx, offsets, rows, slot_of, E):
    """Integer structure of the expert-first buckets, against the GPU's own routing (bit exact)."""
    B, banks, k = idx.shape
    G = banks * E
    assert offsets[0] == 0 and offsets[G] == B * banks * k
    bank_of = np.repeat(np.arange(banks), E)
    exp_of = np.tile(np.arange(E), banks)
    counts = np.zeros(G, dtype=np.int64)
    for bk in range(banks):
        for e in range(E):
            counts[bk * E + e] = int(np.sum(np.any(idx[:, bk, :] == e, axis=-1)))
    assert np.array_equal(np.diff(offsets), counts)
    for g in range(G):
        seg = rows[offsets[g]:offsets[g + 1]]
        expect = np.nonzero(np.any(idx[:, bank_of[g], :] == exp_of[g], axis=-1))[0]
        assert np.array_equal(seg, expect), g        # ascending sample order inside a group
    b_idx = np.arange(B)[:, None, None]
    assert np.array_equal(rows[slot_of], np.broadcast_to(b_idx, slot_of.shape))
    g_of = np.arange(banks)[None, :, None] * E + idx
    assert np.all((slot_of >= offsets[g_of]) & (slot_of < offsets[g_of + 1]))


def near_tie_samples(res, R):
    """[R] bool: samples with a routing decision whose oracle logit gap is below GAP_TOL anywhere
    in the stack (either choice is a valid top-k there, and the outputs differ by the swap)."""
    near = np.zeros(R, dtype=bool)
    for b in res["blocks"]:
        for key in ("mix", "rev"):
            if "gap" in b[key]:
                near |= np.any(b[key]["gap"] < GAP_TOL, axis=1)
    return near


def check_stack(cfg, y, samples=None, down_scale=None):
    """Stack output against the oracle with the model's storage rounding (X_revert and block
    outputs in the config dtype).  Samples without near ties: the stated tolerance; samples
    with one: counted and held to a loose bound only."""
    big = cfg.L * sum(cfg.banks(s) * cfg.width(s) * (cfg.ffn(s).hidden + cfg.ffn(s).E * cfg.ffn(s).hidden_e
                                                     + cfg.ffn(s).hidden_s) for s in (0, 1)) * 3 > 2e9
    # weights of the largest workload are drawn bank by bank and dropped (16 GB in bf16)
    res = oracle.run_stack(cfg, samples, down_scale=down_scale, storage=cfg.dtype, cache=not big)
    o = res["Y"]
    near = near_tie_samples(res, o.shape[0])
    keep = ~near
    e = err(cfg.dtype, y[keep], o[keep]) if keep.any() else 0.0
    assert e <= tol(cfg.dtype), (e, int(near.sum()))
    if near.any():
        assert err_bf16(y[near], o[near]) <= 10 * BF16_TOL, err_bf16(y[near], o[near])
    return e, int(near.sum()), o

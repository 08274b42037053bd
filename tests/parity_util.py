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


def err_stored(dtype, y, o):
    """The stated measure applied to a tensor the model stores in its dtype: for bf16, the error beyond
    one unit in the last place of the stored value, max(0, |y - o| - ulp) / rms(o), ulp the larger of
    the two values' spacings.  bf16 keeps 8 significant bits, so one ulp of an element with |v| >= 4
    already exceeds 2e-2 of an output rms near 1; two correct evaluations (fp32 on the GPU, float64 in
    the oracle) may round the same real value to neighbouring bf16 numbers, and deeper blocks carry
    such a difference on through the residual.  fp32 tensors: the plain relative measure."""
    if dtype == "f32":
        return err_f32(y, o)
    allow = np.maximum(ulp(o, dtype), ulp(y, dtype))
    return float(np.max(np.maximum(np.abs(y - o) - allow, 0.0)) / rms(o))


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


# Lines the parity tests report at the end of the run (printed by the terminal summary hook in
# conftest.py): near-tie counts per workload and the worst error per block.
REPORT = []


def force_near_ties(info, gpu_idx):
    """The oracle's own top-k of each row (info: its unforced routing of a sub-layer), with the GPU's
    choice substituted on rows where the two sets differ and the oracle's logit gap z_(k) - z_(k+1) is
    below GAP_TOL: at that gap either set is a valid top-k of the method, so the comparison follows
    the GPU's.  A differing row must still be a valid top-k under the oracle's logits.
    Returns (forced [R, banks, k], rows differing outside near ties, near-tie rows substituted)."""
    own = np.asarray(info["idx"])
    gi = np.asarray(gpu_idx).astype(np.int64)
    k = own.shape[-1]
    differ = np.any(np.sort(own, -1) != np.sort(gi, -1), axis=-1)
    near = info["gap"] < GAP_TOL
    bad = differ & ~near
    sub = differ & near
    z = info["logits"]
    for r, b in zip(*np.nonzero(sub)):
        zk = np.sort(z[r, b])[::-1][k - 1]
        assert np.all(z[r, b][gi[r, b]] >= zk - GAP_TOL), (r, b)
    forced = np.where(sub[..., None], gi, own)
    return forced, int(bad.sum()), int(sub.sum())


def skip_term(cfg, hist, l):
    """The inter-residual term of block l (1-based) of a stack: X_{l-gap} when gap > 0, l % gap == 0
    and l < L, else None."""
    return hist[l - cfg.gap] if (cfg.gap > 0 and l % cfg.gap == 0 and l < cfg.L) else None


def oracle_stack_forced(cfg, X, get, gpu_routes, gains=None):
    """The oracle's stack on X (float64, storage rounding of the workload dtype), block by block.
    Each MoE sub-layer takes the oracle's own top-k except on rows where it is a near tie and the GPU
    chose the other valid set (force_near_ties); gpu_routes[l] = {"mix": idx, "rev": idx} for the MoE
    sub-layers of block l, each the GPU's choices on its own input to that sub-layer.
    Returns the block outputs Y_l and X_revert_l and the routing counts."""
    hist = [X]
    res = {"Y": [], "Xr": [], "bad": 0, "near": 0, "decisions": 0, "gap_mix0": None}
    for l in range(cfg.L):
        extra = skip_term(cfg, hist, l + 1)
        g = gains[l] if gains else (None, None)
        forced = [None, None]
        b = O.block_forward(hist[l], cfg, l, get, g, extra, cfg.dtype, forced=tuple(forced))
        for s, key in ((0, "mix"), (1, "rev")):
            if not cfg.ffn(s).is_moe:
                continue
            info = b[key]           # unforced in this sub-layer: the oracle's own routing
            if l == 0 and s == 0:
                res["gap_mix0"] = info["gap"]
            f, nbad, nsub = force_near_ties(info, gpu_routes[l][key])
            res["bad"] += nbad
            res["near"] += nsub
            res["decisions"] += int(np.prod(info["gap"].shape))
            if nsub:
                forced[s] = f
                b = O.block_forward(hist[l], cfg, l, get, g, extra, cfg.dtype, forced=tuple(forced))
        hist.append(b["Y"])
        res["Y"].append(b["Y"])
        res["Xr"].append(b["Xr"])
    return res


def gpu_stack_chain(cfg, blocks, X, device, gains_on=False):
    """The GPU's stack on the token tensor X (a device tensor of any batch size), block by block
    through tm_stack_step (the step tm_stack_forward repeats), with every block's X_revert and, for
    each MoE sub-layer, tm_route_topk's choices on that sub-layer's own input."""
    import torch
    from token_sparse_moe_b200 import _abi as A
    from token_sparse_moe_b200 import api
    sh = api.config_shape(cfg.with_(B=X.shape[0]))
    hist, Xr, routes = [X], [], []
    for l in range(cfg.L):
        extra = skip_term(cfg, hist, l + 1)
        xr = torch.empty_like(X)
        y = api.stack_step(hist[l], extra, blocks[l], sh, X_revert=xr)
        r = {}
        if cfg.mix.is_moe:
            r["mix"] = api.route_topk(hist[l], A.TM_LAYOUT_MIXED, sh, blocks[l].mix)
        if cfg.rev.is_moe:
            r["rev"] = api.route_topk(xr, A.TM_LAYOUT_ROWS, sh, blocks[l].rev)
        hist.append(y)
        Xr.append(xr)
        routes.append(r)
    api.get_device_error()
    return hist[1:], Xr, routes


def check_stack(cfg, blocks, y, samples=None, down_scale=None, device="cuda:0", label=None):
    """A GPU stack output y (float64 copy of the sampled rows, or of all rows) against the oracle.

    The sampled rows are run again on the GPU as a batch of their own, block by block
    (gpu_stack_chain): samples are independent, so that batch must give y bit for bit, and it
    yields every block's output, X_revert and routing.  The oracle runs the same blocks from the
    same input (oracle_stack_forced), following the GPU only on near-tie rows.  Every sampled row
    of every block (and X_revert) must meet the workload's tolerance beyond the storage rounding
    (err_stored); a routing difference outside a near tie fails.  The counts go to REPORT."""
    import torch
    from token_sparse_moe_b200 import api
    n = cfg.B if samples is None else len(samples)
    assert n > 0
    X = S.make_x(cfg, samples)
    hist, Xr, routes = gpu_stack_chain(cfg, blocks, api.to_device(X, device), device)
    last = to_np(hist[-1])
    assert np.array_equal(last, y), "the sampled rows run alone differ from the stack over the whole batch"
    big = cfg.L * sum(cfg.banks(s) * cfg.width(s) * (cfg.ffn(s).hidden + cfg.ffn(s).E * cfg.ffn(s).hidden_e
                                                     + cfg.ffn(s).hidden_s) for s in (0, 1)) * 3 > 2e9
    # the largest workload's weights (16 GB in bf16) are drawn one layer at a time, in parallel
    import os
    get = oracle.synth_banks(cfg, down_scale, cache="layer" if big else True,
                             workers=min(16, os.cpu_count() or 1))
    gpu_idx = [{k: v["idx"].cpu().numpy() for k, v in r.items()} for r in routes]
    res = oracle_stack_forced(cfg, S.to_f64(X), get, gpu_idx)
    assert res["bad"] == 0, f"{res['bad']} routing decisions differ outside near ties"
    worst, worst_plain, n_ulp = 0.0, 0.0, 0
    for l in range(cfg.L):
        for name, g, o in (("Y", hist[l], res["Y"][l]), ("X_revert", Xr[l], res["Xr"][l])):
            gy = to_np(g)
            e = err_stored(cfg.dtype, gy, o)
            assert e <= tol(cfg.dtype), (label or cfg.name, l + 1, name, e)
            worst = max(worst, e)
            worst_plain = max(worst_plain, err(cfg.dtype, gy, o))
            if cfg.dtype == "bf16":
                n_ulp += int(np.sum(np.abs(gy - o) > 0.75 * ulp(o, "bf16")))
    gpu_near = sum(int((r[k]["gap"] < GAP_TOL).sum().item()) for r in routes for k in r)
    if res["gap_mix0"] is not None:
        # block 1's mixing routers see the same input on both sides: the reported gaps agree
        gg = routes[0]["mix"]["gap"].cpu().numpy().astype(np.float64)
        og = res["gap_mix0"]
        fin = np.isfinite(og)
        assert np.array_equal(np.isfinite(gg), fin)
        assert np.max(np.abs(gg[fin] - og[fin]), initial=0.0) <= 1e-4
    REPORT.append(f"{label or cfg.name}: {n} samples x {cfg.L} blocks (Y and X_revert of each), worst error beyond "
                  f"storage rounding {worst:.2e} (tol {tol(cfg.dtype):g}), plain max|y-o|/rms {worst_plain:.2e}, "
                  f"elements a whole ulp apart {n_ulp}; routing decisions {res['decisions']}, near-tie rows where "
                  f"the GPU took the other valid set {res['near']}, GPU-reported gaps < {GAP_TOL:g}: {gpu_near}")
    return worst, res

"""Float64 CPU oracle of the TokenMixer-Large block / stack forward.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check of the graft entry
point and the CPU-baseline leg of the benchmark may import this module; the
library path never does, and it shares no code, table or constant with the
CUDA kernels.  It is plain NumPy in float64: library matmuls are its only
building block, with no blocking, fusion or reordering beyond the equations.

Sources (two of the pages on TokenMixer-Large):
  [digest]  "TokenMixer-Large: Scaling Up Large Ranking Models in Industrial
            Recommenders" -- paper digest of arXiv 2602.06563, sections 2.3-2.5.
  [readme]  "tokenmixerlarge" README of the TensorFlow/Keras reproduction:
            block diagram and the list of paper-faithful choices.

Readings where the pages are silent or garbled (each one is listed with its
reason in the design notes of the repository):
  * pre-norm sub-layers  out = FFN(RMSNorm(in)) + residual  ([readme] block
    diagram; [digest] 2.3.3, which moves the norm in front of the FFN), not the post-norm
    form printed in Eq. 8/12/16;
  * Revert is the exact inverse of Mix (Eq. 13 prints the same head index twice);
  * Swish is SiLU (beta = 1);
  * RMSNorm: x / sqrt(mean(x^2) + eps) * gain, eps inside the square root;
  * routing: softmax over all E logits, top-k by probability with ties to the
    lower expert index, gate = alpha * p (no renormalisation after top-k),
    E routed experts plus one always-on shared expert;
  * inter-residual: after block l, X_l += X_{l-gap} when l % gap == 0 and l < L;
  * storage (optional): a model whose dtype is bf16 (or fp32) keeps the tensors it hands
    from one sub-layer to the next in that dtype -- X_revert, and each block output after
    its inter-residual.  With storage="bf16" / "f32" the oracle rounds exactly those
    tensors to nearest-even in that format; every other step stays float64.  Routing
    decisions in deeper layers then see the same stored inputs the model defines.
"""
from __future__ import annotations

from typing import Callable, Dict, List, Optional

import numpy as np

Weights = Dict[str, np.ndarray]


# ------------------------------------------------------------------ Mix / Revert
def mix(X: np.ndarray, H: int) -> np.ndarray:
    """[..., T, D] -> [..., H, T*D/H].  [digest] 2.3.1, Eq. 9-11.

    Eq. 9 splits token t into H heads x_t^(h) of width D/H; Eq. 10 concatenates
    head h over the tokens in token order; Eq. 11 stacks the H rows.
    """
    *lead, T, D = X.shape
    assert D % H == 0
    dh = D // H
    out = np.empty((*lead, H, T * dh), dtype=X.dtype)
    for h in range(H):
        for t in range(T):
            out[..., h, t * dh:(t + 1) * dh] = X[..., t, h * dh:(h + 1) * dh]
    return out


def revert(Hn: np.ndarray, T: int) -> np.ndarray:
    """[..., H, T*dh] -> [..., T, H*dh].  [digest] 2.3.1, Eq. 13-15.

    Eq. 13 splits row h into T pieces of width dh (piece t belongs to token t),
    Eq. 14 concatenates, for token t, its pieces over the heads in head order,
    Eq. 15 stacks the T tokens.
    """
    *lead, H, W = Hn.shape
    assert W % T == 0
    dh = W // T
    out = np.empty((*lead, T, H * dh), dtype=Hn.dtype)
    for t in range(T):
        for h in range(H):
            out[..., t, h * dh:(h + 1) * dh] = Hn[..., h, t * dh:(t + 1) * dh]
    return out


# ------------------------------------------------------------------ norm / FFN
def rmsnorm(x: np.ndarray, eps: float, gain: Optional[np.ndarray] = None) -> np.ndarray:
    """RMSNorm over the last axis, no mean-centering.  [digest] 2.3.3; [readme] (RMSNorm, no bias terms)."""
    r = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return r if gain is None else r * gain


def silu(z: np.ndarray) -> np.ndarray:
    """Swish with beta = 1.  [digest] 2.3.2, Eq. 17.

    For z below about -709, exp(-z) overflows to inf and z / inf gives the limit 0; the overflow is
    expected there and not reported."""
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def swiglu(n: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray, w_down: np.ndarray) -> np.ndarray:
    """FC_down(Swish(FC_gate n) * FC_up n), weights in [out, in] layout, no bias.

    [digest] 2.3.2, Eq. 17-18 (bias terms dropped: the [readme] reproduction leaves them off by default).
    n: [R, W]; w_gate, w_up: [F, W]; w_down: [W, F]  ->  [R, W].
    """
    g = n @ w_gate.T
    u = n @ w_up.T
    return (silu(g) * u) @ w_down.T


def softmax(z: np.ndarray) -> np.ndarray:
    e = np.exp(z - np.max(z, axis=-1, keepdims=True))
    return e / np.sum(e, axis=-1, keepdims=True)


def topk(p: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest entries of each row, largest first; ties go to the lower index."""
    order = np.argsort(-p, axis=-1, kind="stable")
    return order[..., :k]


def route(n: np.ndarray, w_router: np.ndarray, k: int) -> Dict[str, np.ndarray]:
    """Router of one bank: fp64 logits, softmax, top-k.  [digest] 2.4.1 Eq. 19, 2.4.3.

    Returns logits z [R, E], probabilities p [R, E], chosen experts idx [R, k]
    and the logit gap z_(k) - z_(k+1) between the k-th and (k+1)-th largest
    logits (inf when k == E), which tells how close a row is to a tie.
    """
    z = n @ w_router.T
    p = softmax(z)
    idx = topk(p, k)
    zs = -np.sort(-z, axis=-1)
    gap = np.full(z.shape[0], np.inf) if k >= z.shape[1] else zs[:, k - 1] - zs[:, k]
    return {"logits": z, "p": p, "idx": idx, "gap": gap}


def sp_moe(n: np.ndarray, bw: Weights, k: int, alpha: float,
           forced_idx: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """Sparse-Pertoken MoE of one bank on rows n [R, W].  [digest] 2.4, Eq. 19-21.

    out = alpha * sum_{e in topk} p_e * Expert_e(n) + SharedExpert(n), every
    expert a SwiGLU of its own (Eq. 19), the shared expert always on (Eq. 20),
    alpha the gate-value scale (Eq. 21).  Only the chosen experts are evaluated.

    Teacher-forced routing: with forced_idx [R, k] the experts of each row are those given
    (for instance another implementation's choices) instead of the top-k; the gates are still
    alpha * p_e of the oracle's own softmax, so a row whose top-k is a near tie is compared
    on the same experts everywhere else in the computation.
    """
    r = route(n, bw["w_router"], k)
    if forced_idx is not None:
        forced_idx = np.asarray(forced_idx)
        assert forced_idx.shape == r["idx"].shape, (forced_idx.shape, r["idx"].shape)
        assert np.all((forced_idx >= 0) & (forced_idx < r["p"].shape[1]))
        assert all(len(set(row)) == k for row in forced_idx.tolist()), "forced experts repeat within a row"
        r["idx"] = forced_idx
    idx = r["idx"]
    R, E = r["p"].shape
    out = np.zeros_like(n)
    for e in range(E):
        rows = np.nonzero(np.any(idx == e, axis=1))[0]
        if rows.size == 0:
            continue
        ye = swiglu(n[rows], bw["we_gate"][e], bw["we_up"][e], bw["we_down"][e])
        out[rows] += alpha * r["p"][rows, e][:, None] * ye
    if "ws_gate" in bw:
        out += swiglu(n, bw["ws_gate"], bw["ws_up"], bw["ws_down"])
    r["out"] = out
    return r


def sp_moe_dense_masked(n: np.ndarray, bw: Weights, k: int, alpha: float) -> np.ndarray:
    """The "dense compute, sparse output" form of the same MoE ([readme], documented
    deviations): every expert runs on every row, then unchosen outputs are masked.
    Must equal sp_moe; used only as a cross-check."""
    r = route(n, bw["w_router"], k)
    E = r["p"].shape[1]
    mask = np.zeros_like(r["p"])
    np.put_along_axis(mask, r["idx"], 1.0, axis=1)
    out = np.zeros_like(n)
    for e in range(E):
        out += alpha * (mask[:, e] * r["p"][:, e])[:, None] * swiglu(n, bw["we_gate"][e], bw["we_up"][e], bw["we_down"][e])
    if "ws_gate" in bw:
        out += swiglu(n, bw["ws_gate"], bw["ws_up"], bw["ws_down"])
    return out


# ------------------------------------------------------------------ storage rounding
def round_bf16(x: np.ndarray) -> np.ndarray:
    """Nearest-even bf16 value (8 significant bits) of each float64, computed in float64."""
    m, e = np.frexp(x)                     # x = m * 2**e, 0.5 <= |m| < 1
    q = np.ldexp(1.0, e - 8)               # spacing of 8-significant-bit values at |x|
    r = np.round(x / q) * q                # np.round: half to even
    return np.where(x == 0, x, r)


def storage_round(storage):
    """Rounding applied to the tensors a model of this dtype stores between sub-layers."""
    if storage in (None, "f64"):
        return lambda a: a
    if storage == "bf16":
        return round_bf16
    if storage == "f32":
        return lambda a: a.astype(np.float32).astype(np.float64)
    raise ValueError(storage)


# ------------------------------------------------------------------ sub-layer / block / stack
def sublayer(rows: np.ndarray, bank_w: Callable[[int], Weights], spec, eps: float,
             gain: Optional[np.ndarray] = None, forced_idx: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """FFN(RMSNorm(row)) for every row of every bank, without the residual.

    rows: [R, banks, W].  Bank j owns its own weights (parameter isolation,
    [digest] 2.3.2 and 2.4.2, per-token weights).  Returns out [R, banks, W] and, for
    MoE, the routing of each bank.  forced_idx [R, banks, k] (MoE only): teacher-forced
    routing, see sp_moe.
    """
    R, banks, W = rows.shape
    out = np.empty_like(rows)
    info = {"idx": [], "p": [], "logits": [], "gap": []}
    for j in range(banks):
        n = rmsnorm(rows[:, j, :], eps, gain)
        bw = bank_w(j)
        if spec.is_moe:
            r = sp_moe(n, bw, spec.k, spec.alpha, None if forced_idx is None else forced_idx[:, j, :])
            out[:, j, :] = r["out"]
            for key in info:
                info[key].append(r[key])
        else:
            out[:, j, :] = swiglu(n, bw["w_gate"], bw["w_up"], bw["w_down"])
    res = {"out": out}
    if spec.is_moe:
        for key in info:
            res[key] = np.stack(info[key], axis=1)   # [R, banks, ...]
    return res


def block_forward(X: np.ndarray, cfg, layer: int, bank_w: Callable[[int, int, int], Weights],
                  gains=(None, None), extra: Optional[np.ndarray] = None, storage=None,
                  forced=(None, None)) -> Dict[str, np.ndarray]:
    """One TokenMixer-Large block on X [R, T, D].  [readme] block diagram; [digest] Eq. 9-16.

        H      = Mix(X)
        H_next = FFN_mix(Norm(H)) + H
        X_rev  = Revert(H_next)
        X_next = FFN_rev(Norm(X_rev)) + X  (+ extra)   (residual to the block input; extra is
                                                         the inter-residual term of the stack)
    X_rev and X_next are the stored tensors that `storage` rounds.  forced: teacher-forced
    routing [R, banks, k] per sub-layer (MoE sub-layers; see sp_moe), or None.
    """
    rnd = storage_round(storage)
    Hm = mix(X, cfg.H)
    s_mix = sublayer(Hm, lambda j: bank_w(layer, 0, j), cfg.mix, cfg.eps, gains[0], forced[0])
    Hn = s_mix["out"] + Hm
    Xr = rnd(revert(Hn, cfg.T))
    s_rev = sublayer(Xr, lambda j: bank_w(layer, 1, j), cfg.rev, cfg.eps, gains[1], forced[1])
    Xn = s_rev["out"] + X
    if extra is not None:
        Xn = Xn + extra
    return {"Hm": Hm, "Hn": Hn, "Xr": Xr, "Y": rnd(Xn), "mix": s_mix, "rev": s_rev}


def stack_forward(X: np.ndarray, cfg, bank_w: Callable[[int, int, int], Weights],
                  gains: Optional[List] = None, keep: bool = False, storage=None) -> Dict[str, object]:
    """L blocks with the inter-residual.  [digest] 2.3.4; [readme] (inter-residual every 2 layers,
    none after the final one):  X_l = Block_l(X_{l-1}); X_l += X_{l-gap} when
    gap > 0, l % gap == 0 and l < L (layers counted from 1)."""
    hist = [X]
    blocks = []
    for l in range(1, cfg.L + 1):
        extra = hist[l - cfg.gap] if (cfg.gap > 0 and l % cfg.gap == 0 and l < cfg.L) else None
        b = block_forward(hist[-1], cfg, l - 1, bank_w, gains[l - 1] if gains else (None, None), extra, storage)
        Xl = b["Y"]
        hist.append(Xl)
        blocks.append(b if keep else {"mix": b["mix"], "rev": b["rev"]})
    return {"Y": hist[-1], "hist": hist, "blocks": blocks}


# ------------------------------------------------------------------ tokenizer stub
def tokenize(groups: np.ndarray, w_group: np.ndarray, w_global: np.ndarray) -> np.ndarray:
    """Group-wise tokens plus a global token.  [digest] 2.2.1-2.2.2, Eq. 2-4.

    Each group MLP is read as one bias-free linear layer (the pages leave its depth open).
    groups [B, G, dg]; w_group [G, D, dg]; w_global [D, G*dg]  ->  X [B, G+1, D] with
    the global token first (Eq. 4 lists X_G before the group tokens).
    """
    B, G, dg = groups.shape
    D = w_group.shape[1]
    X = np.empty((B, G + 1, D))
    X[:, 0, :] = groups.reshape(B, G * dg) @ w_global.T           # Eq. 3
    for i in range(G):
        X[:, i + 1, :] = groups[:, i, :] @ w_group[i].T            # Eq. 2
    return X


# ------------------------------------------------------------------ model head and end-to-end scoring
def head(X: np.ndarray, w_head: np.ndarray) -> np.ndarray:
    """Scoring head of the model.  [readme] block diagram: mean-pool over tokens, then a
    projection head to one logit per sample (bias off, as the reproduction's default).
    X [B, T, D], w_head [D]  ->  logits [B]."""
    return X.mean(axis=1) @ w_head


def model_forward(groups: np.ndarray, w_group: np.ndarray, w_global: np.ndarray, cfg,
                  bank_w: Callable[[int, int, int], Weights], w_head: np.ndarray, storage=None) -> Dict[str, np.ndarray]:
    """End-to-end scoring of a batch: tokenizer (Eq. 2-4) -> blocks with the inter-residual ->
    head.  With `storage` the token tensor is stored once in the model dtype before the stack,
    as the blocks' stored tensors are."""
    rnd = storage_round(storage)
    X = rnd(tokenize(groups, w_group, w_global))
    st = stack_forward(X, cfg, bank_w, storage=storage)
    return {"X": X, "Y": st["Y"], "logits": head(st["Y"], w_head)}

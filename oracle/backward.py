"""Float64 gradients of the TokenMixer-Large sub-layers (dense and Sparse-Pertoken MoE), block and
stack: the oracle of the training path.

TEST INFRASTRUCTURE ONLY, like the rest of this package: imported by the tests, the smoke
check and the benchmark's CPU leg, never by the library, and sharing no code or table with it.

Source: the pages train the model ([digest] "TokenMixer-Large: Scaling Up Large Ranking Models
in Industrial Recommenders", section 2.5.2: bf16 training; [readme] "tokenmixerlarge", its
training flags) but print no backward pass.  The gradient is therefore the exact derivative of
the forward in oracle.tokenmixer, written out by the chain rule with the forward's own names:

    r   = 1 / sqrt(mean(x^2) + eps),  xh = x * r,  n = xh * gain
    g   = n Wg^T,  u = n Wu^T,  h = silu(g) * u,  y = h Wd^T     (the FFN term of a sub-layer)

    dWd = dy^T h,   dh = dy Wd
    dg  = dh * u * silu'(g),   silu'(g) = s * (1 + g * (1 - s)),  s = sigmoid(g)
    du  = dh * silu(g)
    dWg = dg^T n,   dWu = du^T n,   dn = dg Wg + du Wu
    dgain = sum over rows of dn * xh,   dxh = dn * gain
    dx  = r * (dxh - xh * mean(dxh * xh))                         (RMSNorm, no centring)

The MoE sub-layer ([digest] 2.4, Eq. 19-21) holds the chosen experts fixed (the top-k set is
piecewise constant in the input) and differentiates the gates alpha * p_e through the softmax into
the router, the chosen experts and the shared expert (moe_ffn_backward).

The block (Mix -> mixing sub-layer with its residual -> Revert -> reverting sub-layer with the
residual to the block input) is differentiated through its residuals; Mix and Revert are
permutations, each the other's adjoint.
"""
from __future__ import annotations

from typing import Callable, Dict, List, Optional

import numpy as np

from .tokenmixer import Weights, mix, revert, route, silu, stack_forward, storage_round, sublayer, swiglu


def _sigmoid(z: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-z))


def swiglu_ffn_backward(x: np.ndarray, dy: np.ndarray, bw: Weights, eps: float,
                        gain: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """Gradients of y = SwiGLU(RMSNorm(x)) (one bank, no residual) for the upstream gradient dy.

    x, dy: [R, W]; bw: w_gate, w_up [F, W], w_down [W, F].  Returns dx [R, W], dw_gate,
    dw_up [F, W], dw_down [W, F] and dgain [W] (None without a gain).
    """
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    xh = x * r
    n = xh if gain is None else xh * gain
    g = n @ bw["w_gate"].T
    u = n @ bw["w_up"].T
    s = _sigmoid(g)
    h = g * s * u
    dw_down = dy.T @ h
    dh = dy @ bw["w_down"]
    dg = dh * u * s * (1.0 + g * (1.0 - s))
    du = dh * silu(g)
    dw_gate = dg.T @ n
    dw_up = du.T @ n
    dn = dg @ bw["w_gate"] + du @ bw["w_up"]
    dgain = None if gain is None else np.sum(dn * xh, axis=0)
    dxh = dn if gain is None else dn * gain
    dx = r * (dxh - xh * np.mean(dxh * xh, axis=-1, keepdims=True))
    return {"dx": dx, "dw_gate": dw_gate, "dw_up": dw_up, "dw_down": dw_down, "dgain": dgain}


def swiglu_input_backward(n: np.ndarray, dy: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray,
                          w_down: np.ndarray) -> Dict[str, np.ndarray]:
    """Gradients of y = SwiGLU(n) = (silu(n Wg^T) * (n Wu^T)) Wd^T with respect to its input n and
    its three weights (no normalisation: an expert of the MoE sees the normalised row)."""
    g = n @ w_gate.T
    u = n @ w_up.T
    s = _sigmoid(g)
    dh = dy @ w_down
    dg = dh * u * s * (1.0 + g * (1.0 - s))
    du = dh * silu(g)
    return {"dn": dg @ w_gate + du @ w_up, "dw_gate": dg.T @ n, "dw_up": du.T @ n,
            "dw_down": dy.T @ (g * s * u)}


def rmsnorm_backward(x: np.ndarray, dn: np.ndarray, eps: float, gain: Optional[np.ndarray] = None):
    """The gradient at x of n = RMSNorm(x) * gain for the upstream gradient dn, and dgain (None
    without a gain): dx = r (dxh - xh mean(dxh xh)), xh = x r, dxh = dn * gain."""
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    xh = x * r
    dgain = None if gain is None else np.sum(dn * xh, axis=0)
    dxh = dn if gain is None else dn * gain
    return r * (dxh - xh * np.mean(dxh * xh, axis=-1, keepdims=True)), dgain


def moe_ffn_backward(x: np.ndarray, dy: np.ndarray, bw: Weights, k: int, alpha: float, eps: float,
                     gain: Optional[np.ndarray] = None, forced_idx: Optional[np.ndarray] = None
                     ) -> Dict[str, np.ndarray]:
    """Gradients of y = SpMoE(RMSNorm(x) * gain) of one bank (no residual; the forward is
    oracle.tokenmixer.sp_moe: y = alpha * sum_{chosen e} p_e Expert_e(n) + Shared(n), p the softmax of
    the router logits z = n Wr^T over all E experts).

    The chosen set is piecewise constant in the input (it changes only where two logits tie), so
    the derivative holds it fixed and differentiates the rest:
        dp_e   = alpha * <dy, Expert_e(n)> for a chosen e, 0 otherwise
        dz     = p * (dp - sum_e p_e dp_e)                          (softmax)
        dWr    = dz^T n
        dn     = dz Wr + sum_{chosen e} dExpert_e(n)^T (alpha p_e dy) + dShared(n)^T dy
        dx     = RMSNorm backward of dn
    Every expert's weight gradient sums over the rows that chose it (zero for an expert no row
    chose); forced_idx [R, k] fixes the chosen experts as in sp_moe's teacher-forced mode.
    Returns dx, dgain, dw_router [E, W], dwe_gate / dwe_up [E, Fe, W], dwe_down [E, W, Fe], the
    shared expert's dws_gate / dws_up / dws_down (when present) and the chosen experts idx.
    """
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    n = x * r if gain is None else x * r * gain
    rt = route(n, bw["w_router"], k)
    idx = rt["idx"] if forced_idx is None else np.asarray(forced_idx)
    p = rt["p"]
    R, E = p.shape
    dn = np.zeros_like(n)
    dp = np.zeros_like(p)
    out = {"dwe_gate": np.zeros_like(bw["we_gate"]), "dwe_up": np.zeros_like(bw["we_up"]),
           "dwe_down": np.zeros_like(bw["we_down"])}
    for e in range(E):
        rows = np.nonzero(np.any(idx == e, axis=1))[0]
        if rows.size == 0:
            continue
        ne, dye = n[rows], dy[rows]
        dp[rows, e] = alpha * np.sum(dye * swiglu(ne, bw["we_gate"][e], bw["we_up"][e], bw["we_down"][e]), axis=1)
        ge = swiglu_input_backward(ne, alpha * p[rows, e][:, None] * dye, bw["we_gate"][e], bw["we_up"][e],
                                   bw["we_down"][e])
        dn[rows] += ge["dn"]
        out["dwe_gate"][e], out["dwe_up"][e], out["dwe_down"][e] = ge["dw_gate"], ge["dw_up"], ge["dw_down"]
    dz = p * (dp - np.sum(p * dp, axis=1, keepdims=True))
    out["dw_router"] = dz.T @ n
    dn += dz @ bw["w_router"]
    if "ws_gate" in bw:
        gs = swiglu_input_backward(n, dy, bw["ws_gate"], bw["ws_up"], bw["ws_down"])
        dn += gs["dn"]
        out["dws_gate"], out["dws_up"], out["dws_down"] = gs["dw_gate"], gs["dw_up"], gs["dw_down"]
    out["dx"], out["dgain"] = rmsnorm_backward(x, dn, eps, gain)
    out["idx"] = idx
    return out


MOE_GRADS = ("dw_router", "dwe_gate", "dwe_up", "dwe_down", "dws_gate", "dws_up", "dws_down")


def sublayer_backward(rows: np.ndarray, dy: np.ndarray, bank_w: Callable[[int], Weights], spec, eps: float,
                      gain: Optional[np.ndarray] = None) -> Dict[str, object]:
    """Gradients of the sub-layer's FFN term for every bank (no residual).

    rows, dy: [R, banks, W].  Returns dx [R, banks, W], the per-bank weight gradients as lists
    (dense: dw_gate, dw_up, dw_down; MoE: the keys of MOE_GRADS, see moe_ffn_backward) and dgain
    (the sum over banks: one gain vector is shared).
    """
    R, banks, W = rows.shape
    if spec.is_moe:
        dx = np.empty_like(rows)
        out = {key: [] for key in MOE_GRADS}
        dgain = None if gain is None else np.zeros(W)
        for j in range(banks):
            gj = moe_ffn_backward(rows[:, j, :], dy[:, j, :], bank_w(j), spec.k, spec.alpha, eps, gain)
            dx[:, j, :] = gj["dx"]
            for key in out:
                out[key].append(gj.get(key))
            if gain is not None:
                dgain = dgain + gj["dgain"]
        return {"dx": dx, "dgain": dgain, **out}
    dx = np.empty_like(rows)
    out = {"dw_gate": [], "dw_up": [], "dw_down": []}
    dgain = None if gain is None else np.zeros(W)
    for j in range(banks):
        gj = swiglu_ffn_backward(rows[:, j, :], dy[:, j, :], bank_w(j), eps, gain)
        dx[:, j, :] = gj["dx"]
        for key in out:
            out[key].append(gj[key])
        if gain is not None:
            dgain = dgain + gj["dgain"]
    return {"dx": dx, "dgain": dgain, **out}


def block_backward(X: np.ndarray, cfg, layer: int, bank_w: Callable[[int, int, int], Weights], dY: np.ndarray,
                   gains=(None, None), storage=None) -> Dict[str, object]:
    """Gradients of one dense block Y = Block(X) for the upstream gradient dY [R, T, D].

    The forward is recomputed as oracle.tokenmixer.block_forward computes it (X_rev rounded by
    `storage`, the stored tensor the reverting sub-layer reads); then

        dX_rev = d FFN_rev(Norm(X_rev)) / d X_rev applied to dY
        dH_next = Mix(dX_rev)                          (the adjoint of Revert)
        dH     = d FFN_mix(Norm(H)) / d H applied to dH_next + dH_next
        dX     = dY + Revert(dH)                       (the adjoint of Mix)

    Returns dX, dX_rev and the weight gradients of both sub-layers ("mix", "rev").
    """
    rnd = storage_round(storage)
    Hm = mix(X, cfg.H)
    Hn = sublayer(Hm, lambda j: bank_w(layer, 0, j), cfg.mix, cfg.eps, gains[0])["out"] + Hm
    Xr = rnd(revert(Hn, cfg.T))
    g_rev = sublayer_backward(Xr, dY, lambda j: bank_w(layer, 1, j), cfg.rev, cfg.eps, gains[1])
    dXr = g_rev["dx"]
    dHn = mix(dXr, cfg.H)
    g_mix = sublayer_backward(Hm, dHn, lambda j: bank_w(layer, 0, j), cfg.mix, cfg.eps, gains[0])
    dHm = g_mix["dx"] + dHn
    dX = dY + revert(dHm, cfg.T)
    return {"dX": dX, "dXr": dXr, "Xr": Xr, "mix": g_mix, "rev": g_rev}


def stack_backward(X: np.ndarray, cfg, bank_w: Callable[[int, int, int], Weights], dY: np.ndarray,
                   gains: Optional[List] = None, storage=None) -> Dict[str, object]:
    """Gradients of the dense stack (blocks 1..L, inter-residual X_l += X_{l-gap} after block l when
    gap > 0, l % gap == 0 and l < L) for the upstream gradient dY of its output.

    Each block's input is recomputed by the forward; the inter-residual hands block l's output
    gradient on to X_{l-gap} as well.  Returns dX and the per-layer block gradients.
    """
    L, gap = cfg.L, cfg.gap
    gains = gains or [(None, None)] * L
    xs = stack_forward(X, cfg, bank_w, gains, storage=storage)["hist"]   # xs[l] = X_l, input of block l + 1
    grads = [None] * L
    dx = [np.zeros_like(X) for _ in range(L + 1)]
    dx[L] = dY
    for l in range(L, 0, -1):
        if gap > 0 and l % gap == 0 and l < L:
            dx[l - gap] = dx[l - gap] + dx[l]
        g = block_backward(xs[l - 1], cfg, l - 1, bank_w, dx[l], gains[l - 1], storage)
        grads[l - 1] = g
        dx[l - 1] = dx[l - 1] + g["dX"]
    return {"dX": dx[0], "blocks": grads}

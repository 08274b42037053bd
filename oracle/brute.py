"""Brute-force scalar restatement of the TokenMixer-Large block, for tiny inputs.

TEST INFRASTRUCTURE ONLY (see oracle/tokenmixer.py).  A second, independent
statement of the same equations, in plain Python scalars and nested loops with
the math module only: no NumPy, no matmul, no shared helper with the vectorised
oracle.  It exists to pin that oracle: a transposed operand, a wrong index or a
dropped term in either one makes the two disagree on tiny inputs.

Shapes use nested lists: X[b][t][d]; dense bank weights w_gate[j][f][i],
w_up[j][f][i], w_down[j][i][f]; MoE bank weights w_router[j][e][i],
we_gate[j][e][f][i], we_up[j][e][f][i], we_down[j][e][i][f], ws_gate[j][f][i],
ws_up[j][f][i], ws_down[j][i][f].
"""
from __future__ import annotations

import math


def _mixed_element(X, b, h, c, dh):
    # row h of sample b, column c = t*dh + j holds X[b][t][h*dh + j]  (Eq. 9-11)
    t, j = divmod(c, dh)
    return X[b][t][h * dh + j]


def _norm_row(row, eps, gain):
    ms = 0.0
    for v in row:
        ms += v * v
    ms /= len(row)
    s = 1.0 / math.sqrt(ms + eps)
    return [row[i] * s * (1.0 if gain is None else gain[i]) for i in range(len(row))]


def _swiglu_row(n, wg, wu, wd):
    F, W = len(wg), len(n)
    hid = []
    for f in range(F):
        g = 0.0
        u = 0.0
        for i in range(W):
            g += wg[f][i] * n[i]
            u += wu[f][i] * n[i]
        hid.append(g / (1.0 + math.exp(-g)) * u)
    out = []
    for i in range(W):
        acc = 0.0
        for f in range(F):
            acc += wd[i][f] * hid[f]
        out.append(acc)
    return out


def _moe_row(n, bw, j, k, alpha):
    E = len(bw["w_router"][j])
    z = []
    for e in range(E):
        acc = 0.0
        for i in range(len(n)):
            acc += bw["w_router"][j][e][i] * n[i]
        z.append(acc)
    m = max(z)
    ex = [math.exp(v - m) for v in z]
    tot = sum(ex)
    p = [v / tot for v in ex]
    chosen = []
    for _ in range(k):                       # repeated arg-max; first index wins ties
        best = -1
        for e in range(E):
            if e in chosen:
                continue
            if best < 0 or p[e] > p[best]:
                best = e
        chosen.append(best)
    out = [0.0] * len(n)
    for e in chosen:
        y = _swiglu_row(n, bw["we_gate"][j][e], bw["we_up"][j][e], bw["we_down"][j][e])
        for i in range(len(n)):
            out[i] += alpha * p[e] * y[i]
    if "ws_gate" in bw:
        y = _swiglu_row(n, bw["ws_gate"][j], bw["ws_up"][j], bw["ws_down"][j])
        for i in range(len(n)):
            out[i] += y[i]
    return out, chosen


def _ffn_row(n, bw, j, spec):
    if spec.is_moe:
        return _moe_row(n, bw, j, spec.k, spec.alpha)[0]
    return _swiglu_row(n, bw["w_gate"][j], bw["w_up"][j], bw["w_down"][j])


def block(X, T, D, H, eps, spec_mix, w_mix, spec_rev, w_rev, gain_mix=None, gain_rev=None, rnd=None, extra=None):
    """One block on nested-list X[b][t][d]; returns X_next as nested lists.  `rnd` (a scalar
    rounding function) is applied to the stored X_revert and to the block output after
    `extra` (the inter-residual term) is added."""
    rnd = rnd or (lambda v: v)
    B = len(X)
    dh = D // H
    W = T * dh
    # mixing sub-layer: H_next[b][h][c] = FFN_h(Norm(row))[c] + row[c]
    Hn = []
    for b in range(B):
        rows = []
        for h in range(H):
            row = [_mixed_element(X, b, h, c, dh) for c in range(W)]
            y = _ffn_row(_norm_row(row, eps, gain_mix), w_mix, h, spec_mix)
            rows.append([y[c] + row[c] for c in range(W)])
        Hn.append(rows)
    # revert: X_rev[b][t][h*dh + j] = H_next[b][h][t*dh + j]  (Eq. 13-15)
    Xr = [[[rnd(Hn[b][d // dh][t * dh + d % dh]) for d in range(D)] for t in range(T)] for b in range(B)]
    # reverting sub-layer, residual to the block input X
    out = []
    for b in range(B):
        toks = []
        for t in range(T):
            y = _ffn_row(_norm_row(Xr[b][t], eps, gain_rev), w_rev, t, spec_rev)
            toks.append([rnd(y[d] + X[b][t][d] + (extra[b][t][d] if extra is not None else 0.0)) for d in range(D)])
        out.append(toks)
    return out


def stack(X, T, D, H, eps, L, gap, specs, weights, rnd=None):
    """specs[l] = (spec_mix, spec_rev), weights[l] = (w_mix, w_rev); inter-residual per the
    reading X_l += X_{l-gap} when l % gap == 0 and l < L."""
    hist = [X]
    for l in range(1, L + 1):
        (sm, sr), (wm, wr) = specs[l - 1], weights[l - 1]
        extra = hist[l - gap] if (gap > 0 and l % gap == 0 and l < L) else None
        Y = block(hist[-1], T, D, H, eps, sm, wm, sr, wr, rnd=rnd, extra=extra)
        hist.append(Y)
    return hist[-1]


def round_bf16(v):
    """Nearest-even value with 8 significant bits, by scalar arithmetic."""
    if v == 0.0 or not math.isfinite(v):
        return v
    m, e = math.frexp(v)
    q = math.ldexp(1.0, e - 8)
    n = v / q
    f = math.floor(n)
    d = n - f
    if d > 0.5 or (d == 0.5 and f % 2 == 1):
        f += 1
    return f * q


def tokenize(groups, w_group, w_global):
    """Scalar loops: X[b][0][d] = sum_{i,c} w_global[d][i*dg + c] * groups[b][i][c];
    X[b][i+1][d] = sum_c w_group[i][d][c] * groups[b][i][c]."""
    B, G, dg = len(groups), len(groups[0]), len(groups[0][0])
    D = len(w_group[0])
    X = []
    for b in range(B):
        toks = [[sum(w_global[d][i * dg + c] * groups[b][i][c] for i in range(G) for c in range(dg)) for d in range(D)]]
        for i in range(G):
            toks.append([sum(w_group[i][d][c] * groups[b][i][c] for c in range(dg)) for d in range(D)])
        X.append(toks)
    return X

"""FP8 E4M3 serving path of the per-token FFNs (dense SwiGLU banks and Sparse-Pertoken MoE banks):
the float64 oracle.

TEST INFRASTRUCTURE ONLY, like the rest of this package: imported by the tests, the smoke
check and the benchmark's CPU leg, never by the library, and sharing no code or table with it.

Source: [digest] "TokenMixer-Large: Scaling Up Large Ranking Models in Industrial
Recommenders", section 2.5.2 (FP8 quantization): serving uses FP8 E4M3 post-training
quantization of a model trained in bf16.  The page names the format only; the readings here
(each one also listed in the repository's design notes):
  * E4M3 is the 8-bit format with 1 sign bit, 4 exponent bits of bias 7 and 3 mantissa bits:
    normal values 2^(e-7) * (1 + m/8) for exponent fields e = 1..15, subnormals m * 2^-9 for
    e = 0, largest finite 448 (the all-ones pattern S.1111.111 is NaN; there are no
    infinities).  Conversion rounds to nearest with ties to even and saturates at +-448.
  * Scales are powers of two: for values with largest magnitude m > 0 the scale is 2^e with e
    the smallest integer such that m * 2^-e <= 448 (m = f * 2^x with f in [0.5, 1) gives
    e = x - 9 when f <= 0.875, else x - 8); 1 when m = 0.  Then v * 2^-e is exact and the only
    rounding is E4M3's own; the largest value lands in (224, 448].  E4M3 is a floating-point
    format, so its 3-bit relative precision does not depend on the scale; a power-of-two scale
    moves only the underflow threshold, by less than one binade.
  * Weights: the gate and up projections of each bank (with the RMSNorm gain folded in and
    rounded to bf16 first, as the bf16 path stores them) are quantized per matrix, one scale per
    bank: q = E4M3(w * 2^-e).  Every value inside E4M3's normal range (2^-6 .. 448 times the
    scale) keeps a 3-bit mantissa whatever the scale, so per-row scales would change nothing for
    rows whose magnitudes sit within that 2^15 range of the matrix maximum, as these projections'
    rows do.
  * Activations: every sub-layer row x (width W, the input of the RMSNorm) is quantized on its
    own: q_a = E4M3(x * 2^-e_a), s_a = 2^e_a.
  * GEMM1 runs on the quantized operands: gate_n = (q_a . q_gate_n) * s_a * s_gate / rms(x),
    up_n likewise, with rms taken over the unquantized row exactly as in the bf16 path.  The
    SwiGLU, the down projection and the residual are those of the bf16 path (the down
    projection keeps its bf16 weights): GEMM1 carries two thirds of the FFN's flops.
  * MoE banks: every expert (the k routed ones a row reaches and the shared one) is such an FFN,
    its gate and up matrices quantized with one scale each (per (bank, expert)); a row is
    quantized once for all of them; the router is not quantized, so the routing (top-k, gates
    alpha * p) is the bf16 path's.
"""
from __future__ import annotations

from typing import Callable, Dict, Optional, Tuple

import numpy as np

from .tokenmixer import mix, revert, rmsnorm, round_bf16, route, silu, storage_round

E4M3_MAX = 448.0


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """fp32 values -> E4M3 codes (uint8), nearest with ties to even, saturating at +-448.

    Rounding is done on |v| against the step of its binade: 2^(e-3) for normal values with
    2^e <= |v| < 2^(e+1), e >= -6, and 2^-9 below 2^-6 (the subnormal spacing, which equals
    the step of the lowest normal binade).  Codes are monotonic in |v|, so a magnitude that
    rounds up to the next binade gets the right code from the same formula.
    """
    v = np.asarray(v, dtype=np.float32).astype(np.float64)
    if np.isnan(v).any():
        raise ValueError("NaN has no place in the quantized operands")
    sign = np.signbit(v)
    a = np.minimum(np.abs(v), E4M3_MAX)
    _, ex = np.frexp(a)                                   # a = f * 2^ex, f in [0.5, 1)
    e = np.maximum(ex - 1, -6)                            # binade exponent, floored at the lowest normal
    step = np.ldexp(1.0, e - 3)
    q = np.rint(a / step) * step                          # round half to even on the step grid
    q = np.minimum(q, E4M3_MAX)
    # encode the (exactly representable) magnitude q
    _, qex = np.frexp(q)
    qe = qex - 1
    normal = q >= 2.0 ** -6
    exp_field = np.where(normal, qe + 7, 0)
    mant = np.where(normal, q / np.ldexp(1.0, qe) - 1.0, q / 2.0 ** -9) * np.where(normal, 8.0, 1.0)
    code = (exp_field.astype(np.int64) << 3) | np.rint(mant).astype(np.int64)
    code = np.where(q == 0, 0, code)
    return (code | (sign.astype(np.int64) << 7)).astype(np.uint8)


def e4m3_decode(code: np.ndarray) -> np.ndarray:
    """E4M3 codes -> float64 values (NaN for the two NaN patterns)."""
    c = np.asarray(code, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.ldexp(1.0, e - 7))
    val = np.where((c & 0x7F) == 0x7F, np.nan, val)
    return s * val


def pow2_scale_exponent(amax: np.ndarray) -> np.ndarray:
    """The smallest e with amax * 2^-e <= 448 (0 where amax == 0), from amax = f * 2^x, f in
    [0.5, 1): 448 = 0.875 * 2^9, so e = x - 9 when f <= 0.875 and x - 8 otherwise."""
    f, x = np.frexp(np.asarray(amax, dtype=np.float64))
    e = np.where(f <= 0.875, x - 9, x - 8)
    return np.where(np.asarray(amax) > 0, e, 0).astype(np.int64)


def quantize_rows(x: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Per-row E4M3 quantization of a [R, K] array whose values are fp32-representable.

    Returns (codes [R, K] uint8, scales [R] float32): scale = 2^e with e the smallest integer
    such that max|row| * 2^-e <= 448 (1 for an all-zero row), codes = E4M3(row * 2^-e) (exact
    scaling).
    """
    x32 = np.asarray(x, dtype=np.float32)
    e = pow2_scale_exponent(np.max(np.abs(x32), axis=1))
    s = np.ldexp(np.float32(1.0), e).astype(np.float32)
    return e4m3_encode(np.ldexp(x32.astype(np.float64), -e[:, None])), s


def quantize_matrix(w: np.ndarray) -> Tuple[np.ndarray, np.float32]:
    """E4M3 quantization of a whole matrix with one power-of-two scale (as quantize_rows)."""
    w32 = np.asarray(w, dtype=np.float32)
    e = int(pow2_scale_exponent(np.max(np.abs(w32)) if w32.size else 0.0))
    return e4m3_encode(np.ldexp(w32.astype(np.float64), -e)), np.float32(np.ldexp(1.0, e))


def fold_gain(w: np.ndarray, gain: Optional[np.ndarray]) -> np.ndarray:
    """The stored gate / up weights of a sub-layer with a norm gain: bf16(w * gain) per input column."""
    return w if gain is None else round_bf16(w * gain[None, :])


def quantize_bank(bw: Dict[str, np.ndarray], gain: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """E4M3 gate / up weights of one dense bank (one scale per matrix), bf16 down weights kept."""
    qg, sg = quantize_matrix(fold_gain(bw["w_gate"], gain))
    qu, su = quantize_matrix(fold_gain(bw["w_up"], gain))
    return {"q_gate": qg, "s_gate": sg, "q_up": qu, "s_up": su, "w_down": bw["w_down"]}


def swiglu_fp8(rows: np.ndarray, qb: Dict[str, np.ndarray], eps: float) -> np.ndarray:
    """FFN of one bank on the FP8 path, without the residual: rows [R, W] -> [R, W].

    gate = (q_a . q_gate) * s_a * s_gate / rms(x), up likewise; silu(gate) * up; then the bf16
    down projection.  s_gate, s_up: the bank's matrix scales.
    """
    ca, sa = quantize_rows(rows)
    a = e4m3_decode(ca)                                   # [R, W] quantized row values / s_a
    inv = 1.0 / np.sqrt(np.mean(rows * rows, axis=1) + eps)
    rs = sa.astype(np.float64) * inv                      # per-row factor
    g = (a @ e4m3_decode(qb["q_gate"]).T) * (rs * np.float64(qb["s_gate"]))[:, None]
    u = (a @ e4m3_decode(qb["q_up"]).T) * (rs * np.float64(qb["s_up"]))[:, None]
    return (silu(g) * u) @ qb["w_down"].T


def sublayer_fp8(rows: np.ndarray, qbank: Callable[[int], Dict[str, np.ndarray]], eps: float) -> np.ndarray:
    """rows [R, banks, W] -> FFN output [R, banks, W] (no residual), bank j with its own weights."""
    out = np.empty_like(rows)
    for j in range(rows.shape[1]):
        out[:, j, :] = swiglu_fp8(rows[:, j, :], qbank(j), eps)
    return out


# ------------------------------------------------------------------ Sparse-Pertoken MoE on the FP8 path
def quantize_moe_bank(bw: Dict[str, np.ndarray], gain: Optional[np.ndarray] = None) -> Dict[str, object]:
    """E4M3 gate / up weights of one MoE bank: one scale per routed expert's matrix and per shared
    matrix (the gain folded in first, as the bf16 path stores them); the fp32 router and the bf16
    down projections kept."""
    E = bw["we_gate"].shape[0]
    q = {"w_router": bw["w_router"],
         "experts": [quantize_bank({"w_gate": bw["we_gate"][e], "w_up": bw["we_up"][e], "w_down": bw["we_down"][e]},
                                   gain) for e in range(E)]}
    if "ws_gate" in bw:
        q["shared"] = quantize_bank({"w_gate": bw["ws_gate"], "w_up": bw["ws_up"], "w_down": bw["ws_down"]}, gain)
    return q


def sp_moe_fp8(rows: np.ndarray, qb: Dict[str, object], k: int, alpha: float, eps: float,
               gain: Optional[np.ndarray] = None, forced_idx: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """Sparse-Pertoken MoE of one bank ([digest] 2.4, Eq. 19-21) with every expert's GEMM1 on the FP8
    path ([digest] 2.5.2): rows [R, W] (the sub-layer's rows, before the RMSNorm) -> [R, W].

    The routing is the bf16 path's (RMSNorm with the gain, fp32 router, softmax, top-k, gates
    alpha * p): quantization changes the experts, not which of them a row uses.  Each chosen expert
    and the shared expert run swiglu_fp8 on the row (per-row E4M3 activations, per-matrix E4M3
    weights, 1/rms of the unquantized row), combined as alpha * sum p_e * Expert_e + Shared.
    forced_idx [R, k]: the experts of each row, as in the bf16 oracle's teacher forcing."""
    n = rmsnorm(rows, eps, gain)
    r = route(n, qb["w_router"], k)
    if forced_idx is not None:
        forced_idx = np.asarray(forced_idx)
        assert forced_idx.shape == r["idx"].shape
        assert all(len(set(row)) == k for row in forced_idx.tolist()), "forced experts repeat within a row"
        r["idx"] = forced_idx
    idx = r["idx"]
    out = np.zeros_like(rows)
    for e in range(r["p"].shape[1]):
        sel = np.nonzero(np.any(idx == e, axis=1))[0]
        if sel.size:
            out[sel] += alpha * r["p"][sel, e][:, None] * swiglu_fp8(rows[sel], qb["experts"][e], eps)
    if "shared" in qb:
        out += swiglu_fp8(rows, qb["shared"], eps)
    r["out"] = out
    return r


def sublayer_moe_fp8(rows: np.ndarray, qbank: Callable[[int], Dict[str, object]], spec, eps: float,
                     gain: Optional[np.ndarray] = None, forced_idx: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """rows [R, banks, W] -> {"out": FFN output [R, banks, W] (no residual), routing per bank}."""
    R, banks, W = rows.shape
    out = np.empty_like(rows)
    info = {"idx": [], "p": [], "logits": [], "gap": []}
    for j in range(banks):
        r = sp_moe_fp8(rows[:, j, :], qbank(j), spec.k, spec.alpha, eps, gain,
                       None if forced_idx is None else forced_idx[:, j, :])
        out[:, j, :] = r["out"]
        for key in info:
            info[key].append(r[key])
    res = {"out": out}
    for key in info:
        res[key] = np.stack(info[key], axis=1)
    return res


def block_forward_fp8(X: np.ndarray, cfg, qbank: Callable[[int, int], Dict[str, np.ndarray]],
                      storage=None) -> Dict[str, np.ndarray]:
    """A dense block on the FP8 path: the bf16 block with each sub-layer's GEMM1 quantized.

    qbank(sub, j) gives the quantized weights of bank j of sub-layer sub (0 mixing, 1 reverting).
    X_rev and the output are the stored tensors `storage` rounds, as in the bf16 block.
    """
    rnd = storage_round(storage)
    Hm = mix(X, cfg.H)
    Hn = sublayer_fp8(Hm, lambda j: qbank(0, j), cfg.eps) + Hm
    Xr = rnd(revert(Hn, cfg.T))
    Xn = sublayer_fp8(Xr, lambda j: qbank(1, j), cfg.eps) + X
    return {"Hm": Hm, "Xr": Xr, "Y": rnd(Xn)}


def block_forward_fp8_any(X: np.ndarray, cfg, qbank: Callable[[int, int], Dict[str, object]],
                          extra: Optional[np.ndarray] = None, storage=None, forced=(None, None),
                          gains=(None, None)) -> Dict[str, object]:
    """A block on the FP8 path whose sub-layers may be dense or Sparse-Pertoken MoE banks: the bf16
    block ([digest] 2.3, Eq. 9-16, residual to the block input, `extra` the stack's inter-residual
    term of 2.3.4) with every sub-layer's GEMM1 quantized as 2.5.2 serves it.  qbank(sub, j) gives
    bank j of sub-layer sub as quantize_bank (dense) or quantize_moe_bank (MoE) makes it; gains: the
    RMSNorm gains the MoE routers apply (already folded into the quantized weights); forced: the
    experts of each row per sub-layer, as sublayer_moe_fp8 takes them.  X_rev and the output are the
    stored tensors `storage` rounds."""
    rnd = storage_round(storage)
    info = {}

    def ffn(rows, sub):
        spec = cfg.ffn(sub)
        if spec.is_moe:
            r = sublayer_moe_fp8(rows, lambda j: qbank(sub, j), spec, cfg.eps, gains[sub], forced[sub])
            info[sub] = r
            return r["out"]
        return sublayer_fp8(rows, lambda j: qbank(sub, j), cfg.eps)
    Hm = mix(X, cfg.H)
    Xr = rnd(revert(ffn(Hm, 0) + Hm, cfg.T))
    Y = ffn(Xr, 1) + X
    if extra is not None:
        Y = Y + extra
    return {"Xr": Xr, "Y": rnd(Y), "mix": info.get(0), "rev": info.get(1)}

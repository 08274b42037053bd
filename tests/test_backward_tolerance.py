"""The parity bars of the backward (tests/test_gpu_backward.py) checked against the arithmetic they
are derived from, on the CPU.

A bf16 backward stores its operands and results in bf16.  Two facts fix the bars:
  * gradients are products of several normal factors, so their largest elements sit far out in
    the tails (8-12 times the rms); one bf16 ulp there is a few percent of the rms, and rounding
    even the exact gradient once to bf16 reaches a plain max error near the forward's 2e-2 bar;
  * a float64 model that rounds to bf16 every tensor a bf16 path keeps between its contractions
    (normalised rows, recomputed projections, the hidden gradients, the gradient at the
    normalised row and the result) stays well inside rms <= 1e-2 and max beyond one ulp <= 5e-2.
"""
import numpy as np

import oracle
import tm_synth as S
from oracle import backward as BW
from oracle.tokenmixer import round_bf16
from tm_synth import FFNSpec

from parity_util import rms, ulp

RMS_TOL = 1e-2
MAX_TOL = 5e-2
KEYS = ("dx", "dw_gate", "dw_up", "dw_down")


def measures(g, o):
    den = rms(o)
    return (rms(g - o) / den, float(np.max(np.abs(g - o)) / den),
            float(np.max(np.maximum(np.abs(g - o) - ulp(o, "bf16"), 0.0)) / den))


def rounded_model(x, dy, bw, eps):
    """The FFN-term gradients with every stored tensor rounded to bf16 (float64 arithmetic
    otherwise); dy and the weights are bf16 values already."""
    rb = round_bf16
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    xh = rb(x * r)
    g, u = rb(xh @ bw["w_gate"].T), rb(xh @ bw["w_up"].T)
    dh = rb(dy @ bw["w_down"])
    s = 1.0 / (1.0 + np.exp(-g))
    dg, du, h = rb(dh * u * s * (1.0 + g * (1.0 - s))), rb(dh * g * s), rb(g * s * u)
    dn = rb(dg @ bw["w_gate"] + du @ bw["w_up"])
    dx = rb(r * (dn - xh * np.mean(dn * xh, axis=-1, keepdims=True)))
    return {"dx": dx, "dw_gate": rb(dg.T @ xh), "dw_up": rb(du.T @ xh), "dw_down": rb(dy.T @ h)}


def _case():
    cfg = S.Config("bwd_tol", B=300, T=16, D=256, H=16, L=1, dtype="bf16", mix=FFNSpec("dense", hidden=384),
                   rev=FFNSpec("dense", hidden=256))
    X = S.to_f64(S.make_x(cfg))
    dY = S.to_f64(S.make_x(cfg.with_(seed=cfg.seed + 17)))
    return cfg, X, dY, oracle.synth_banks(cfg)


def test_rounding_the_exact_gradient_alone_nears_the_plain_max_bar():
    cfg, X, dY, get = _case()
    worst = {k: 0.0 for k in KEYS}
    for j in range(4):
        o = BW.swiglu_ffn_backward(X[:, j], dY[:, j], get(0, 1, j), cfg.eps)
        for k in KEYS:
            e_rms, e_max, e_ulp = measures(round_bf16(o[k]), o[k])
            assert e_ulp == 0.0                  # round to nearest: within half an ulp
            assert e_rms <= 2e-3
            worst[k] = max(worst[k], e_max)
    assert max(worst.values()) >= 1.2e-2, worst  # one rounding already uses most of a 2e-2 max bar


def test_rounded_model_within_the_backward_bars():
    cfg, X, dY, get = _case()
    for j in range(4):
        o = BW.swiglu_ffn_backward(X[:, j], dY[:, j], get(0, 1, j), cfg.eps)
        m = rounded_model(X[:, j], dY[:, j], get(0, 1, j), cfg.eps)
        for k in KEYS:
            e_rms, _, e_ulp = measures(m[k], o[k])
            assert e_rms <= RMS_TOL / 2, (k, e_rms)
            assert e_ulp <= MAX_TOL * 0.7, (k, e_ulp)


def test_bars_catch_a_planted_mistake():
    """A dropped term (the up projection's part of the gradient at the normalised row) or a
    transposed weight gradient fails the bars by far."""
    cfg, X, dY, get = _case()
    bw = get(0, 1, 0)
    o = BW.swiglu_ffn_backward(X[:, 0], dY[:, 0], bw, cfg.eps)
    m = rounded_model(X[:, 0], dY[:, 0], bw, cfg.eps)
    # dropped term: recompute dx without du Wu
    r = 1.0 / np.sqrt(np.mean(X[:, 0] ** 2, axis=-1, keepdims=True) + cfg.eps)
    xh = X[:, 0] * r
    g, u = xh @ bw["w_gate"].T, xh @ bw["w_up"].T
    s = 1.0 / (1.0 + np.exp(-g))
    dh = dY[:, 0] @ bw["w_down"]
    dn = (dh * u * s * (1.0 + g * (1.0 - s))) @ bw["w_gate"]
    bad_dx = r * (dn - xh * np.mean(dn * xh, axis=-1, keepdims=True))
    assert measures(bad_dx, o["dx"])[0] > 10 * RMS_TOL
    # a weight gradient taken from the wrong bank's rows
    bad_dw = BW.swiglu_ffn_backward(X[:, 1], dY[:, 0], bw, cfg.eps)["dw_gate"]
    assert measures(bad_dw, o["dw_gate"])[0] > 10 * RMS_TOL
    assert measures(m["dx"], o["dx"])[0] <= RMS_TOL

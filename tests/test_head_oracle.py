"""Pins of the oracle's scoring head and end-to-end model forward (oracle/tokenmixer.py: head,
model_forward) against things other than themselves: scalar loops, token-permutation invariance,
the T = 1 case (a plain dot product), and a stack that is the identity (zero down projections),
where the model's logits must be the head of the tokenizer's output."""
import numpy as np

import oracle
import tm_synth as S
from oracle import tokenmixer as O
from tm_synth import FFNSpec


def test_head_against_scalar_loops_and_invariances():
    rng = np.random.default_rng(0)
    B, T, D = 5, 7, 12
    X = rng.standard_normal((B, T, D))
    w = rng.standard_normal(D)
    got = O.head(X, w)
    want = np.array([sum(X[b, t, d] * w[d] for t in range(T) for d in range(D)) / T for b in range(B)])
    assert np.allclose(got, want, rtol=1e-13, atol=1e-13)
    assert np.allclose(O.head(X[:, rng.permutation(T), :], w), got, rtol=1e-13, atol=1e-13)   # pooling is order-free
    assert np.allclose(O.head(X[:, :1, :], w), X[:, 0, :] @ w, rtol=1e-13, atol=1e-13)        # T = 1
    assert np.allclose(O.head(np.full((2, 3, D), 0.5), w), 0.5 * w.sum())                       # constant tokens


def test_model_forward_with_an_identity_stack_scores_the_tokens():
    # zero down projections: every sub-layer adds zero, each block returns its input, and with gap 2
    # over 3 layers X_2 = 2 X_0 (the inter-residual), X_3 = X_2
    cfg = S.Config("head_id", B=6, T=5, D=16, H=4, L=3, gap=2, dtype="f32",
                   mix=FFNSpec("dense", hidden=8), rev=FFNSpec("dense", hidden=8))
    rng = np.random.default_rng(1)
    G, dg = cfg.T - 1, 3
    groups = rng.standard_normal((cfg.B, G, dg))
    w_group = rng.standard_normal((G, cfg.D, dg))
    w_global = rng.standard_normal((cfg.D, G * dg))
    w_head = rng.standard_normal(cfg.D)
    banks = oracle.synth_banks(cfg, down_scale=0.0)
    out = O.model_forward(groups, w_group, w_global, cfg, banks, w_head)
    X = O.tokenize(groups, w_group, w_global)
    assert np.allclose(out["X"], X)
    assert np.allclose(out["logits"], O.head(2 * X, w_head), rtol=1e-12, atol=1e-12)

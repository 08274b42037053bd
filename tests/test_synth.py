"""The seeded input recipe: shapes, distributions, determinism and bf16 rounding."""
import numpy as np
import pytest

import oracle
import tm_synth as S


def test_configs_shapes():
    c = S.CONFIGS
    assert [c[n].W for n in S.CONFIG_ORDER] == [64, 256, 768, 512, 768]
    assert c["nonsquare_dense_bf16"].banks(0) == 8 and c["nonsquare_dense_bf16"].banks(1) == 16
    assert c["large_moe_stack_bf16"].dh == 16 and c["nonsquare_dense_bf16"].dh == 48
    for n in ("moe_stack_bf16", "large_moe_stack_bf16"):
        m = c[n].mix
        assert m.alpha == m.E / m.k


def test_bf16_rounding_is_nearest_even():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5, 3.0e38, 1e-40], dtype=np.float32)
    back = S.bf16_to_f32(S.bf16_bits(vals))
    assert back[0] == 1.0
    assert back[1] == 1.0                       # tie -> even (down)
    assert back[2] == 1.0 + 4 * 2 ** -8         # tie -> even (up)
    assert back[3] == 1.0                       # below half ulp
    assert back[4] == -2.5
    t = None
    try:
        import torch
        t = torch.from_numpy(vals).to(torch.bfloat16).to(torch.float32).numpy()
    except Exception:
        pass
    if t is not None:
        assert np.array_equal(back, t)


def test_draws_are_deterministic_and_scaled():
    cfg = S.CONFIGS["moe_stack_bf16"]
    a = S.bank_weights(cfg, 1, 0, 5)
    b = S.bank_weights(cfg, 1, 0, 5)
    for k in a:
        assert np.array_equal(a[k], b[k])
    c = S.bank_weights(cfg, 1, 0, 6)
    assert not np.array_equal(a["we_gate"], c["we_gate"])
    W = cfg.width(0)
    assert S.to_f64(a["we_gate"]).std() == pytest.approx(W ** -0.5, rel=0.01)
    assert S.to_f64(a["we_down"]).std() == pytest.approx(0.01 * 256 ** -0.5, rel=0.01)
    assert a["w_router"].dtype == np.float32
    assert a["w_router"].std() == pytest.approx(W ** -0.5, rel=0.02)


def test_x_subsample_matches_full():
    cfg = S.CONFIGS["dense_block_bf16"].with_(B=3000)
    full = S.make_x(cfg)
    idx = S.subsample(cfg.B, 40)
    assert idx[0] == 0 and idx[-1] == cfg.B - 1 and len(np.unique(idx)) == 40
    assert np.array_equal(S.make_x(cfg, idx), full[idx])
    assert S.to_f64(full).std() == pytest.approx(1.0, rel=0.01)


def test_oracle_runs_tiny_config():
    cfg = S.CONFIGS["tiny_f32_dense"]
    out = oracle.run_stack(cfg)
    X = S.to_f64(S.make_x(cfg))
    d = out["Y"] - X
    # down-matrix small init: each sub-layer adds about 1% of the signal
    assert 1e-3 < np.sqrt(np.mean(d * d)) < 5e-2

"""Pins of the backward oracle (oracle/backward.py) against things other than its own formulas:
central finite differences of the (separately pinned) forward oracle, the scale invariance of
RMSNorm, and the special case of a zero down projection, where the block is the identity.
"""
import numpy as np
import pytest

from oracle import backward as BW
from oracle import tokenmixer as O
from tm_synth import Config, FFNSpec


def fd_grad(f, a, h=1e-6):
    """Central differences of the scalar f() with respect to every element of the array a
    (perturbed in place and restored)."""
    g = np.zeros_like(a)
    it = np.nditer(a, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        v = a[i]
        a[i] = v + h
        fp = f()
        a[i] = v - h
        fm = f()
        a[i] = v
        g[i] = (fp - fm) / (2 * h)
    return g


def close(got, want, rel=1e-6):
    scale = max(np.max(np.abs(want)), 1e-12)
    return np.max(np.abs(got - want)) <= rel * scale


@pytest.mark.parametrize("with_gain", [False, True])
def test_ffn_backward_matches_finite_differences(with_gain):
    rng = np.random.default_rng(0)
    R, W, F = 5, 8, 6
    x = rng.standard_normal((R, W))
    dy = rng.standard_normal((R, W))
    bw = {"w_gate": rng.standard_normal((F, W)), "w_up": rng.standard_normal((F, W)),
          "w_down": rng.standard_normal((W, F))}
    gain = 1 + 0.3 * rng.standard_normal(W) if with_gain else None
    eps = 1e-3                              # large enough that the eps term is exercised

    def loss():
        return float(np.sum(dy * O.swiglu(O.rmsnorm(x, eps, gain), bw["w_gate"], bw["w_up"], bw["w_down"])))
    g = BW.swiglu_ffn_backward(x, dy, bw, eps, gain)
    assert close(g["dx"], fd_grad(loss, x))
    for key in ("w_gate", "w_up", "w_down"):
        assert close(g["d" + key], fd_grad(loss, bw[key])), key
    if with_gain:
        assert close(g["dgain"], fd_grad(loss, gain))
    else:
        assert g["dgain"] is None


def test_rmsnorm_backward_is_orthogonal_to_the_input_without_eps():
    # with eps = 0 the normalised row does not change under x -> c x, so the gradient has no
    # component along x: sum_k x_k dx_k = 0 for every row
    rng = np.random.default_rng(1)
    R, W, F = 7, 16, 12
    x = rng.standard_normal((R, W)) * rng.uniform(0.1, 10, (R, 1))
    bw = {"w_gate": rng.standard_normal((F, W)), "w_up": rng.standard_normal((F, W)),
          "w_down": rng.standard_normal((W, F))}
    g = BW.swiglu_ffn_backward(x, rng.standard_normal((R, W)), bw, 0.0)
    dots = np.sum(x * g["dx"], axis=1)
    assert np.all(np.abs(dots) <= 1e-12 * np.linalg.norm(x, axis=1) * np.linalg.norm(g["dx"], axis=1))
    # and dx scales as 1/c
    g2 = BW.swiglu_ffn_backward(3.0 * x, np.ones((R, W)), bw, 0.0)
    g1 = BW.swiglu_ffn_backward(x, np.ones((R, W)), bw, 0.0)
    assert np.allclose(g2["dx"] * 3.0, g1["dx"], rtol=1e-12, atol=1e-12)


def _cfg(T, D, H, L=1, gap=0, F1=5, F2=3):
    return Config("tiny", B=2, T=T, D=D, H=H, L=L, dtype="f32", mix=FFNSpec("dense", hidden=F1),
                  rev=FFNSpec("dense", hidden=F2), gap=gap, eps=1e-6)


def _weights(cfg, rng, down=0.7):
    w = {}
    for l in range(cfg.L):
        for sub in (0, 1):
            F, W = cfg.ffn(sub).hidden, cfg.width(sub)
            for j in range(cfg.banks(sub)):
                w[(l, sub, j)] = {"w_gate": rng.standard_normal((F, W)), "w_up": rng.standard_normal((F, W)),
                                  "w_down": down * rng.standard_normal((W, F))}
    return w


@pytest.mark.parametrize("T,D,H", [(2, 4, 2), (3, 4, 2), (2, 6, 1), (4, 4, 4)])
def test_block_backward_matches_finite_differences(T, D, H):
    cfg = _cfg(T, D, H)
    rng = np.random.default_rng(T * 100 + D * 10 + H)
    w = _weights(cfg, rng)
    get = lambda l, s, j: w[(l, s, j)]
    X = rng.standard_normal((cfg.B, T, D))
    dY = rng.standard_normal((cfg.B, T, D))

    def loss():
        return float(np.sum(dY * O.block_forward(X, cfg, 0, get)["Y"]))
    g = BW.block_backward(X, cfg, 0, get, dY)
    assert close(g["dX"], fd_grad(loss, X))
    for sub, key in ((0, "mix"), (1, "rev")):
        j = cfg.banks(sub) - 1
        for name in ("w_gate", "w_up", "w_down"):
            assert close(g[key]["d" + name][j], fd_grad(loss, w[(0, sub, j)][name])), (key, name)


def test_stack_backward_with_inter_residual_matches_finite_differences():
    cfg = _cfg(2, 4, 2, L=3, gap=2)          # inter-residual after block 2 (block 3 is the last)
    rng = np.random.default_rng(5)
    w = _weights(cfg, rng)
    get = lambda l, s, j: w[(l, s, j)]
    X = rng.standard_normal((cfg.B, 2, 4))
    dY = rng.standard_normal((cfg.B, 2, 4))

    def loss():
        return float(np.sum(dY * O.stack_forward(X, cfg, get)["Y"]))
    g = BW.stack_backward(X, cfg, get, dY)
    assert close(g["dX"], fd_grad(loss, X))
    assert close(g["blocks"][0]["mix"]["dw_up"][0], fd_grad(loss, w[(0, 0, 0)]["w_up"]))
    assert close(g["blocks"][2]["rev"]["dw_down"][1], fd_grad(loss, w[(2, 1, 1)]["w_down"]))
    # without the inter-residual the gradient differs (the skip carries gradient to X_0)
    cfg0 = _cfg(2, 4, 2, L=3, gap=0)
    assert not np.allclose(BW.stack_backward(X, cfg0, get, dY)["dX"], g["dX"])


@pytest.mark.parametrize("L,gap", [(3, 1), (4, 2)])
def test_stack_backward_gap_forms_match_finite_differences(L, gap):
    """gap 1 (every block but the last adds its input back) and two blocks after an
    inter-residual (L = 4, gap = 2: X_2 += X_0, nothing after the last block)."""
    cfg = _cfg(2, 4, 2, L=L, gap=gap)
    rng = np.random.default_rng(10 + L + gap)
    w = _weights(cfg, rng)
    get = lambda l, s, j: w[(l, s, j)]
    X = rng.standard_normal((cfg.B, 2, 4))
    dY = rng.standard_normal((cfg.B, 2, 4))

    def loss():
        return float(np.sum(dY * O.stack_forward(X, cfg, get)["Y"]))
    g = BW.stack_backward(X, cfg, get, dY)
    assert close(g["dX"], fd_grad(loss, X))
    assert close(g["blocks"][0]["rev"]["dw_gate"][1], fd_grad(loss, w[(0, 1, 1)]["w_gate"]))
    assert close(g["blocks"][L - 2]["mix"]["dw_down"][0], fd_grad(loss, w[(L - 2, 0, 0)]["w_down"]))


def test_zero_down_projection_block_is_identity():
    cfg = _cfg(2, 4, 2)
    rng = np.random.default_rng(6)
    w = _weights(cfg, rng, down=0.0)
    get = lambda l, s, j: w[(l, s, j)]
    X = rng.standard_normal((cfg.B, 2, 4))
    dY = rng.standard_normal((cfg.B, 2, 4))
    g = BW.block_backward(X, cfg, 0, get, dY)
    assert np.array_equal(g["dX"], dY)
    # the reverting sub-layer's residual is the block input, so with its FFN term zero nothing
    # downstream reads the mixing sub-layer: every mixing gradient vanishes
    for j in range(cfg.banks(0)):
        for name in ("dw_gate", "dw_up", "dw_down"):
            assert not np.any(g["mix"][name][j])
    for j in range(cfg.banks(1)):
        assert not np.any(g["rev"]["dw_gate"][j]) and not np.any(g["rev"]["dw_up"][j])
        assert np.any(g["rev"]["dw_down"][j])


# ------------------------------------------------------------------ Sparse-Pertoken MoE
def _moe_bank(rng, W, E, Fe, Fs, down=0.7):
    bw = {"w_router": rng.standard_normal((E, W)),
          "we_gate": rng.standard_normal((E, Fe, W)), "we_up": rng.standard_normal((E, Fe, W)),
          "we_down": down * rng.standard_normal((E, W, Fe))}
    if Fs:
        bw.update({"ws_gate": rng.standard_normal((Fs, W)), "ws_up": rng.standard_normal((Fs, W)),
                   "ws_down": down * rng.standard_normal((W, Fs))})
    return bw


def _clear_of_ties(x, bw, k, eps, gain=None, min_gap=1e-3):
    """Finite differences of a top-k MoE are valid only away from routing ties (the chosen set
    must not change under the 1e-6 perturbations)."""
    return O.route(O.rmsnorm(x, eps, gain), bw["w_router"], k)["gap"].min() > min_gap


@pytest.mark.parametrize("E,k,Fs,with_gain", [(4, 2, 3, False), (4, 2, 0, True), (3, 3, 2, False), (5, 1, 4, True)])
def test_moe_backward_matches_finite_differences(E, k, Fs, with_gain):
    rng = np.random.default_rng(20 + E * 10 + k + Fs)
    R, W, Fe = 6, 8, 5
    alpha = E / k
    bw = _moe_bank(rng, W, E, Fe, Fs)
    gain = 1 + 0.3 * rng.standard_normal(W) if with_gain else None
    x = rng.standard_normal((R, W))
    dy = rng.standard_normal((R, W))
    eps = 1e-3
    assert _clear_of_ties(x, bw, k, eps, gain)

    def loss():
        return float(np.sum(dy * O.sp_moe(O.rmsnorm(x, eps, gain), bw, k, alpha)["out"]))
    g = BW.moe_ffn_backward(x, dy, bw, k, alpha, eps, gain)
    assert close(g["dx"], fd_grad(loss, x))
    assert close(g["dw_router"], fd_grad(loss, bw["w_router"]))
    chosen = sorted(set(g["idx"].ravel().tolist()))
    for e in (chosen[0], chosen[-1]):
        for name in ("we_gate", "we_up", "we_down"):
            assert close(g["d" + name][e], fd_grad(loss, bw[name][e])), (name, e)
    if Fs:
        for name in ("ws_gate", "ws_up", "ws_down"):
            assert close(g["d" + name], fd_grad(loss, bw[name])), name
    else:
        assert "dws_gate" not in g
    if with_gain:
        assert close(g["dgain"], fd_grad(loss, gain))


def test_moe_backward_special_cases():
    rng = np.random.default_rng(31)
    R, W, Fe = 9, 8, 4
    x = rng.standard_normal((R, W))
    dy = rng.standard_normal((R, W))
    # E = k = 1: p = 1 whatever the logit, so the router gets no gradient, exactly
    b1 = _moe_bank(rng, W, 1, Fe, 3)
    g1 = BW.moe_ffn_backward(x, dy, b1, 1, 1.0, 1e-6)
    assert not np.any(g1["dw_router"])
    # ... and the expert then acts as a second shared expert: its gradients are the dense ones
    dense = BW.swiglu_ffn_backward(x, dy, {"w_gate": b1["we_gate"][0], "w_up": b1["we_up"][0],
                                           "w_down": b1["we_down"][0]}, 1e-6)
    assert np.allclose(g1["dwe_down"][0], dense["dw_down"], rtol=1e-12, atol=1e-12)
    # an expert that no row chose gets exactly zero gradients (choices forced to experts 0..4)
    b = _moe_bank(rng, W, 6, Fe, 0)
    forced = np.array([[i % 5, (i + 1) % 5] for i in range(R)])
    g = BW.moe_ffn_backward(x, dy, b, 2, 3.0, 1e-6, forced_idx=forced)
    assert 5 not in g["idx"]
    assert not np.any(g["dwe_gate"][5]) and not np.any(g["dwe_up"][5]) and not np.any(g["dwe_down"][5])
    # the router gradient of every row sums to zero over the experts (softmax shift invariance):
    # sum_e dz_e = 0, hence sum_e dWr_e = 0
    assert np.allclose(g["dw_router"].sum(axis=0), 0.0, atol=1e-10 * np.abs(g["dw_router"]).max())


def test_moe_backward_scales_with_alpha():
    """Without a shared expert the output is linear in alpha, so every gradient is too."""
    rng = np.random.default_rng(32)
    x = rng.standard_normal((7, 8))
    dy = rng.standard_normal((7, 8))
    b = _moe_bank(rng, 8, 4, 5, 0)
    g1 = BW.moe_ffn_backward(x, dy, b, 2, 1.0, 1e-6)
    g3 = BW.moe_ffn_backward(x, dy, b, 2, 3.0, 1e-6)
    for key in ("dx", "dw_router", "dwe_gate", "dwe_down"):
        assert np.allclose(g3[key], 3.0 * g1[key], rtol=1e-12, atol=1e-12), key


def test_moe_block_backward_matches_finite_differences():
    cfg = Config("tiny_moe", B=3, T=2, D=4, H=2, L=1, dtype="f32",
                 mix=FFNSpec("moe", E=3, k=2, hidden_e=3, hidden_s=2, alpha=1.5),
                 rev=FFNSpec("moe", E=4, k=1, hidden_e=2, hidden_s=3, alpha=4.0), gap=0, eps=1e-6)
    rng = np.random.default_rng(33)
    w = {}
    for sub in (0, 1):
        s = cfg.ffn(sub)
        for j in range(cfg.banks(sub)):
            w[(0, sub, j)] = _moe_bank(rng, cfg.width(sub), s.E, s.hidden_e, s.hidden_s)
    get = lambda l, s, j: w[(l, s, j)]
    X = rng.standard_normal((cfg.B, cfg.T, cfg.D))
    dY = rng.standard_normal((cfg.B, cfg.T, cfg.D))
    # every routed row of both sub-layers clear of ties
    fwd = O.block_forward(X, cfg, 0, get)
    for key in ("mix", "rev"):
        assert np.min(fwd[key]["gap"]) > 1e-3, key

    def loss():
        return float(np.sum(dY * O.block_forward(X, cfg, 0, get)["Y"]))
    g = BW.block_backward(X, cfg, 0, get, dY)
    assert close(g["dX"], fd_grad(loss, X))
    assert close(g["mix"]["dw_router"][1], fd_grad(loss, w[(0, 0, 1)]["w_router"]))
    assert close(g["rev"]["dws_up"][0], fd_grad(loss, w[(0, 1, 0)]["ws_up"]))

"""Pins of the float64 oracle against what the pages and the mathematics fix.

None of these compares the oracle with itself: each test checks it against a
hand-worked example from the equations (tests/golden), a closed form, a
library routine, an invariant the method guarantees, or the independent
scalar brute-force restatement in oracle/brute.py.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import brute
from oracle import tokenmixer as O
from tm_synth import Config, FFNSpec

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load_mix_golden(name):
    lines = [l.strip() for l in open(os.path.join(GOLDEN, name)) if l.strip() and not l.startswith("#")]
    T, H, D = (int(lines[i].split()[1]) for i in range(3))
    xi = lines.index("X")
    mi = lines.index("MIXED")
    X = np.array([[float(v) for v in l.split()] for l in lines[xi + 1:mi]])
    M = np.array([[float(v) for v in l.split()] for l in lines[mi + 1:]])
    assert X.shape == (T, D) and M.shape == (H, T * D // H)
    return T, H, D, X, M


@pytest.mark.parametrize("name", sorted(f for f in os.listdir(GOLDEN) if f.startswith("mix_")))
def test_mix_matches_hand_worked_example(name):
    T, H, D, X, M = load_mix_golden(name)
    assert np.array_equal(O.mix(X[None], H)[0], M)
    assert np.array_equal(O.revert(M[None], T)[0], X)


@pytest.mark.parametrize("T,D,H", [(16, 256, 16), (16, 384, 8), (8, 64, 8), (32, 512, 32),
                                   (3, 6, 2), (5, 10, 1), (1, 8, 4), (7, 12, 6)])
def test_revert_is_inverse_of_mix(T, D, H):
    X = np.arange(2 * T * D, dtype=np.float64).reshape(2, T, D)
    Hm = O.mix(X, H)
    assert Hm.shape == (2, H, T * D // H)
    assert np.array_equal(O.revert(Hm, T), X)
    Y = np.arange(2 * T * D, dtype=np.float64).reshape(2, H, T * D // H) * 3 + 1
    assert np.array_equal(O.mix(O.revert(Y, T), H), Y)
    # Mix is a permutation: every element appears exactly once
    assert np.array_equal(np.sort(Hm.ravel()), X.ravel())


def test_mix_with_T_equal_H_is_block_transpose():
    T = H = 4
    D = 12
    dh = D // H
    X = np.arange(T * D, dtype=np.float64).reshape(T, D)
    grid = X.reshape(T, H, dh)                        # [t][h][j]
    expected = grid.transpose(1, 0, 2).reshape(H, T * dh)
    assert np.array_equal(O.mix(X, H), expected)
    assert np.array_equal(O.mix(O.mix(X, H), H), X)   # an involution when T == H
    assert np.array_equal(O.mix(X, H), O.revert(X, T))


def test_mix_degenerate_reshapes():
    X = np.arange(5 * 8, dtype=np.float64).reshape(5, 8)
    assert np.array_equal(O.mix(X, 1), X.reshape(1, 40))          # H = 1
    x1 = np.arange(12, dtype=np.float64).reshape(1, 12)
    assert np.array_equal(O.mix(x1, 4), x1.reshape(4, 3))         # T = 1


# ------------------------------------------------------------------ RMSNorm / SiLU / SwiGLU
def test_rmsnorm_closed_form_constant_row():
    for c in (-3.0, 0.5, 2.0):
        x = np.full((1, 6), c)
        for eps in (0.0, 1e-6, 0.1):
            r = O.rmsnorm(x, eps)
            assert np.allclose(r, c / math.sqrt(c * c + eps), rtol=1e-15, atol=0)
    g = np.array([1.0, 2.0, -1.0, 0.5])
    assert np.allclose(O.rmsnorm(np.full((1, 4), 2.0), 0.0, g), g, rtol=1e-15)


def test_rmsnorm_matches_torch():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((7, 33))
    g = rng.standard_normal(33)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (33,), weight=torch.from_numpy(g), eps=1e-6).numpy()
    assert np.allclose(O.rmsnorm(x, 1e-6, g), ref, rtol=1e-13, atol=1e-14)


def test_rmsnorm_scale_invariance():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((4, 16))
    for c in (1e-2, 3.0, 1e3):
        assert np.allclose(O.rmsnorm(c * x, 0.0), O.rmsnorm(x, 0.0), rtol=1e-13, atol=1e-14)


def test_silu_identities_and_library():
    z = np.linspace(-30, 30, 1201)
    s = O.silu(z)
    assert O.silu(np.array([0.0]))[0] == 0.0
    assert np.allclose(s - O.silu(-z), z, rtol=1e-13, atol=1e-13)     # z*sig(z) + z*sig(-z) = z
    assert np.allclose(s, torch.nn.functional.silu(torch.from_numpy(z)).numpy(), rtol=1e-14, atol=1e-300)


def test_swiglu_identity_weights_closed_form():
    n = np.array([[-2.0, -0.5, 0.0, 0.7, 3.0]])
    I = np.eye(5)
    expected = n / (1.0 + np.exp(-n)) * n                              # silu(n_i) * n_i
    assert np.allclose(O.swiglu(n, I, I, I), expected, rtol=1e-15)


def test_swiglu_matches_torch_linear():
    rng = np.random.default_rng(3)
    n = rng.standard_normal((6, 10))
    wg, wu, wd = rng.standard_normal((7, 10)), rng.standard_normal((7, 10)), rng.standard_normal((10, 7))
    t = lambda a: torch.from_numpy(a)
    F = torch.nn.functional
    ref = F.linear(F.silu(F.linear(t(n), t(wg))) * F.linear(t(n), t(wu)), t(wd)).numpy()
    assert np.allclose(O.swiglu(n, wg, wu, wd), ref, rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------------ router / MoE
def test_softmax_of_two_is_sigmoid():
    z = np.array([[0.3, -1.2], [5.0, 5.0], [-40.0, 2.0]])
    p = O.softmax(z)
    assert np.allclose(p[:, 0], 1.0 / (1.0 + np.exp(z[:, 1] - z[:, 0])), rtol=1e-14)
    assert np.allclose(p.sum(1), 1.0, rtol=1e-15)


def test_topk_ties_go_to_lower_index():
    assert O.topk(np.full((1, 4), 0.25), 2).tolist() == [[0, 1]]
    assert O.topk(np.array([[0.1, 0.3, 0.3, 0.3]]), 2).tolist() == [[1, 2]]
    assert O.topk(np.array([[0.4, 0.1, 0.4, 0.1]]), 3).tolist() == [[0, 2, 1]]


def test_route_gap_and_positive_scaling():
    rng = np.random.default_rng(4)
    n = rng.standard_normal((50, 12))
    wr = rng.standard_normal((6, 12))
    r = O.route(n, wr, 2)
    z = n @ wr.T
    for i in range(50):
        s = sorted(z[i], reverse=True)
        assert r["gap"][i] == pytest.approx(s[1] - s[2], rel=1e-12)
        assert set(r["idx"][i]) == set(np.argsort(z[i])[::-1][:2])
    for c in (1e-3, 7.0):
        assert np.array_equal(O.route(n, c * wr, 2)["idx"], r["idx"])   # top-k ignores logit scale
    assert np.all(np.isinf(O.route(n, wr, 6)["gap"]))


def _moe_bank(rng, W, E, Fe, Fs, scale=0.6):
    bw = {"w_router": rng.standard_normal((E, W)),
          "we_gate": scale * rng.standard_normal((E, Fe, W)),
          "we_up": scale * rng.standard_normal((E, Fe, W)),
          "we_down": scale * rng.standard_normal((E, W, Fe))}
    if Fs:
        bw.update(ws_gate=scale * rng.standard_normal((Fs, W)), ws_up=scale * rng.standard_normal((Fs, W)),
                  ws_down=scale * rng.standard_normal((W, Fs)))
    return bw


def test_moe_k_equals_E_is_dense_softmax_sum():
    rng = np.random.default_rng(5)
    n = rng.standard_normal((9, 8))
    bw = _moe_bank(rng, 8, 4, 5, 3)
    from scipy.special import softmax as sp_softmax
    p = sp_softmax(n @ bw["w_router"].T, axis=1)
    dense = sum(p[:, e:e + 1] * O.swiglu(n, bw["we_gate"][e], bw["we_up"][e], bw["we_down"][e]) for e in range(4))
    dense = dense + O.swiglu(n, bw["ws_gate"], bw["ws_up"], bw["ws_down"])
    assert np.allclose(O.sp_moe(n, bw, 4, 1.0)["out"], dense, rtol=1e-12, atol=1e-12)


def test_moe_single_expert_is_expert_plus_shared():
    rng = np.random.default_rng(6)
    n = rng.standard_normal((5, 6))
    bw = _moe_bank(rng, 6, 1, 4, 2)
    r = O.sp_moe(n, bw, 1, 2.5)
    assert np.all(r["p"] == 1.0)
    exp = 2.5 * O.swiglu(n, bw["we_gate"][0], bw["we_up"][0], bw["we_down"][0]) + \
        O.swiglu(n, bw["ws_gate"], bw["ws_up"], bw["ws_down"])
    assert np.allclose(r["out"], exp, rtol=1e-13, atol=1e-14)


def test_moe_dense_masked_form_equals_sparse():
    rng = np.random.default_rng(7)
    n = rng.standard_normal((40, 8))
    for Fs in (0, 3):
        bw = _moe_bank(rng, 8, 6, 4, Fs)
        for k in (1, 2, 5):
            assert np.allclose(O.sp_moe(n, bw, k, 3.0)["out"], O.sp_moe_dense_masked(n, bw, k, 3.0),
                               rtol=1e-12, atol=1e-12)


def test_moe_expert_permutation_invariance_and_alpha_linearity():
    rng = np.random.default_rng(8)
    n = rng.standard_normal((30, 8))
    bw = _moe_bank(rng, 8, 5, 4, 3)
    perm = np.array([3, 0, 4, 1, 2])
    pw = dict(bw)
    for key in ("w_router", "we_gate", "we_up", "we_down"):
        pw[key] = bw[key][perm]
    base = O.sp_moe(n, bw, 2, 2.0)["out"]
    assert np.allclose(O.sp_moe(n, pw, 2, 2.0)["out"], base, rtol=1e-12, atol=1e-13)
    shared = O.swiglu(n, bw["ws_gate"], bw["ws_up"], bw["ws_down"])
    o5 = O.sp_moe(n, bw, 2, 5.0)["out"]
    assert np.allclose(o5 - shared, 2.5 * (base - shared), rtol=1e-12, atol=1e-13)


def test_moe_rows_are_independent():
    rng = np.random.default_rng(9)
    n = rng.standard_normal((20, 8))
    bw = _moe_bank(rng, 8, 4, 3, 2)
    perm = rng.permutation(20)
    assert np.allclose(O.sp_moe(n[perm], bw, 2, 2.0)["out"], O.sp_moe(n, bw, 2, 2.0)["out"][perm], rtol=1e-13)


# ------------------------------------------------------------------ block / stack
def _tiny_cfg(T, D, H, moe, L=1, gap=0):
    if moe:
        sm = FFNSpec("moe", E=3, k=2, hidden_e=3, hidden_s=2, alpha=1.5)
        sr = FFNSpec("moe", E=4, k=1, hidden_e=2, hidden_s=3, alpha=4.0)
    else:
        sm, sr = FFNSpec("dense", hidden=5), FFNSpec("dense", hidden=3)
    return Config("tiny", B=2, T=T, D=D, H=H, L=L, dtype="f32", mix=sm, rev=sr, gap=gap, eps=1e-6)


def _tiny_weights(cfg, rng, down=0.7):
    out = {}
    for l in range(cfg.L):
        for sub in (0, 1):
            spec, W, banks = cfg.ffn(sub), cfg.width(sub), cfg.banks(sub)
            for j in range(banks):
                if spec.is_moe:
                    bw = _moe_bank(rng, W, spec.E, spec.hidden_e, spec.hidden_s)
                    bw["we_down"] *= down
                    if spec.hidden_s:
                        bw["ws_down"] *= down
                else:
                    bw = {"w_gate": rng.standard_normal((spec.hidden, W)), "w_up": rng.standard_normal((spec.hidden, W)),
                          "w_down": down * rng.standard_normal((W, spec.hidden))}
                out[(l, sub, j)] = bw
    return out


def _as_lists(cfg, weights, l, sub):
    banks = cfg.banks(sub)
    keys = weights[(l, sub, 0)].keys()
    return {k: [weights[(l, sub, j)][k].tolist() for j in range(banks)] for k in keys}


@pytest.mark.parametrize("H", [1, 2, 4])
@pytest.mark.parametrize("moe", [False, True])
def test_block_matches_bruteforce(H, moe):
    cfg = _tiny_cfg(2, 4, H, moe)
    rng = np.random.default_rng(10 + H + 10 * moe)
    w = _tiny_weights(cfg, rng)
    X = rng.standard_normal((2, 2, 4))
    got = O.block_forward(X, cfg, 0, lambda l, s, j: w[(l, s, j)])["Y"]
    ref = brute.block(X.tolist(), 2, 4, H, cfg.eps, cfg.mix, _as_lists(cfg, w, 0, 0), cfg.rev, _as_lists(cfg, w, 0, 1))
    assert np.allclose(got, np.array(ref), rtol=1e-12, atol=1e-12)


def test_block_nonsquare_matches_bruteforce():
    cfg = _tiny_cfg(3, 6, 2, True)     # T=3 tokens, H=2 heads, rows of width 9
    rng = np.random.default_rng(21)
    w = _tiny_weights(cfg, rng)
    X = rng.standard_normal((2, 3, 6))
    got = O.block_forward(X, cfg, 0, lambda l, s, j: w[(l, s, j)])["Y"]
    ref = brute.block(X.tolist(), 3, 6, 2, cfg.eps, cfg.mix, _as_lists(cfg, w, 0, 0), cfg.rev, _as_lists(cfg, w, 0, 1))
    assert np.allclose(got, np.array(ref), rtol=1e-12, atol=1e-12)


def test_stack_matches_bruteforce_with_inter_residual():
    cfg = _tiny_cfg(2, 4, 2, True, L=3, gap=2)
    rng = np.random.default_rng(22)
    w = _tiny_weights(cfg, rng, down=0.4)
    X = rng.standard_normal((2, 2, 4))
    got = O.stack_forward(X, cfg, lambda l, s, j: w[(l, s, j)])["Y"]
    specs = [(cfg.mix, cfg.rev)] * 3
    wl = [(_as_lists(cfg, w, l, 0), _as_lists(cfg, w, l, 1)) for l in range(3)]
    ref = brute.stack(X.tolist(), 2, 4, 2, cfg.eps, 3, 2, specs, wl)
    assert np.allclose(got, np.array(ref), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("moe", [False, True])
def test_zero_down_projection_makes_block_identity(moe):
    cfg = _tiny_cfg(4, 8, 2, moe, L=5, gap=2)
    rng = np.random.default_rng(23)
    w = _tiny_weights(cfg, rng, down=0.0)
    X = rng.standard_normal((3, 4, 8))
    b = O.block_forward(X, cfg, 0, lambda l, s, j: w[(l, s, j)])
    assert np.array_equal(b["Y"], X)
    hist = O.stack_forward(X, cfg, lambda l, s, j: w[(l, s, j)])["hist"]
    # X1 = X0, X2 = X1 + X0, X3 = X2, X4 = X3 + X2, X5 = X4 (the last layer takes no inter-residual)
    for l, c in enumerate([1, 1, 2, 2, 4, 4]):
        assert np.array_equal(hist[l], c * X), l
    # L = 4 is a multiple of the gap: the last layer still takes no inter-residual
    hist4 = O.stack_forward(X, cfg.with_(L=4), lambda l, s, j: w[(l, s, j)])["hist"]
    for l, c in enumerate([1, 1, 2, 2, 2]):
        assert np.array_equal(hist4[l], c * X), l


def test_per_bank_isolation():
    cfg = _tiny_cfg(4, 8, 2, True)       # dh = 4, mixing rows of width 16
    rng = np.random.default_rng(24)
    w = _tiny_weights(cfg, rng)
    X = rng.standard_normal((3, 4, 8))
    get = lambda l, s, j: w[(l, s, j)]
    base = O.block_forward(X, cfg, 0, get)
    w2 = dict(w)
    w2[(0, 0, 1)] = {k: v * 1.3 for k, v in w[(0, 0, 1)].items()}   # perturb mixing bank h = 1
    pert = O.block_forward(X, cfg, 0, lambda l, s, j: w2[(l, s, j)])
    dHn = np.abs(pert["Hn"] - base["Hn"]).max(axis=(0, 2))
    assert dHn[0] == 0 and dHn[1] > 0
    dXr = np.abs(pert["Xr"] - base["Xr"]).max(axis=(0, 1))
    assert np.all(dXr[:4] == 0) and np.all(dXr[4:] > 0)             # only head-1 columns of every token
    w3 = dict(w)
    w3[(0, 1, 2)] = {k: v * 1.3 for k, v in w[(0, 1, 2)].items()}   # perturb reverting bank t = 2
    pert = O.block_forward(X, cfg, 0, lambda l, s, j: w3[(l, s, j)])
    dY = np.abs(pert["Y"] - base["Y"]).max(axis=(0, 2))
    assert np.all(dY[[0, 1, 3]] == 0) and dY[2] > 0


def test_samples_are_independent():
    cfg = _tiny_cfg(4, 8, 4, True, L=2, gap=2)
    rng = np.random.default_rng(25)
    w = _tiny_weights(cfg, rng)
    X = rng.standard_normal((6, 4, 8))
    get = lambda l, s, j: w[(l, s, j)]
    full = O.stack_forward(X, cfg, get)["Y"]
    perm = np.array([4, 1, 5, 0, 3, 2])
    assert np.allclose(O.stack_forward(X[perm], cfg, get)["Y"], full[perm], rtol=1e-13, atol=1e-14)
    assert np.allclose(O.stack_forward(X[2:3], cfg, get)["Y"], full[2:3], rtol=1e-13, atol=1e-14)


def test_tokenize_matches_bruteforce_and_identity():
    rng = np.random.default_rng(26)
    g = rng.standard_normal((3, 4, 5))
    wg = rng.standard_normal((4, 6, 5))
    wG = rng.standard_normal((6, 20))
    got = O.tokenize(g, wg, wG)
    assert got.shape == (3, 5, 6)
    assert np.allclose(got, np.array(brute.tokenize(g.tolist(), wg.tolist(), wG.tolist())), rtol=1e-13, atol=1e-13)
    # identity group maps copy each group; a global map picking element c of group i puts it at d
    gi = rng.standard_normal((2, 3, 4))
    eye = np.stack([np.eye(4)] * 3)
    wsel = np.zeros((4, 12))
    wsel[0, 5] = wsel[1, 0] = wsel[2, 11] = wsel[3, 6] = 1.0
    X = O.tokenize(gi, eye, wsel)
    assert np.array_equal(X[:, 1:, :], gi)
    flat = gi.reshape(2, 12)
    assert np.array_equal(X[:, 0, :], flat[:, [5, 0, 11, 6]])


def test_round_bf16_matches_bit_rounding_and_scalar_form():
    import tm_synth
    rng = np.random.default_rng(30)
    v = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-6, 6, 20000),
                        [0.0, 1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 255.5, 256.5]])
    v32 = v.astype(np.float32)                               # values exactly representable in fp32
    bits = tm_synth.bf16_to_f32(tm_synth.bf16_bits(v32)).astype(np.float64)
    assert np.array_equal(O.round_bf16(v32.astype(np.float64)), bits)
    assert all(brute.round_bf16(float(x)) == float(r) for x, r in zip(v32[:500], bits[:500]))
    assert O.round_bf16(np.array([1.0 + 2 ** -8]))[0] == 1.0                 # tie to even
    assert O.round_bf16(np.array([1.0 + 3 * 2 ** -8]))[0] == 1.0 + 2 ** -6   # tie to even (up)


@pytest.mark.parametrize("moe", [False, True])
def test_stack_with_storage_rounding_matches_bruteforce(moe):
    cfg = _tiny_cfg(2, 4, 2, moe, L=3, gap=2)
    rng = np.random.default_rng(31)
    w = _tiny_weights(cfg, rng, down=0.5)
    X = O.round_bf16(rng.standard_normal((2, 2, 4)))
    got = O.stack_forward(X, cfg, lambda l, s, j: w[(l, s, j)], storage="bf16")["Y"]
    specs = [(cfg.mix, cfg.rev)] * 3
    wl = [(_as_lists(cfg, w, l, 0), _as_lists(cfg, w, l, 1)) for l in range(3)]
    ref = brute.stack(X.tolist(), 2, 4, 2, cfg.eps, 3, 2, specs, wl, rnd=brute.round_bf16)
    assert np.allclose(got, np.array(ref), rtol=0, atol=1e-12)
    assert np.array_equal(got, O.round_bf16(got))                           # the output is a stored tensor
    plain = O.stack_forward(X, cfg, lambda l, s, j: w[(l, s, j)])["Y"]
    assert 0 < np.max(np.abs(plain - got)) < 0.5                            # a rounding-size perturbation


def test_storage_rounding_keeps_zero_down_identity():
    cfg = _tiny_cfg(4, 8, 2, True, L=4, gap=2)
    rng = np.random.default_rng(32)
    w = _tiny_weights(cfg, rng, down=0.0)
    X = O.round_bf16(rng.standard_normal((3, 4, 8)))
    hist = O.stack_forward(X, cfg, lambda l, s, j: w[(l, s, j)], storage="bf16")["hist"]
    for l, c in enumerate([1, 1, 2, 2, 2]):
        assert np.array_equal(hist[l], c * X), l


def test_teacher_forced_routing():
    """The oracle's teacher-forced routing: forcing its own choices (in any order) reproduces its
    output; forcing another expert set on one row changes that row alone, to alpha * sum over the
    forced experts of p_e * Expert_e plus the shared expert, written out here row by row."""
    rng = np.random.default_rng(21)
    R, W, E, k, Fe = 12, 16, 5, 2, 8
    n = rng.standard_normal((R, W))
    bw = {"w_router": rng.standard_normal((E, W)) / 4,
          "we_gate": rng.standard_normal((E, Fe, W)) / 4, "we_up": rng.standard_normal((E, Fe, W)) / 4,
          "we_down": rng.standard_normal((E, W, Fe)) / 4,
          "ws_gate": rng.standard_normal((Fe, W)) / 4, "ws_up": rng.standard_normal((Fe, W)) / 4,
          "ws_down": rng.standard_normal((W, Fe)) / 4}
    base = O.sp_moe(n, bw, k, 2.5)
    assert np.array_equal(O.sp_moe(n, bw, k, 2.5, base["idx"])["out"], base["out"])
    assert np.allclose(O.sp_moe(n, bw, k, 2.5, base["idx"][:, ::-1])["out"], base["out"], rtol=1e-14, atol=1e-14)
    forced = base["idx"].copy()
    row = 3
    other = [e for e in range(E) if e not in set(forced[row].tolist())][:k]
    forced[row] = other
    got = O.sp_moe(n, bw, k, 2.5, forced)["out"]
    keep = np.arange(R) != row
    assert np.array_equal(got[keep], base["out"][keep])
    p = O.softmax(n[row] @ bw["w_router"].T)
    want = sum(2.5 * p[e] * O.swiglu(n[row:row + 1], bw["we_gate"][e], bw["we_up"][e], bw["we_down"][e])[0]
               for e in other) + O.swiglu(n[row:row + 1], bw["ws_gate"], bw["ws_up"], bw["ws_down"])[0]
    assert np.allclose(got[row], want, rtol=1e-12, atol=1e-12)
    with pytest.raises(AssertionError):
        O.sp_moe(n, bw, k, 2.5, np.zeros_like(forced))       # an expert chosen twice in a row

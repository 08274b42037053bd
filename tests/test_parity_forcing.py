"""The near-tie forcing that the GPU parity checks rest on, on the CPU with the oracle alone:
fed the oracle's own routing as "GPU" choices it substitutes nothing and reproduces the oracle's
stack; a different expert set on a row clear of any tie is counted as a failure; a different set
on a near-tie row is substituted and changes that sample alone."""
import numpy as np

import oracle
import tm_synth as S
from parity_util import GAP_TOL, err_stored, force_near_ties, oracle_stack_forced, rms
from tm_synth import FFNSpec


def _cfg():
    spec = FFNSpec("moe", E=6, k=2, hidden_e=16, hidden_s=16, alpha=3.0)
    return S.Config("forcing", B=40, T=4, D=32, H=4, L=3, gap=2, dtype="bf16", mix=spec, rev=spec)


def _own_routes(cfg, get):
    res = oracle.run_stack(cfg, keep=True, storage="bf16")
    return res, [{"mix": b["mix"]["idx"], "rev": b["rev"]["idx"]} for b in res["blocks"]]


def test_own_routing_substitutes_nothing_and_reproduces_the_stack():
    cfg = _cfg()
    get = oracle.synth_banks(cfg)
    ref, routes = _own_routes(cfg, get)
    res = oracle_stack_forced(cfg, S.to_f64(S.make_x(cfg)), get, routes)
    assert res["bad"] == 0 and res["near"] == 0
    assert res["decisions"] == cfg.L * cfg.B * (cfg.H + cfg.T)
    for l in range(cfg.L):
        assert np.array_equal(res["Y"][l], ref["hist"][l + 1])


def test_other_set_outside_a_tie_is_a_failure_and_inside_one_is_followed():
    cfg = _cfg()
    get = oracle.synth_banks(cfg)
    ref, routes = _own_routes(cfg, get)
    info = ref["blocks"][0]["mix"]
    # a row far from a tie: swapping its second choice for an unchosen expert must count as bad
    r, b = np.argwhere(info["gap"] > 10 * GAP_TOL)[0]
    gi = info["idx"].copy()
    gi[r, b, 1] = next(e for e in range(cfg.mix.E) if e not in gi[r, b])
    forced, bad, sub = force_near_ties(info, gi)
    assert (bad, sub) == (1, 0)
    assert np.array_equal(forced, info["idx"])
    # the same row declared a near tie (gap below the bar): the GPU's set is followed there alone
    near = dict(info)
    near["gap"] = info["gap"].copy()
    near["gap"][r, b] = 0.0
    # the substituted set must be a valid top-k under the oracle's logits: make its logit tie
    near["logits"] = info["logits"].copy()
    zk = np.sort(near["logits"][r, b])[::-1][1]
    near["logits"][r, b, gi[r, b, 1]] = zk
    forced, bad, sub = force_near_ties(near, gi)
    assert (bad, sub) == (0, 1)
    assert np.array_equal(forced[r, b], gi[r, b])
    others = np.ones(forced.shape[:2], dtype=bool)
    others[r, b] = False
    assert np.array_equal(forced[others], info["idx"][others])


def test_layer_prefetch_getter_gives_the_same_weights():
    """The layer-at-a-time getter (parallel draws, storage dtype held) returns the very weights of the
    plain getter, in any order of requests across layers."""
    cfg = _cfg()
    plain = oracle.synth_banks(cfg)
    layer = oracle.synth_banks(cfg, cache="layer", workers=2)
    for l in (0, 2, 1, 1, 0):
        for s in (1, 0):
            for j in (3, 0, 2):
                wa, wb = plain(l, s, j), layer(l, s, j)
                assert set(wa) == set(wb)
                assert all(np.array_equal(wa[k], wb[k]) for k in wa)


def test_stored_measure_allows_one_ulp_and_no_more():
    """err_stored: a bf16 value one ulp away from the oracle's counts as no error (the two sides may
    round one real number to neighbouring bf16 values); anything beyond that ulp counts in full."""
    o = np.array([5.0, -0.25, 1.0, 3.0])          # rms 2.96
    y = o.copy()
    y[0] = 5.03125                                 # one ulp above 5 (bf16 spacing 2^-5 in [4, 8))
    assert err_stored("bf16", y, o) == 0.0
    y[0] = 5.0625                                  # two ulps
    assert np.isclose(err_stored("bf16", y, o), 0.03125 / rms(o))
    y = o.copy()
    y[1] = -0.25 - 0.1                             # far beyond the ulp of a small value
    assert np.isclose(err_stored("bf16", y, o), (0.1 - 2.0 ** -9) / rms(o))   # ulp in [0.25, 0.5): 2^-9
    assert err_stored("f32", o * (1 + 1e-6), o) <= 1.01e-6

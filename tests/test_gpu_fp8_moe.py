"""GPU parity of the Sparse-Pertoken MoE sub-layer on the FP8 path (every expert's GEMM1 on E4M3
operands, kind::f8f6f4) against the float64 oracle in oracle/fp8.py, through the C ABI.

The weight and row quantizers are integer work decided by fp32 arithmetic on both sides, so the
codes and scales match bit for bit; the routing is the bf16 path's, and the oracle follows the
GPU's own expert choices (teacher forcing, as for the bf16 MoE).  With identical operands the
sub-layer differs from the oracle by fp32 accumulation order, the bf16 roundings of the hidden rows
and of each gate-scaled routed expert row (up to 2^-8 of |alpha p_e Expert_e|, allowed per element)
and the output's own ulp: the bf16 tolerance applies to what remains.
"""
import numpy as np
import pytest
import torch

import oracle
import tm_synth as S
from oracle import fp8 as F
from oracle import tokenmixer as O
from tm_synth import FFNSpec
from token_sparse_moe_b200 import api
from token_sparse_moe_b200 import _abi as A

from parity_util import GAP_TOL, err_moe_delta, to_np, tol

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def moe(E, k, Fe, Fs, alpha=None):
    return FFNSpec("moe", E=E, k=k, hidden_e=Fe, hidden_s=Fs, alpha=float(E) / k if alpha is None else alpha)


def small(name, B, T, D, H, mix, rev):
    return S.Config(name, B=B, T=T, D=D, H=H, L=1, dtype="bf16", mix=mix, rev=rev)


CASES = [
    # Mix map with dh = 16 and the tensor-core router; reverting top-1; 300 rows = 2 tiles + 44
    small("fp8moe_sq", 300, 16, 256, 16, moe(8, 2, 128, 128, 4.0), moe(4, 1, 128, 256, 4.0)),
    # mixing width 768 (dh = 96), 16 experts top-4; reverting width 384
    small("fp8moe_ns", 260, 8, 384, 4, moe(16, 4, 128, 256), moe(6, 3, 256, 128)),
    # 24 experts: the CUDA-core router
    small("fp8moe_e24", 170, 8, 256, 8, moe(24, 3, 128, 128), moe(24, 2, 128, 128)),
    # degenerate routing: k = E (every row reaches every expert) and a single expert
    small("fp8moe_kE", 200, 8, 256, 8, moe(4, 4, 128, 128, 1.0), moe(1, 1, 128, 128, 2.0)),
]


def dev(a):
    return api.to_device(a, DEV)


def layout_of(sub):
    return A.TM_LAYOUT_MIXED if sub == 0 else A.TM_LAYOUT_ROWS


def qbank(cfg, layer, sub, down_scale=None, gain=None):
    banks = oracle.synth_banks(cfg, down_scale)
    return lambda j: F.quantize_moe_bank(banks(layer, sub, j), gain)


def fp8_routed_abs_contrib(rows, qb, spec, eps, gain, forced_idx):
    """Per element: sum over the row's chosen experts of |alpha * p_e * Expert_e(row)| on the FP8 path
    (the size of the gate-scaled routed rows that the GPU stores in bf16 before the combine)."""
    R, banks, W = rows.shape
    out = np.zeros_like(rows)
    for j in range(banks):
        q = qb(j)
        r = O.route(O.rmsnorm(rows[:, j, :], eps, gain), q["w_router"], spec.k)
        for e in range(spec.E):
            sel = np.nonzero(np.any(forced_idx[:, j, :] == e, axis=1))[0]
            if sel.size:
                ye = F.swiglu_fp8(rows[sel, j, :], q["experts"][e], eps)
                out[sel, j, :] += np.abs(spec.alpha * r["p"][sel, e][:, None] * ye)
    return out


def check_fp8_moe(cfg, sub, X, R, y, gi, down_scale, gain=None, samples=None):
    """y (the GPU's output on all samples) against the oracle on `samples` (all when None), routed by
    the GPU's choices gi [B, banks, k]; the GPU's choices differ from the oracle's own only in near ties."""
    spec = cfg.ffn(sub)
    s = np.arange(cfg.B) if samples is None else np.asarray(samples)
    X64, R64 = S.to_f64(X[s]), S.to_f64(R[s])
    rows = O.mix(X64, cfg.H) if sub == 0 else X64
    res = O.mix(R64, cfg.H) if sub == 0 else R64
    qb = qbank(cfg, 0, sub, down_scale, gain)
    forced = gi[s]
    r = F.sublayer_moe_fp8(rows, qb, spec, cfg.eps, gain, forced_idx=forced)
    o = r["out"] + res
    c = fp8_routed_abs_contrib(rows, qb, spec, cfg.eps, gain, forced)
    if sub == 0:
        o, c = O.revert(o, cfg.T), O.revert(c, cfg.T)
    e = err_moe_delta(y[s], o, R64, c, "bf16")
    assert e <= tol("bf16"), e
    own = F.sublayer_moe_fp8(rows, qb, spec, cfg.eps, gain)
    flip = np.any(np.sort(forced, -1) != np.sort(own["idx"], -1), axis=-1)
    assert np.all(own["gap"][flip] < GAP_TOL), "routing differs outside a near tie"
    return e, int(flip.sum())


@pytest.mark.parametrize("with_gain", [False, True], ids=["gain1", "gain"])
@pytest.mark.parametrize("cfg", CASES[:2], ids=lambda c: c.name)
def test_moe_weight_quantizer_bit_exact(cfg, with_gain):
    for sub in (0, 1):
        sw = api.sublayer_from_synth(cfg, 0, sub, DEV, None, with_gain)
        s8 = api.MoeSubLayer8.from_bf16(sw)
        torch.cuda.synchronize()
        g = S.to_f64(S.gain(cfg, 0, sub)) if with_gain else None
        qb = qbank(cfg, 0, sub, None, g)
        spec = cfg.ffn(sub)
        t = {k: v.cpu().numpy() for k, v in s8.tensors.items() if v.dtype != torch.bfloat16}
        for j in range(cfg.banks(sub)):
            o = qb(j)
            for e in range(spec.E):
                ge = j * spec.E + e
                assert np.array_equal(t["qe_gate"][ge], o["experts"][e]["q_gate"])
                assert np.array_equal(t["qe_up"][ge], o["experts"][e]["q_up"])
                assert t["se_gate"][ge] == o["experts"][e]["s_gate"] and t["se_up"][ge] == o["experts"][e]["s_up"]
            assert np.array_equal(t["qs_gate"][j], o["shared"]["q_gate"])
            assert np.array_equal(t["qs_up"][j], o["shared"]["q_up"])
            assert t["ss_gate"][j] == o["shared"]["s_gate"] and t["ss_up"][j] == o["shared"]["s_up"]


@pytest.mark.parametrize("resid", [False, True], ids=["no_resid", "resid"])
@pytest.mark.parametrize("sub", [0, 1])
@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_fp8_moe_sublayer(cfg, sub, resid):
    """Every row of the FP8 MoE sub-layer, down projections at std x 1 so that the FFN term is as
    large as the residual."""
    X = S.make_x(cfg)
    R = S.make_x(cfg.with_(seed=cfg.seed + 17))
    sh = api.config_shape(cfg)
    sw = api.sublayer_from_synth(cfg, 0, sub, DEV, 1.0)
    s8 = api.MoeSubLayer8.from_bf16(sw)
    gi = api.route_topk(dev(X), layout_of(sub), sh, sw)["idx"].cpu().numpy().astype(np.int64)
    Rd = dev(R) if resid else None
    y = api.sparse_pertoken_moe_fp8(dev(X), Rd, layout_of(sub), sh, s8)
    api.get_device_error()
    y2 = api.sublayer_forward_fp8(dev(X), Rd, None, layout_of(sub), sh, s8)
    api.get_device_error()
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    Rz = R if resid else np.zeros_like(R)
    check_fp8_moe(cfg, sub, X, Rz, to_np(y), gi, 1.0)


@pytest.mark.parametrize("cfg", CASES[:1], ids=lambda c: c.name)
def test_fp8_moe_gain_and_extra(cfg):
    """A norm gain (folded into the codes by the quantizer, applied by the router) and an
    inter-residual term beside the residual."""
    X = S.make_x(cfg)
    R = S.make_x(cfg.with_(seed=cfg.seed + 17))
    Xe = S.make_x(cfg.with_(seed=cfg.seed + 29))
    sh = api.config_shape(cfg)
    for sub in (0, 1):
        sw = api.sublayer_from_synth(cfg, 0, sub, DEV, 1.0, with_gain=True)
        s8 = api.MoeSubLayer8.from_bf16(sw)
        gi = api.route_topk(dev(X), layout_of(sub), sh, sw)["idx"].cpu().numpy().astype(np.int64)
        y = to_np(api.sublayer_forward_fp8(dev(X), dev(R), dev(Xe), layout_of(sub), sh, s8))
        api.get_device_error()
        g = S.to_f64(S.gain(cfg, 0, sub))
        # the oracle's residual term is R + Xe (both added before y's single rounding)
        Rs = (S.to_f64(R) + S.to_f64(Xe)).astype(np.float64)
        check_fp8_moe(cfg, sub, X, Rs, y, gi, 1.0, gain=g)


@pytest.mark.parametrize("sub", [0, 1])
def test_fp8_moe_full_size_sampled(sub):
    """The MoE stack workload's first block (B = 8192, 32 banks, E = 8, top-2) on the FP8 path, on a
    sample of rows: rows are independent, so the oracle on the sampled samples is exact for them."""
    cfg = S.CONFIGS["moe_stack_bf16"]
    samples = S.subsample(cfg.B, 48)
    X = S.make_x(cfg)
    R = S.make_x(cfg.with_(seed=cfg.seed + 17))
    sh = api.config_shape(cfg)
    sw = api.sublayer_from_synth(cfg, 0, sub, DEV)
    s8 = api.MoeSubLayer8.from_bf16(sw)
    gi = api.route_topk(dev(X), layout_of(sub), sh, sw)["idx"].cpu().numpy().astype(np.int64)
    y = to_np(api.sparse_pertoken_moe_fp8(dev(X), dev(R), layout_of(sub), sh, s8))
    api.get_device_error()
    check_fp8_moe(cfg, sub, X, R, y, gi, None, samples=samples)


def test_fp8_moe_rejects_what_it_does_not_cover():
    cfg = small("fp8moe_bad", 64, 8, 256, 8, moe(8, 2, 64, 128), moe(8, 2, 128, 128))   # hidden_e 64
    sh = api.config_shape(cfg)
    s8 = api.MoeSubLayer8.from_bf16(api.sublayer_from_synth(cfg, 0, 0, DEV))
    with pytest.raises(A.TMError) as e:
        api.sparse_pertoken_moe_fp8(dev(S.make_x(cfg)), None, A.TM_LAYOUT_MIXED, sh, s8)
    assert e.value.status == A.TM_ERR_UNSUPPORTED


STACK = S.Config("fp8moe_stack", B=300, T=16, D=256, H=16, L=3, gap=2, dtype="bf16",
                 mix=moe(8, 2, 128, 128, 4.0), rev=moe(8, 2, 256, 128, 4.0))


def test_fp8_moe_stack():
    """A three-block MoE stack with the inter-residual (gap 2) on the FP8 path: Fp8StackRunner against
    the same blocks run one sub-layer at a time, and every block's X_revert and output against the
    oracle's FP8 block chain, which follows the GPU's expert choices on near-tie rows only."""
    from parity_util import err_stored, force_near_ties, skip_term
    cfg = STACK
    sh = api.config_shape(cfg)
    bf = api.blocks_from_synth(cfg, DEV)
    b8 = [(api.MoeSubLayer8.from_bf16(b.mix), api.MoeSubLayer8.from_bf16(b.rev)) for b in bf]
    X = S.make_x(cfg)
    Xd = dev(X)
    Y = torch.empty_like(Xd)
    api.Fp8StackRunner(b8, sh, cfg.gap, DEV)(Xd, Y)
    api.get_device_error()
    # the chain, sub-layer by sub-layer, with every block's X_revert and routing
    hist, xrs, routes = [Xd], [], []
    for l in range(cfg.L):
        extra = skip_term(cfg, hist, l + 1)
        xr = api.sublayer_forward_fp8(hist[l], hist[l], None, A.TM_LAYOUT_MIXED, sh, b8[l][0])
        y = api.sublayer_forward_fp8(xr, hist[l], extra, A.TM_LAYOUT_ROWS, sh, b8[l][1])
        routes.append({0: api.route_topk(hist[l], A.TM_LAYOUT_MIXED, sh, bf[l].mix)["idx"].cpu().numpy(),
                       1: api.route_topk(xr, A.TM_LAYOUT_ROWS, sh, bf[l].rev)["idx"].cpu().numpy()})
        hist.append(y)
        xrs.append(xr)
    api.get_device_error()
    assert torch.equal(hist[-1].view(torch.int16), Y.view(torch.int16))
    get = oracle.synth_banks(cfg)
    q = {}

    def qb(l):
        return lambda s, j: q.setdefault((l, s, j), F.quantize_moe_bank(get(l, s, j)))
    ohist = [S.to_f64(X)]
    near = 0
    for l in range(cfg.L):
        extra = skip_term(cfg, ohist, l + 1)
        forced = [None, None]
        b = F.block_forward_fp8_any(ohist[l], cfg, qb(l), extra, "bf16")
        for s, key in ((0, "mix"), (1, "rev")):
            f, bad, nsub = force_near_ties(b[key], routes[l][s])
            assert bad == 0, f"block {l + 1} {key}: {bad} rows routed differently outside near ties"
            near += nsub
            if nsub:
                forced[s] = f
                b = F.block_forward_fp8_any(ohist[l], cfg, qb(l), extra, "bf16", forced=tuple(forced))
        for name, g, o in (("X_revert", xrs[l], b["Xr"]), ("Y", hist[l + 1], b["Y"])):
            e = err_stored("bf16", to_np(g), o)
            assert e <= tol("bf16"), (l + 1, name, e)
        ohist.append(b["Y"])

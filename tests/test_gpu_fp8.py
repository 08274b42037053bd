"""GPU parity of the FP8 E4M3 serving path (GEMM1 on E4M3 operands) against the float64 oracle
in oracle/fp8.py, through the C ABI.

The quantizers are integer work decided by fp32 arithmetic on both sides, so their codes and
scales must match bit for bit.  With the operands identical, the FFN differs from the oracle
only by fp32 accumulation order and the bf16 roundings of the hidden and output rows: the bf16
tolerance applies.
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

from parity_util import BF16_TOL, err_bf16, err_delta, to_np, tol

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def small(name, B, T, D, H, F1, F2):
    return S.Config(name, B=B, T=T, D=D, H=H, L=1, dtype="bf16", mix=FFNSpec("dense", hidden=F1),
                    rev=FFNSpec("dense", hidden=F2))


CASES = [
    # mixing width 256 through the Mix map (dh = 16), reverting width 256; 300 rows = 2 tiles + 44
    small("fp8_sq", 300, 16, 256, 16, 384, 256),
    # mixing width 256 (dh = 32), reverting width 128; 5 row tiles
    small("fp8_w128", 600, 8, 128, 4, 128, 256),
    # both widths 128 (T = H = 8, dh = 16)
    small("fp8_t8", 260, 8, 128, 8, 256, 128),
]


def rows_of(cfg, X, sub):
    return O.mix(X, cfg.H) if sub == 0 else X


def qbank_oracle(cfg, sub, down_scale=None, with_gain=False):
    banks = oracle.synth_banks(cfg, down_scale)
    g = S.to_f64(S.gain(cfg, 0, sub)) if with_gain else None
    return lambda j: F.quantize_bank(banks(0, sub, j), g)


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
@pytest.mark.parametrize("with_gain", [False, True], ids=["gain1", "gain"])
def test_weight_quantizer_bit_exact(cfg, with_gain):
    for sub in (0, 1):
        sw = api.sublayer_from_synth(cfg, 0, sub, DEV, None, with_gain)
        s8 = api.SubLayer8.from_bf16(sw)
        torch.cuda.synchronize()
        qb = qbank_oracle(cfg, sub, None, with_gain)
        for j in range(cfg.banks(sub)):
            o = qb(j)
            assert np.array_equal(s8.tensors["q_gate"][j].cpu().numpy(), o["q_gate"])
            assert np.array_equal(s8.tensors["q_up"][j].cpu().numpy(), o["q_up"])
            assert s8.tensors["s_gate"][j].cpu().numpy() == o["s_gate"]
            assert s8.tensors["s_up"][j].cpu().numpy() == o["s_up"]


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_activation_quantizer_bit_exact(cfg):
    X = S.make_x(cfg)
    Xf = S.to_f64(X)
    sh = api.config_shape(cfg)
    for sub, layout in ((0, A.TM_LAYOUT_MIXED), (1, A.TM_LAYOUT_ROWS)):
        q, rs = api.quantize_fp8_act(api.to_device(X, DEV), layout, sh, cfg.banks(sub), cfg.width(sub))
        rows = rows_of(cfg, Xf, sub).reshape(-1, cfg.width(sub))
        codes, s = F.quantize_rows(rows)
        assert np.array_equal(q.cpu().numpy(), codes)
        inv = 1.0 / np.sqrt(np.mean(rows * rows, axis=1) + cfg.eps)
        # the scale factor is exact; 1/rms differs by the fp32 summation order only
        assert np.allclose(rs.cpu().numpy(), s.astype(np.float64) * inv, rtol=2e-6, atol=0)


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
@pytest.mark.parametrize("resid", [False, True], ids=["no_resid", "resid"])
def test_fp8_sublayer(cfg, resid):
    # down weights at std x 1 so that the FFN term is as large as the residual
    X = S.make_x(cfg)
    R = S.make_x(cfg.with_(seed=cfg.seed + 17))
    Xf, Rf = S.to_f64(X), S.to_f64(R)
    sh = api.config_shape(cfg)
    for sub, layout in ((0, A.TM_LAYOUT_MIXED), (1, A.TM_LAYOUT_ROWS)):
        s8 = api.SubLayer8.from_bf16(api.sublayer_from_synth(cfg, 0, sub, DEV, 1.0))
        y = api.pertoken_swiglu_fp8(api.to_device(X, DEV), api.to_device(R, DEV) if resid else None, layout, sh, s8)
        api.get_device_error()
        y = to_np(y)
        ffn = F.sublayer_fp8(rows_of(cfg, Xf, sub), qbank_oracle(cfg, sub, 1.0), cfg.eps)
        if sub == 0:
            ffn = O.revert(ffn, cfg.T)
        # the FFN's error beyond one ulp of the stored output, relative to the FFN term's rms (with no
        # residual the stored value is the FFN term itself)
        base = Rf if resid else np.zeros_like(ffn)
        e = err_delta(y, ffn + base, base, "bf16")
        assert e <= tol("bf16"), e


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_fp8_block(cfg, monkeypatch):
    """The FP8 block: one launch when both sub-layers have the same row width (T == H; reverting
    tiles wait for their row block's mixing tiles), the same bits as one launch per sub-layer,
    within tolerance of the oracle, and the same bits from one call to the next."""
    X = S.make_x(cfg)
    blk = api.Block8.from_bf16(api.blocks_from_synth(cfg, DEV)[0])
    sh = api.config_shape(cfg)
    Xd = api.to_device(X, DEV)

    def run():
        Xr = torch.empty_like(Xd)
        api.profile_start()
        Y = api.block_forward_fp8(Xd, blk, sh, X_revert=Xr)
        api.get_device_error()
        return Y, Xr, api.profile_stop()
    Y, Xr, prof = run()
    one_launch = cfg.width(0) == cfg.width(1)
    assert prof["fused_swiglu_fp8"]["launches"] == (1 if one_launch else 2) and "fp8_quant_rows" not in prof
    monkeypatch.setenv("TM_FUSED_BLOCK", "0")
    Y0, Xr0, prof0 = run()
    monkeypatch.delenv("TM_FUSED_BLOCK")
    assert prof0["fused_swiglu_fp8"]["launches"] == 2
    assert torch.equal(Y.view(torch.int16), Y0.view(torch.int16))
    assert torch.equal(Xr.view(torch.int16), Xr0.view(torch.int16))
    qb = {sub: qbank_oracle(cfg, sub) for sub in (0, 1)}
    b = F.block_forward_fp8(S.to_f64(X), cfg, lambda sub, j: qb[sub](j), storage="bf16")
    assert err_bf16(to_np(Xr), b["Xr"]) <= BF16_TOL
    assert err_bf16(to_np(Y), b["Y"]) <= BF16_TOL
    Y2, _, _ = run()
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))


def test_fp8_block_full_size_sampled():
    """The dense block workload (B = 4096) on the FP8 path, checked on a sample of rows: samples
    are independent, so the oracle's block on those samples is exact for them."""
    cfg = S.CONFIGS["dense_block_bf16"]
    samples = S.subsample(cfg.B, 128)
    X = S.make_x(cfg)
    blk = api.Block8.from_bf16(api.blocks_from_synth(cfg, DEV)[0])
    Y = to_np(api.block_forward_fp8(api.to_device(X, DEV), blk, api.config_shape(cfg)))
    api.get_device_error()
    qb = {sub: qbank_oracle(cfg, sub) for sub in (0, 1)}
    b = F.block_forward_fp8(S.to_f64(S.make_x(cfg, samples)), cfg, lambda sub, j: qb[sub](j), storage="bf16")
    assert err_bf16(Y[samples], b["Y"]) <= BF16_TOL


def test_fp8_rejects_what_it_does_not_cover():
    cfg = small("fp8_bad", 64, 16, 384, 8, 256, 256)      # mixing width 768: not a fused width
    sh = api.config_shape(cfg)
    s8 = api.SubLayer8.from_bf16(api.sublayer_from_synth(cfg, 0, 0, DEV))
    with pytest.raises(A.TMError) as e:
        api.pertoken_swiglu_fp8(api.to_device(S.make_x(cfg), DEV), None, A.TM_LAYOUT_MIXED, sh, s8)
    assert e.value.status == A.TM_ERR_UNSUPPORTED

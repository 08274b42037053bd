"""Pins of the FP8 E4M3 serving oracle (oracle/fp8.py) against things other than itself:
PyTorch's float8_e4m3fn conversion (a library routine), the code table's closed forms, the
rounding bound of a 3-bit mantissa, and the special case in which quantization is exact, where
the FP8 FFN must equal the bf16 oracle's FFN.
"""
import numpy as np
import torch

from oracle import fp8 as F
from oracle import tokenmixer as O


def torch_codes(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_codec_matches_torch_float8_conversion():
    rng = np.random.default_rng(0)
    parts = [
        rng.standard_normal(20000).astype(np.float32) * 30,          # the normal range
        rng.uniform(-2.0 ** -6, 2.0 ** -6, 20000).astype(np.float32),  # subnormals
        rng.uniform(-448, 448, 20000).astype(np.float32),
    ]
    # exact ties between neighbouring codes in every binade (and the subnormal spacing)
    vals = F.e4m3_decode(np.arange(0, 0x7E, dtype=np.uint8))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    parts += [mids, -mids, np.float32([0.0, -0.0, 448.0, -448.0, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -11])]
    x = np.concatenate(parts)
    assert np.array_equal(F.e4m3_encode(x), torch_codes(x))


def test_code_table_closed_forms():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    assert np.array_equal(F.e4m3_encode(F.e4m3_decode(codes).astype(np.float32)), codes)
    e = F.e4m3_encode(np.float32([448.0, 2.0 ** -9, 2.0 ** -6, 1.0, 1.0 + 1 / 16, 1.0 + 3 / 16, 1000.0, -1000.0,
                                  2.0 ** -10, 1.5 * 2.0 ** -9]))
    # 448 = 1.75*2^8 -> exponent field 15, mantissa 6; the smallest subnormal; the smallest normal;
    # 1.0; ties go to the even mantissa (1.0 and 1.25); saturation; half the smallest subnormal is a
    # tie that rounds to zero (even), 1.5 of it rounds up to 2 subnormal steps
    assert list(e) == [0x7E, 0x01, 0x08, 0x38, 0x38, 0x3A, 0x7E, 0xFE, 0x00, 0x02]
    assert F.e4m3_decode(np.uint8([0x7E]))[0] == 448.0
    assert np.isnan(F.e4m3_decode(np.uint8([0x7F, 0xFF]))).all()


def test_row_quantization_bounds():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((64, 256)) * rng.uniform(0.01, 100, (64, 1))).astype(np.float32)
    x[3] = 0.0
    x[5] = rng.uniform(-1, 1, 256).astype(np.float32)
    x[5, 7] = 448.0 * 2.0 ** -4                                 # a row maximum exactly on the top code
    codes, s = F.quantize_rows(x)
    assert s.dtype == np.float32 and s[3] == 1.0 and s[5] == 2.0 ** -4
    assert np.all(np.frexp(s)[0] == 0.5)                        # powers of two
    q = F.e4m3_decode(codes)
    nz = np.arange(64) != 3
    # the smallest power-of-two scale that fits: the largest element scales into (224, 448] and
    # rounds to a code in [224, 448]
    m = np.max(np.abs(x[nz]), axis=1) / s[nz]
    assert np.all((m > 224.0) & (m <= 448.0))
    top = np.max(np.abs(q[nz]), axis=1)
    assert np.all((top >= 224.0) & (top <= 448.0))
    assert np.max(np.abs(q[5])) == 448.0
    err = np.abs(q * s[:, None].astype(np.float64) - x)
    # half a step of a 3-bit mantissa (2^-4 relative) in the normal range, half the subnormal
    # spacing (2^-10 * s) below it
    bound = np.maximum(2.0 ** -4 * np.abs(x), 2.0 ** -10 * s[:, None])
    assert np.all(err <= bound * (1 + 1e-6))


def test_fp8_ffn_equals_bf16_ffn_when_quantization_is_exact():
    # rows and weights already on the E4M3 grid, each row's (and each weight matrix's) largest
    # magnitude exactly 448 * 2^k: the scale is 2^k, the scaling exact and every code reproduces
    # its value
    rng = np.random.default_rng(2)
    W, Fh, R = 64, 96, 24

    def grid_rows(n, k, scale_pow):
        c = rng.integers(0, 0x7E, (n, k)).astype(np.uint8) | (rng.integers(0, 2, (n, k)).astype(np.uint8) << 7)
        c[:, 0] = 0x7E                                      # +448 in every row
        return F.e4m3_decode(c) * 2.0 ** scale_pow
    x = grid_rows(R, W, -6)
    bw = {"w_gate": grid_rows(Fh, W, -12), "w_up": grid_rows(Fh, W, -12),
          "w_down": O.round_bf16(rng.standard_normal((W, Fh)) * 0.05)}
    qb = F.quantize_bank(bw)
    assert qb["s_gate"] == np.float32(2.0 ** -12)
    assert np.array_equal(F.e4m3_decode(qb["q_gate"]) * np.float64(qb["s_gate"]), bw["w_gate"])
    eps = 1e-6
    got = F.swiglu_fp8(x, qb, eps)
    want = O.swiglu(O.rmsnorm(x, eps), bw["w_gate"], bw["w_up"], bw["w_down"])
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_fp8_ffn_tracks_bf16_ffn_within_the_quantization_error():
    # generic inputs: the FP8 FFN is the bf16 FFN up to the E4M3 rounding of both GEMM1 operands
    rng = np.random.default_rng(3)
    W, Fh, R = 128, 256, 64
    x = O.round_bf16(rng.standard_normal((R, W)))
    bw = {k: O.round_bf16(rng.standard_normal(shape) / np.sqrt(shape[1]))
          for k, shape in (("w_gate", (Fh, W)), ("w_up", (Fh, W)), ("w_down", (W, Fh)))}
    got = F.swiglu_fp8(x, F.quantize_bank(bw), 1e-6)
    want = O.swiglu(O.rmsnorm(x, 1e-6), bw["w_gate"], bw["w_up"], bw["w_down"])
    rel = np.sqrt(np.mean((got - want) ** 2) / np.mean(want ** 2))
    assert 1e-3 < rel < 0.08, rel


def test_gain_is_folded_then_quantized():
    rng = np.random.default_rng(4)
    w = O.round_bf16(rng.standard_normal((8, 32)))
    g = O.round_bf16(1 + 0.1 * rng.standard_normal(32))
    qb = F.quantize_bank({"w_gate": w, "w_up": w, "w_down": w.T}, g)
    c, s = F.quantize_matrix(O.round_bf16(w * g[None, :]))
    assert np.array_equal(qb["q_gate"], c) and qb["s_gate"] == s


def test_matrix_scale_is_the_matrix_maximum():
    rng = np.random.default_rng(5)
    w = (rng.standard_normal((16, 40)) * rng.uniform(0.1, 10, (16, 1))).astype(np.float32)
    codes, s = F.quantize_matrix(w)
    m = np.max(np.abs(w))
    assert np.frexp(s)[0] == 0.5 and m / s <= 448.0 < 2 * m / s   # the smallest power of two that fits
    q = F.e4m3_decode(codes)
    assert 224.0 <= np.max(np.abs(q)) <= 448.0
    # every value above the subnormal range keeps the 2^-4 relative rounding bound, whatever its row
    big = np.abs(w) >= 2.0 ** -6 * s
    assert np.all(np.abs(q * np.float64(s) - w)[big] <= 2.0 ** -4 * np.abs(w)[big] * (1 + 1e-6))
    assert np.array_equal(F.quantize_matrix(np.zeros((3, 4)))[0], np.zeros((3, 4), np.uint8))
    assert F.quantize_matrix(np.zeros((3, 4)))[1] == 1.0


def _grid(rng, n, k, scale_pow):
    """[n, k] values on the E4M3 grid, each row's largest magnitude exactly 448 * 2^scale_pow."""
    c = rng.integers(0, 0x7E, (n, k)).astype(np.uint8) | (rng.integers(0, 2, (n, k)).astype(np.uint8) << 7)
    c[:, 0] = 0x7E
    return F.e4m3_decode(c) * 2.0 ** scale_pow


def _moe_bank(rng, W, E, Fe, Fs, on_grid):
    if on_grid:
        gu = lambda n: _grid(rng, n, W, -12)
    else:
        gu = lambda n: O.round_bf16(rng.standard_normal((n, W)) / np.sqrt(W))
    return {"w_router": rng.standard_normal((E, W)) / np.sqrt(W),
            "we_gate": np.stack([gu(Fe) for _ in range(E)]), "we_up": np.stack([gu(Fe) for _ in range(E)]),
            "we_down": O.round_bf16(rng.standard_normal((E, W, Fe)) * 0.05),
            "ws_gate": gu(Fs), "ws_up": gu(Fs), "ws_down": O.round_bf16(rng.standard_normal((W, Fs)) * 0.05)}


def test_fp8_moe_equals_bf16_moe_when_quantization_is_exact():
    # on-grid rows and expert weights: every expert's GEMM1 is exact, so the FP8 MoE is the bf16
    # oracle's MoE (same routing, same gates alpha * p, same shared expert) up to float64 rounding
    rng = np.random.default_rng(11)
    W, E, k, Fe, Fs, R = 64, 6, 2, 32, 48, 40
    bw = _moe_bank(rng, W, E, Fe, Fs, on_grid=True)
    x = _grid(rng, R, W, -6)
    qb = F.quantize_moe_bank(bw)
    assert [q["s_gate"] for q in qb["experts"]] == [np.float32(2.0 ** -12)] * E
    got = F.sp_moe_fp8(x, qb, k, 3.0, 1e-6)
    want = O.sp_moe(O.rmsnorm(x, 1e-6), bw, k, 3.0)
    assert np.array_equal(got["idx"], want["idx"])
    assert np.allclose(got["out"], want["out"], rtol=1e-12, atol=1e-12 * np.abs(want["out"]).max())
    # a dropped expert scale (a plausible mistake) shows
    bad = dict(qb)
    bad["experts"] = [dict(q, s_gate=np.float32(1.0)) for q in qb["experts"]]
    assert not np.allclose(F.sp_moe_fp8(x, bad, k, 3.0, 1e-6)["out"], want["out"], rtol=1e-3)


def test_fp8_moe_with_k_equal_E_is_the_dense_softmax_sum_of_fp8_experts():
    rng = np.random.default_rng(12)
    W, E, Fe, Fs, R = 32, 4, 16, 16, 20
    bw = _moe_bank(rng, W, E, Fe, Fs, on_grid=False)
    x = O.round_bf16(rng.standard_normal((R, W)))
    qb = F.quantize_moe_bank(bw)
    got = F.sp_moe_fp8(x, qb, E, 1.0, 1e-6)["out"]
    p = O.softmax(O.rmsnorm(x, 1e-6) @ bw["w_router"].T)
    want = sum(p[:, e:e + 1] * F.swiglu_fp8(x, qb["experts"][e], 1e-6) for e in range(E)) + F.swiglu_fp8(x, qb["shared"], 1e-6)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-13)


def test_fp8_moe_tracks_bf16_moe_and_forcing_works():
    rng = np.random.default_rng(13)
    W, E, k, Fe, Fs, R = 64, 8, 2, 32, 32, 64
    bw = _moe_bank(rng, W, E, Fe, Fs, on_grid=False)
    x = O.round_bf16(rng.standard_normal((R, W)))
    qb = F.quantize_moe_bank(bw)
    got = F.sp_moe_fp8(x, qb, k, 4.0, 1e-6)
    want = O.sp_moe(O.rmsnorm(x, 1e-6), bw, k, 4.0)
    assert np.array_equal(got["idx"], want["idx"])              # quantization leaves the routing alone
    rel = np.sqrt(np.mean((got["out"] - want["out"]) ** 2) / np.mean(want["out"] ** 2))
    assert 1e-3 < rel < 0.08, rel
    forced = got["idx"][:, ::-1].copy()                       # the same sets, other order: same output
    assert np.allclose(F.sp_moe_fp8(x, qb, k, 4.0, 1e-6, forced_idx=forced)["out"], got["out"], rtol=1e-12, atol=1e-15)


def _moe_cfg():
    import tm_synth as S
    spec = S.FFNSpec("moe", E=4, k=2, hidden_e=16, hidden_s=16, alpha=2.0)
    return S.Config("fp8_block_pin", B=12, T=4, D=64, H=4, L=1, dtype="bf16", mix=spec, rev=spec)


def test_fp8_moe_block_reductions():
    """block_forward_fp8_any against what fixes it: (1) zero down projections make the block the
    identity, plus the inter-residual term; (2) on E4M3-grid rows and weights the mixing sub-layer's
    GEMM1s are exact, so X_rev is the bf16 oracle block's; (3) with dense banks it is block_forward_fp8."""
    import tm_synth as S
    cfg = _moe_cfg()
    rng = np.random.default_rng(21)
    banks = {(s, j): _moe_bank(rng, cfg.width(s), 4, 16, 16, on_grid=True) for s in (0, 1) for j in range(4)}
    X = _grid(rng, cfg.B * cfg.T, cfg.D, -6).reshape(cfg.B, cfg.T, cfg.D)
    q = {key: F.quantize_moe_bank(bw) for key, bw in banks.items()}
    got = F.block_forward_fp8_any(X, cfg, lambda s, j: q[(s, j)])
    want = O.block_forward(X, cfg, 0, lambda l, s, j: banks[(s, j)])
    assert np.allclose(got["Xr"], want["Xr"], rtol=1e-12, atol=1e-12)
    assert np.array_equal(got["mix"]["idx"], want["mix"]["idx"])
    # zero down projections: Y = X + extra exactly, X_rev = X
    zq = {key: dict(v, experts=[dict(e, w_down=0 * e["w_down"]) for e in v["experts"]],
                    shared=dict(v["shared"], w_down=0 * v["shared"]["w_down"])) for key, v in q.items()}
    extra = O.round_bf16(rng.standard_normal(X.shape))
    z = F.block_forward_fp8_any(X, cfg, lambda s, j: zq[(s, j)], extra=extra)
    assert np.array_equal(z["Xr"], X) and np.array_equal(z["Y"], X + extra)
    # dense banks: the dense FP8 block
    dcfg = S.Config("fp8_block_pin_dense", B=12, T=4, D=64, H=4, L=1, dtype="bf16",
                    mix=S.FFNSpec("dense", hidden=32), rev=S.FFNSpec("dense", hidden=32))
    dq = {(s, j): F.quantize_bank({"w_gate": O.round_bf16(rng.standard_normal((32, 64)) / 8),
                                   "w_up": O.round_bf16(rng.standard_normal((32, 64)) / 8),
                                   "w_down": O.round_bf16(rng.standard_normal((64, 32)) / 8)})
          for s in (0, 1) for j in range(4)}
    Xd = O.round_bf16(rng.standard_normal(X.shape))
    a = F.block_forward_fp8_any(Xd, dcfg, lambda s, j: dq[(s, j)], storage="bf16")
    b = F.block_forward_fp8(Xd, dcfg, lambda s, j: dq[(s, j)], storage="bf16")
    assert np.array_equal(a["Y"], b["Y"]) and np.array_equal(a["Xr"], b["Xr"])

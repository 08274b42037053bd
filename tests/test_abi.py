"""The C ABI on the CPU: the library loads, exports every entry point include/tm.h
declares, its struct layouts match the C compiler's, and host-side validation and
workspace queries answer without touching a GPU."""
import ctypes
import os
import re
import subprocess

import pytest

import tm_synth as S
from token_sparse_moe_b200 import _abi as A
from token_sparse_moe_b200 import api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tm.h")


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"TM_API[^;]*?\b(tm_\w+)\s*\(", text)))


def test_header_and_binding_agree():
    assert declared_functions() == sorted(A.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = A.load()
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", A.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (tm_\w+)", out))
    assert set(declared_functions()) <= exported
    assert lib.tm_version() == 100


def test_struct_layout_matches_c(tmp_path):
    src = tmp_path / "layout.c"
    src.write_text(r'''
#include <stdio.h>
#include <stddef.h>
#include "tm.h"
#define P(T, f) printf(#T "." #f " %zu\n", offsetof(T, f));
int main(void) {
  printf("tm_shape %zu\ntm_swiglu_w %zu\ntm_moe_w %zu\ntm_sublayer %zu\ntm_block %zu\n",
         sizeof(tm_shape), sizeof(tm_swiglu_w), sizeof(tm_moe_w), sizeof(tm_sublayer), sizeof(tm_block));
  P(tm_shape, eps) P(tm_swiglu_w, w_gate) P(tm_swiglu_w, w_down) P(tm_moe_w, alpha) P(tm_moe_w, w_router)
  P(tm_moe_w, ws_down) P(tm_sublayer, dense) P(tm_sublayer, moe) P(tm_block, rev)
  printf("tm_swiglu_w8 %zu\ntm_block_fp8 %zu\n", sizeof(tm_swiglu_w8), sizeof(tm_block_fp8));
  P(tm_swiglu_w8, q_gate) P(tm_swiglu_w8, s_up) P(tm_swiglu_w8, w_down) P(tm_block_fp8, rev)
  printf("tm_swiglu_grads %zu\ntm_block_grads %zu\n", sizeof(tm_swiglu_grads), sizeof(tm_block_grads));
  P(tm_swiglu_grads, dw_up) P(tm_swiglu_grads, dw_down) P(tm_block_grads, rev)
  printf("tm_moe_w8 %zu\ntm_sublayer8 %zu\n", sizeof(tm_moe_w8), sizeof(tm_sublayer8));
  P(tm_moe_w8, alpha) P(tm_moe_w8, w_router) P(tm_moe_w8, se_up) P(tm_moe_w8, we_down) P(tm_moe_w8, ss_up)
  P(tm_moe_w8, ws_down) P(tm_sublayer8, dense) P(tm_sublayer8, moe)
  printf("TM_TP_TOKEN_SHARD %d\nTM_TP_HEAD_SHARD %d\n", TM_TP_TOKEN_SHARD, TM_TP_HEAD_SHARD);
  return 0;
}
''')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = dict(l.split() for l in subprocess.run([str(exe)], capture_output=True, text=True).stdout.splitlines())
    want = {
        "tm_shape": ctypes.sizeof(A.tm_shape), "tm_swiglu_w": ctypes.sizeof(A.tm_swiglu_w),
        "tm_moe_w": ctypes.sizeof(A.tm_moe_w), "tm_sublayer": ctypes.sizeof(A.tm_sublayer),
        "tm_block": ctypes.sizeof(A.tm_block),
        "tm_shape.eps": A.tm_shape.eps.offset, "tm_swiglu_w.w_gate": A.tm_swiglu_w.w_gate.offset,
        "tm_swiglu_w.w_down": A.tm_swiglu_w.w_down.offset, "tm_moe_w.alpha": A.tm_moe_w.alpha.offset,
        "tm_moe_w.w_router": A.tm_moe_w.w_router.offset, "tm_moe_w.ws_down": A.tm_moe_w.ws_down.offset,
        "tm_sublayer.dense": A.tm_sublayer.dense.offset, "tm_sublayer.moe": A.tm_sublayer.moe.offset,
        "tm_block.rev": A.tm_block.rev.offset,
        "tm_swiglu_w8": ctypes.sizeof(A.tm_swiglu_w8), "tm_block_fp8": ctypes.sizeof(A.tm_block_fp8),
        "tm_swiglu_w8.q_gate": A.tm_swiglu_w8.q_gate.offset, "tm_swiglu_w8.s_up": A.tm_swiglu_w8.s_up.offset,
        "tm_swiglu_w8.w_down": A.tm_swiglu_w8.w_down.offset, "tm_block_fp8.rev": A.tm_block_fp8.rev.offset,
        "tm_swiglu_grads": ctypes.sizeof(A.tm_swiglu_grads), "tm_block_grads": ctypes.sizeof(A.tm_block_grads),
        "tm_swiglu_grads.dw_up": A.tm_swiglu_grads.dw_up.offset,
        "tm_swiglu_grads.dw_down": A.tm_swiglu_grads.dw_down.offset,
        "tm_block_grads.rev": A.tm_block_grads.rev.offset,
        "tm_moe_w8": ctypes.sizeof(A.tm_moe_w8), "tm_sublayer8": ctypes.sizeof(A.tm_sublayer8),
        "tm_moe_w8.alpha": A.tm_moe_w8.alpha.offset, "tm_moe_w8.w_router": A.tm_moe_w8.w_router.offset,
        "tm_moe_w8.se_up": A.tm_moe_w8.se_up.offset, "tm_moe_w8.we_down": A.tm_moe_w8.we_down.offset,
        "tm_moe_w8.ss_up": A.tm_moe_w8.ss_up.offset, "tm_moe_w8.ws_down": A.tm_moe_w8.ws_down.offset,
        "tm_sublayer8.dense": A.tm_sublayer8.dense.offset, "tm_sublayer8.moe": A.tm_sublayer8.moe.offset,
        "TM_TP_TOKEN_SHARD": A.TM_TP_TOKEN_SHARD, "TM_TP_HEAD_SHARD": A.TM_TP_HEAD_SHARD,
    }
    assert {k: int(v) for k, v in got.items()} == want


def test_status_strings():
    lib = A.load()
    assert lib.tm_status_string(0) == b"ok"
    assert lib.tm_status_string(3) == b"workspace missing or too small"


class _FakeTensor:
    """Stands in for a device tensor in host-only calls: only its address is passed."""

    def __init__(self, addr=0x10000):
        self.addr = addr

    def data_ptr(self):
        return self.addr


def _fake_sub(cfg, sub):
    spec = cfg.ffn(sub)
    names = (["w_router", "we_gate", "we_up", "we_down", "ws_gate", "ws_up", "ws_down"] if spec.is_moe
             else ["w_gate", "w_up", "w_down"])
    t = {n: _FakeTensor(0x100000 * (i + 1)) for i, n in enumerate(names)}
    if spec.is_moe:
        return api.SubLayer(True, cfg.banks(sub), cfg.width(sub), t, E=spec.E, k=spec.k, hidden_e=spec.hidden_e,
                            hidden_s=spec.hidden_s, alpha=spec.alpha)
    return api.SubLayer(False, cfg.banks(sub), cfg.width(sub), t, hidden=spec.hidden)


@pytest.mark.parametrize("name", S.CONFIG_ORDER)
def test_workspace_queries(name):
    cfg = S.CONFIGS[name]
    sh = api.config_shape(cfg)
    blocks = [api.Block(_fake_sub(cfg, 0), _fake_sub(cfg, 1)) for _ in range(cfg.L)]
    n = api.workspace_bytes(sh, blocks, cfg.gap)
    tok = cfg.B * cfg.T * cfg.D * (2 if cfg.dtype == "bf16" else 4)
    assert n > tok
    m = api.sublayer_workspace_bytes(sh, A.TM_LAYOUT_MIXED, blocks[0].mix)
    r = api.sublayer_workspace_bytes(sh, A.TM_LAYOUT_ROWS, blocks[0].rev)
    assert n >= max(m, r) + tok
    if cfg.mix.is_moe:
        w = blocks[0].mix.moe_c()
        assert A.load().tm_route_workspace_bytes(ctypes.byref(sh), A.TM_LAYOUT_MIXED, ctypes.byref(w)) > 0


def test_host_validation_rejects_before_launch():
    lib = A.load()
    cfg = S.CONFIGS["dense_block_bf16"]
    sub = _fake_sub(cfg, 0)
    w = sub.dense_c()
    good = api.config_shape(cfg)
    bad = api.shape(cfg.B, cfg.T, 250, cfg.H, "bf16")          # D % H != 0
    x, y, ws = ctypes.c_void_p(0x200000), ctypes.c_void_p(0x400000), ctypes.c_void_p(0x800000)
    assert lib.tm_pertoken_swiglu(x, None, A.TM_LAYOUT_MIXED, ctypes.byref(bad), None, ctypes.byref(w), y, ws, 1 << 30,
                                  None) == A.TM_ERR_INVALID_ARG
    # workspace too small
    assert lib.tm_pertoken_swiglu(x, None, A.TM_LAYOUT_MIXED, ctypes.byref(good), None, ctypes.byref(w), y, ws, 16,
                                  None) == A.TM_ERR_WORKSPACE
    # misaligned output
    assert lib.tm_pertoken_swiglu(x, None, A.TM_LAYOUT_MIXED, ctypes.byref(good), None, ctypes.byref(w),
                                  ctypes.c_void_p(0x400002), ws, 1 << 30, None) == A.TM_ERR_INVALID_ARG
    # mixed layout needs banks == H
    w2 = A.tm_swiglu_w(cfg.H + 1, cfg.W, 1024, 0x100000, 0x200000, 0x300000)
    assert lib.tm_pertoken_swiglu(x, None, A.TM_LAYOUT_MIXED, ctypes.byref(good), None, ctypes.byref(w2), y, ws,
                                  1 << 30, None) == A.TM_ERR_INVALID_ARG
    # hidden not a multiple of the 64-wide K slab
    w3 = A.tm_swiglu_w(cfg.H, cfg.W, 1000, 0x100000, 0x200000, 0x300000)
    assert lib.tm_pertoken_swiglu(x, None, A.TM_LAYOUT_MIXED, ctypes.byref(good), None, ctypes.byref(w3), y, ws,
                                  1 << 30, None) == A.TM_ERR_UNSUPPORTED
    # MoE: k > E
    mcfg = S.CONFIGS["moe_stack_bf16"]
    msub = _fake_sub(mcfg, 0)
    mw = msub.moe_c()
    mw.k = 9
    msh = api.config_shape(mcfg)
    assert lib.tm_sparse_pertoken_moe(x, None, A.TM_LAYOUT_MIXED, ctypes.byref(msh), None, ctypes.byref(mw), y, ws,
                                      1 << 30, None) == A.TM_ERR_INVALID_ARG
    # stack: bad gap / L
    blocks = (A.tm_block * 1)(api.Block(sub, _fake_sub(cfg, 1)).c())
    assert lib.tm_stack_forward(x, blocks, 0, 0, ctypes.byref(good), y, ws, 1 << 30, None) == A.TM_ERR_INVALID_ARG
    assert lib.tm_stack_forward(x, blocks, 1, 0, ctypes.byref(good), x, ws, 1 << 30, None) == A.TM_ERR_INVALID_ARG


def test_backward_queries_and_validation():
    lib = A.load()
    cfg = S.CONFIGS["dense_block_bf16"]
    sh = api.config_shape(cfg)
    mix, rev = _fake_sub(cfg, 0), _fake_sub(cfg, 1)
    w = mix.dense_c()
    n = lib.tm_pertoken_swiglu_backward_workspace_bytes(ctypes.byref(sh), A.TM_LAYOUT_MIXED, ctypes.byref(w))
    rows = cfg.B * cfg.H
    assert n >= rows * (5 * cfg.W + 9 * 1024) * 2        # the bf16 copies and transposed operands
    blk = api.Block(mix, rev).c()
    nb = lib.tm_block_backward_workspace_bytes(ctypes.byref(sh), ctypes.byref(blk))
    assert nb >= n + 2 * cfg.B * cfg.T * cfg.D * 2
    x, dy, dx, ws = (ctypes.c_void_p(a) for a in (0x200000, 0x400000, 0x600000, 0x800000))
    g = A.tm_swiglu_grads(0x1000000, 0x2000000, 0x3000000)
    call = lambda **kw: lib.tm_pertoken_swiglu_backward(
        kw.get("x", x), kw.get("dy", dy), None, kw.get("layout", A.TM_LAYOUT_MIXED), ctypes.byref(kw.get("sh", sh)),
        kw.get("gain", None), ctypes.byref(kw.get("w", w)), kw.get("dx", dx), ctypes.byref(kw.get("g", g)), ws,
        kw.get("wsb", 1 << 40), None)
    assert call(wsb=16) == A.TM_ERR_WORKSPACE
    assert call(gain=ctypes.c_void_p(0x900000)) == A.TM_ERR_UNSUPPORTED       # RMSNorm gain: forward only
    assert call(sh=api.shape(cfg.B, cfg.T, cfg.D, cfg.H, "fp32")) == A.TM_ERR_UNSUPPORTED
    assert call(w=A.tm_swiglu_w(cfg.H, cfg.W, 960, 0x100000, 0x200000, 0x300000)) == A.TM_ERR_UNSUPPORTED
    assert call(dx=x) == A.TM_ERR_INVALID_ARG                                 # dx aliases x
    assert call(dx=ctypes.c_void_p(0x600008)) == A.TM_ERR_INVALID_ARG         # misaligned
    assert call(g=A.tm_swiglu_grads(0x1000000, None, 0x3000000)) == A.TM_ERR_INVALID_ARG
    # MoE blocks have no backward here
    mcfg = S.CONFIGS["moe_stack_bf16"]
    mblk = api.Block(_fake_sub(mcfg, 0), _fake_sub(mcfg, 1)).c()
    msh = api.config_shape(mcfg)
    assert lib.tm_block_backward_workspace_bytes(ctypes.byref(msh), ctypes.byref(mblk)) == 0
    bg = A.tm_block_grads(g, g)
    assert lib.tm_block_backward(x, dy, ctypes.byref(mblk), ctypes.byref(msh), dx, ctypes.byref(bg), ws, 1 << 40,
                                 None) == A.TM_ERR_UNSUPPORTED
    assert lib.tm_block_backward(x, dy, ctypes.byref(blk), ctypes.byref(sh), dx, ctypes.byref(bg), ws, 16,
                                 None) == A.TM_ERR_WORKSPACE


def test_stack_backward_queries():
    lib = A.load()
    cfg = S.CONFIGS["dense_block_bf16"]
    sh = api.config_shape(cfg)
    blk = api.Block(_fake_sub(cfg, 0), _fake_sub(cfg, 1)).c()
    one = lib.tm_block_backward_workspace_bytes(ctypes.byref(sh), ctypes.byref(blk))
    arr = (A.tm_block * 4)(*[blk] * 4)
    four = lib.tm_stack_backward_workspace_bytes(ctypes.byref(sh), arr, 4, 2)
    tok = cfg.B * cfg.T * cfg.D * 2
    assert four >= one + 6 * tok                       # X_1..X_3 and their gradients
    assert lib.tm_stack_backward_workspace_bytes(ctypes.byref(sh), arr, 0, 2) == 0
    mcfg = S.CONFIGS["moe_stack_bf16"]
    marr = (A.tm_block * 1)(api.Block(_fake_sub(mcfg, 0), _fake_sub(mcfg, 1)).c())
    msh = api.config_shape(mcfg)
    assert lib.tm_stack_backward_workspace_bytes(ctypes.byref(msh), marr, 1, 0) == 0
    g = A.tm_swiglu_grads(0x1000000, 0x2000000, 0x3000000)
    garr = (A.tm_block_grads * 4)(*[A.tm_block_grads(g, g)] * 4)
    x, dy, dx, ws = (ctypes.c_void_p(a) for a in (0x200000, 0x400000, 0x600000, 0x800000))
    assert lib.tm_stack_backward(x, dy, arr, 4, 2, ctypes.byref(sh), dx, garr, ws, 16, None) == A.TM_ERR_WORKSPACE
    assert lib.tm_stack_backward(x, dy, arr, 4, 2, ctypes.byref(sh), x, garr, ws, 1 << 40, None) == A.TM_ERR_INVALID_ARG


def test_plain_c_client_links_and_calls(tmp_path):
    """A C program (no Python, no torch) includes tm.h, links libtm.so and gets answers from the
    host-side calls: version, status strings, workspace sizes and argument validation."""
    src = tmp_path / "client.c"
    src.write_text(r'''
#include <stdio.h>
#include "tm.h"
int main(void) {
  tm_shape s = {4096, 16, 256, 16, TM_BF16, 1e-6f};
  tm_swiglu_w mix = {16, 256, 1024, (void*)0x100000, (void*)0x200000, (void*)0x300000};
  tm_swiglu_w rev = {16, 256, 1024, (void*)0x400000, (void*)0x500000, (void*)0x600000};
  tm_block b = {{0, 0, mix}, {0, 0, rev}};
  size_t ws = tm_workspace_bytes(&s, &b, 1, 0);
  size_t bw = tm_block_backward_workspace_bytes(&s, &b);
  tm_shape bad = s; bad.D = 250;
  tm_status st = tm_pertoken_swiglu((void*)0x700000, 0, TM_LAYOUT_MIXED, &bad, 0, &mix, (void*)0x800000,
                                    (void*)0x900000, (size_t)1 << 30, 0);
  printf("%d %zu %zu %d %s\n", tm_version(), ws, bw, (int)st, tm_status_string(st));
  return 0;
}
''')
    exe = tmp_path / "client"
    libdir = os.path.dirname(A.LIB_PATH)
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L", libdir, "-ltm",
                    "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    assert out[0] == "100"
    assert int(out[1]) > 4096 * 16 * 256 * 2 and int(out[2]) > int(out[1])
    assert int(out[3]) == A.TM_ERR_INVALID_ARG


def _fake_moe8(cfg, sub, hidden_e=None):
    spec = cfg.ffn(sub)
    names = ["w_router", "qe_gate", "qe_up", "se_gate", "se_up", "we_down", "qs_gate", "qs_up", "ss_gate", "ss_up",
             "ws_down"]
    t = {n: _FakeTensor(0x100000 * (i + 1)) for i, n in enumerate(names)}
    return api.MoeSubLayer8(cfg.banks(sub), cfg.width(sub), spec.E, spec.k, hidden_e or spec.hidden_e, spec.hidden_s,
                            spec.alpha, t)


@pytest.mark.parametrize("name", ["moe_stack_bf16", "large_moe_stack_bf16"])
def test_fp8_moe_workspace_and_validation(name):
    """The FP8 MoE sub-layer's workspace query and host checks (no launch): the bf16 MoE workspace
    plus one fp32 row factor per row; unsupported hidden widths and misaligned pointers are refused."""
    lib = A.load()
    cfg = S.CONFIGS[name]
    sh = api.config_shape(cfg)
    for sub, layout in ((0, A.TM_LAYOUT_MIXED), (1, A.TM_LAYOUT_ROWS)):
        s8 = _fake_moe8(cfg, sub)
        n8 = api.sublayer_fp8_workspace_bytes(sh, layout, s8)
        n16 = api.sublayer_workspace_bytes(sh, layout, _fake_sub(cfg, sub))
        assert n16 < n8 <= n16 + cfg.B * cfg.banks(sub) * 4 + 512
        c = s8.sub_c()
        x, y, ws = ctypes.c_void_p(0x200000), ctypes.c_void_p(0x400000), ctypes.c_void_p(0x800000)
        assert lib.tm_sublayer_forward_fp8(x, None, None, layout, ctypes.byref(sh), ctypes.byref(c), y, ws, 16,
                                           None) == A.TM_ERR_WORKSPACE
        assert lib.tm_sublayer_forward_fp8(x, None, None, layout, ctypes.byref(sh), ctypes.byref(c),
                                           ctypes.c_void_p(0x400002), ws, n8, None) == A.TM_ERR_INVALID_ARG
        bad = _fake_moe8(cfg, sub, hidden_e=64).sub_c()
        assert lib.tm_sublayer_fp8_workspace_bytes(ctypes.byref(sh), layout, ctypes.byref(bad)) == 0
        assert lib.tm_sublayer_forward_fp8(x, None, None, layout, ctypes.byref(sh), ctypes.byref(bad), y, ws, n8,
                                           None) == A.TM_ERR_UNSUPPORTED


def test_tp_exchange_layout_validation():
    """tm_tp_exchange_layout refuses bad arguments on the host, before any launch."""
    lib = A.load()
    src, dst = ctypes.c_void_p(0x200000), ctypes.c_void_p(0x400000)
    bad = [
        (src, dst, 0, 4, 2, 64, A.TM_BF16, A.TM_TP_TOKEN_SHARD, 1),      # P < 1
        (src, src, 2, 4, 2, 64, A.TM_BF16, A.TM_TP_TOKEN_SHARD, 1),      # in place
        (src, dst, 2, 4, 2, 64, A.TM_BF16, 7, 1),                        # unknown layout
        (src, dst, 2, 4, 2, 64, 5, A.TM_TP_HEAD_SHARD, 0),               # unknown dtype
        (ctypes.c_void_p(0x200002), dst, 2, 4, 2, 64, A.TM_BF16, A.TM_TP_HEAD_SHARD, 0),   # misaligned
        (None, dst, 2, 4, 2, 64, A.TM_F32, A.TM_TP_HEAD_SHARD, 0),       # null
        (src, ctypes.c_void_p(0x400002), 2, 4, 2, 3, A.TM_F32, A.TM_TP_TOKEN_SHARD, 1),  # f32 element path, 2-byte aligned
        (ctypes.c_void_p(0x200001), dst, 2, 4, 2, 3, A.TM_BF16, A.TM_TP_TOKEN_SHARD, 0),  # bf16 element path, odd address
    ]
    for args in bad:
        assert lib.tm_tp_exchange_layout(*args, None) == A.TM_ERR_INVALID_ARG, args


def test_empty_batch_is_refused_everywhere():
    """B = 0 (an empty batch) is an invalid shape for every entry point that takes one, refused on
    the host before any launch; so are a non-positive token count and an eps that is negative."""
    lib = A.load()
    cfg = S.CONFIGS["moe_stack_bf16"]
    x, y, ws = ctypes.c_void_p(0x200000), ctypes.c_void_p(0x400000), ctypes.c_void_p(0x800000)
    for bad in (api.shape(0, cfg.T, cfg.D, cfg.H, "bf16"), api.shape(cfg.B, 0, cfg.D, cfg.H, "bf16"),
                api.shape(cfg.B, cfg.T, cfg.D, cfg.H, "bf16", eps=-1.0)):
        blk = A.tm_block(_fake_sub(cfg, 0).c(), _fake_sub(cfg, 1).c())
        assert lib.tm_stack_forward(x, ctypes.byref(blk), 1, 0, ctypes.byref(bad), y, ws, 1 << 30,
                                    None) == A.TM_ERR_INVALID_ARG
        assert lib.tm_block_forward(x, ctypes.byref(blk), ctypes.byref(bad), y, None, ws, 1 << 30,
                                    None) == A.TM_ERR_INVALID_ARG
        mw = _fake_sub(cfg, 1).moe_c()
        assert lib.tm_sparse_pertoken_moe(x, None, A.TM_LAYOUT_ROWS, ctypes.byref(bad), None, ctypes.byref(mw), y, ws,
                                          1 << 30, None) == A.TM_ERR_INVALID_ARG
        s8 = _fake_moe8(cfg, 1).sub_c()
        assert lib.tm_sublayer_forward_fp8(x, None, None, A.TM_LAYOUT_ROWS, ctypes.byref(bad), ctypes.byref(s8), y, ws,
                                           1 << 30, None) == A.TM_ERR_INVALID_ARG
        assert lib.tm_sublayer_fp8_workspace_bytes(ctypes.byref(bad), A.TM_LAYOUT_ROWS, ctypes.byref(s8)) == 0
        assert lib.tm_route_workspace_bytes(ctypes.byref(bad), A.TM_LAYOUT_ROWS, ctypes.byref(mw)) == 0


def test_elementwise_utilities_refuse_misaligned_pointers():
    """tm_mix, tm_revert and tm_tokenize_stub take element-aligned pointers; one that is not aligned
    to its element is refused on the host (an element-wise kernel would fault on it)."""
    lib = A.load()
    a, b = ctypes.c_void_p(0x200000), ctypes.c_void_p(0x400000)
    for dtype, off in (("f32", 2), ("bf16", 1)):
        sh = api.shape(4, 8, 16, 4, dtype)
        odd = ctypes.c_void_p(0x400000 + off)
        assert lib.tm_mix(a, odd, ctypes.byref(sh), None) == A.TM_ERR_INVALID_ARG
        assert lib.tm_revert(odd, b, ctypes.byref(sh), None) == A.TM_ERR_INVALID_ARG
        assert lib.tm_tokenize_stub(a, a, a, 4, ctypes.byref(sh), odd, None) == A.TM_ERR_INVALID_ARG
        assert lib.tm_tokenize_stub(odd, a, a, 4, ctypes.byref(sh), b, None) == A.TM_ERR_INVALID_ARG


def test_sizes_past_32_bit_indexing_are_unsupported():
    """Shapes whose per-sample element count or per-sub-layer row count would overflow the kernels'
    32-bit indices and tensor-map coordinates are refused on the host as unsupported."""
    lib = A.load()
    a, b = ctypes.c_void_p(0x200000), ctypes.c_void_p(0x400000)
    wide = api.shape(2, 65536, 65536, 64, "bf16")          # T * D = 2^32 elements per sample
    assert lib.tm_mix(a, b, ctypes.byref(wide), None) == A.TM_ERR_UNSUPPORTED
    cfg = S.CONFIGS["moe_stack_bf16"]
    many = api.shape((1 << 28) // cfg.T + 1, cfg.T, cfg.D, cfg.H, "bf16")   # B * T > 2^28 rows
    blk = A.tm_block(_fake_sub(cfg, 0).c(), _fake_sub(cfg, 1).c())
    assert lib.tm_workspace_bytes(ctypes.byref(many), ctypes.byref(blk), 1, 0) == 0
    assert lib.tm_block_forward(a, ctypes.byref(blk), ctypes.byref(many), b, None, a, 1 << 30,
                                None) == A.TM_ERR_UNSUPPORTED
    ok = api.shape((1 << 28) // cfg.T, cfg.T, cfg.D, cfg.H, "bf16")
    assert lib.tm_workspace_bytes(ctypes.byref(ok), ctypes.byref(blk), 1, 0) > 0


def test_binding_refuses_host_tensors_and_strided_views():
    """The binding passes only addresses of dense device tensors to the library: a host tensor or a
    strided view raises before any call (a tensor that claims to be on the device stands in for one
    here); a slice along the leading axis is dense and passes."""
    import torch

    class _OnDevice(torch.Tensor):
        @property
        def is_cuda(self):
            return True

    with pytest.raises(ValueError, match="device"):
        api._p(torch.zeros(4))
    with pytest.raises(ValueError, match="contiguous"):
        api._p(torch.zeros(4, 6).t().as_subclass(_OnDevice))
    rows = torch.zeros(4, 6).as_subclass(_OnDevice)
    assert api._p(rows[1:3]).value == rows.data_ptr() + 6 * 4
    assert api._p(None) is None
    assert api._p(_FakeTensor(0x1230)).value == 0x1230


def test_moe_without_shared_expert_routes_but_has_no_forward():
    """hidden_s = 0 (no shared expert): tm_route_topk takes it (its workspace query answers), every
    forward call refuses it as unsupported before any launch."""
    lib = A.load()
    cfg = S.CONFIGS["moe_stack_bf16"]
    spec = cfg.ffn(1)
    x, y, ws = ctypes.c_void_p(0x200000), ctypes.c_void_p(0x400000), ctypes.c_void_p(0x800000)
    sh = api.shape(cfg.B, cfg.T, cfg.D, cfg.H, "bf16")
    w = A.tm_moe_w(cfg.T, cfg.D, spec.E, spec.k, spec.hidden_e, 0, spec.alpha, 0x100000, 0x200000, 0x300000, 0x400000,
                   None, None, None)
    assert lib.tm_route_workspace_bytes(ctypes.byref(sh), A.TM_LAYOUT_ROWS, ctypes.byref(w)) > 0
    assert lib.tm_sublayer_workspace_bytes(ctypes.byref(sh), A.TM_LAYOUT_ROWS,
                                           ctypes.byref(A.tm_sublayer(None, 1, A.tm_swiglu_w(), w))) == 0
    assert lib.tm_sparse_pertoken_moe(x, None, A.TM_LAYOUT_ROWS, ctypes.byref(sh), None, ctypes.byref(w), y, ws,
                                      1 << 30, None) == A.TM_ERR_UNSUPPORTED
    sub = A.tm_sublayer(None, 1, A.tm_swiglu_w(), w)
    assert lib.tm_sublayer_forward(x, None, None, A.TM_LAYOUT_ROWS, ctypes.byref(sh), ctypes.byref(sub), y, ws,
                                   1 << 30, None) == A.TM_ERR_UNSUPPORTED


def test_bf16_moe_on_mixed_rows_with_narrow_heads_is_refused_before_launch():
    """A bf16 MoE sub-layer on mixed rows whose head width is not a multiple of 16 (here 8) is
    refused by the host checks (its combine reads the residual through a tensor map); the router
    alone still takes those rows."""
    lib = A.load()
    T, D, H, E, k = 8, 64, 8, 4, 2
    W = T * D // H
    x, y, ws = ctypes.c_void_p(0x200000), ctypes.c_void_p(0x400000), ctypes.c_void_p(0x800000)
    sh = api.shape(256, T, D, H, "bf16")
    w = A.tm_moe_w(H, W, E, k, 64, 64, 2.0, 0x100000, 0x200000, 0x300000, 0x400000, 0x500000, 0x600000, 0x700000)
    sub = A.tm_sublayer(None, 1, A.tm_swiglu_w(), w)
    assert lib.tm_route_workspace_bytes(ctypes.byref(sh), A.TM_LAYOUT_MIXED, ctypes.byref(w)) > 0
    assert lib.tm_sublayer_workspace_bytes(ctypes.byref(sh), A.TM_LAYOUT_MIXED, ctypes.byref(sub)) == 0
    assert lib.tm_sparse_pertoken_moe(x, None, A.TM_LAYOUT_MIXED, ctypes.byref(sh), None, ctypes.byref(w), y, ws,
                                      1 << 30, None) == A.TM_ERR_UNSUPPORTED
    # the same shapes on rows (the reverting layout) pass the checks: only the workspace is short
    wr = A.tm_moe_w(T, D, E, k, 64, 64, 2.0, 0x100000, 0x200000, 0x300000, 0x400000, 0x500000, 0x600000, 0x700000)
    assert lib.tm_sparse_pertoken_moe(x, None, A.TM_LAYOUT_ROWS, ctypes.byref(sh), None, ctypes.byref(wr), y, ws,
                                      16, None) == A.TM_ERR_WORKSPACE

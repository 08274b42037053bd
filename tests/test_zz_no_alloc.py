"""The routing entry point that allocates nothing (tm_route_topk_noalloc).

It serves callers that cannot allocate device memory themselves -- a host framework that
gives this library only its input and output buffers, or a serving loop that reserves all
memory at start-up.  Its scratch is a fixed array inside the library, so this file checks
that it gives exactly what the workspace entry point (tm_route_topk) gives, on two calls in
a row with different shapes (the second call finds the first call's leftovers in the array),
and that a problem too large for the array is refused before any launch.  pytest collects
this file last; it must pass on its own in a fresh process as well.
"""
import ctypes

import pytest
import torch

import tm_synth as S
from tm_synth import FFNSpec
from token_sparse_moe_b200 import api
from token_sparse_moe_b200 import _abi as A

DEV = "cuda:0"


def _case(B, T, D, H, E, k, layout):
    spec = FFNSpec("moe", E=E, k=k, hidden_e=64, hidden_s=64, alpha=float(E) / k)
    cfg = S.Config("noalloc", B=B, T=T, D=D, H=H, L=1, dtype="bf16", mix=spec, rev=spec)
    sub = 0 if layout == A.TM_LAYOUT_MIXED else 1
    return cfg, api.sublayer_from_synth(cfg, 0, sub, DEV)


@pytest.mark.gpu
def test_noalloc_routing_matches_workspace_routing_on_two_calls():
    # tensor-core router (E <= 21, bf16 rows through a tensor map) on two shapes in a row, then the
    # CUDA-core router (E = 32), whose scratch holds only the counts and the tile prefix
    layouts = [A.TM_LAYOUT_MIXED, A.TM_LAYOUT_ROWS, A.TM_LAYOUT_ROWS]
    cases = [_case(300, 16, 256, 16, 8, 2, layouts[0]),
             _case(170, 8, 384, 4, 16, 4, layouts[1]),
             _case(210, 8, 256, 8, 32, 4, layouts[2])]
    for (cfg, sw), layout in zip(cases, layouts):
        x = api.to_device(S.make_x(cfg), DEV)
        sh = api.config_shape(cfg)
        got = api.route_topk_noalloc(x, layout, sh, sw)
        api.get_device_error()
        ref = api.route_topk(x, layout, sh, sw)
        api.get_device_error()
        for key in ("idx", "offsets", "rows", "slot_of"):
            assert torch.equal(got[key], ref[key]), key
        for key in ("gate", "gap", "inv_rms"):       # same kernels on the same input: the same bits
            assert torch.equal(got[key], ref[key]), key


def test_noalloc_routing_refuses_problems_beyond_its_scratch():
    # host-side check: refused before any launch, so this runs without a GPU too
    # 48 banks x 16 experts x ceil(400000/128) chunks of int32 counts is 9.6 MB > 8 MiB
    B, T, D, H, E = 400000, 48, 768, 48, 16
    spec = FFNSpec("moe", E=E, k=4, hidden_e=64, hidden_s=64, alpha=4.0)
    cfg = S.Config("too_big", B=B, T=T, D=D, H=H, L=1, dtype="bf16", mix=spec, rev=spec)
    sh = api.config_shape(cfg)
    fake = {n: ctypes.c_void_p(0x1000 * (i + 1)) for i, n in enumerate(
        ["x", "r", "wg", "wu", "wd", "sg", "su", "sd", "idx", "gate", "inv", "off", "rows", "slot"])}
    w = A.tm_moe_w(H, T * D // H, E, 4, 64, 64, 4.0, fake["r"], fake["wg"], fake["wu"], fake["wd"], fake["sg"],
                   fake["su"], fake["sd"])
    st = api.lib().tm_route_topk_noalloc(fake["x"], A.TM_LAYOUT_MIXED, ctypes.byref(sh), None, ctypes.byref(w),
                                         fake["idx"], fake["gate"], None, fake["inv"], fake["off"], fake["rows"],
                                         fake["slot"], None)
    assert st == A.TM_ERR_WORKSPACE
    assert b"fixed limit" in api.lib().tm_last_cuda_error()

"""Token Parallel on one GPU: P ranks' shards run in one process on the library's kernels (the
all-to-all becomes a transpose of the ranks' chunks).  Each rank computes its heads' mixing rows
and its tokens' reverting rows with tm_sublayer_forward; reassembled, the result must be the same
bits as tm_stack_forward over the whole model, since every row is computed by the same kernels on
the same data."""
import pytest
import torch

import tm_synth as S
from tm_synth import FFNSpec
from token_sparse_moe_b200 import api
from token_sparse_moe_b200 import token_parallel as TP

pytestmark = pytest.mark.gpu
DEV = "cuda:0"

CASES = [
    S.Config("tp_moe", B=300, T=16, D=256, H=16, L=3, gap=2, dtype="bf16",
             mix=FFNSpec("moe", E=8, k=2, hidden_e=128, hidden_s=128, alpha=4.0),
             rev=FFNSpec("moe", E=8, k=2, hidden_e=128, hidden_s=128, alpha=4.0)),
    S.Config("tp_dense", B=200, T=16, D=256, H=16, L=2, gap=1, dtype="bf16",
             mix=FFNSpec("dense", hidden=256), rev=FFNSpec("dense", hidden=384)),
]


@pytest.mark.parametrize("P", [2, 4])
@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_token_parallel_shards_reproduce_the_stack(cfg, P):
    blocks = api.blocks_from_synth(cfg, DEV)
    sh = api.config_shape(cfg)
    X = api.to_device(S.make_x(cfg), DEV)
    Y = api.stack_forward(X, blocks, cfg.gap, sh)
    plan = TP.ShardPlan(cfg.T, cfg.D, cfg.H, P)
    stages = [TP.RankStage(blocks, plan, p, sh, DEV) for p in range(P)]
    xs = [X[:, slice(*plan.tokens(p))].contiguous() for p in range(P)]
    ys = TP.forward_all_ranks(stages, plan, xs, cfg.L, cfg.gap)
    api.get_device_error()
    Yp = torch.cat(ys, dim=1)
    assert torch.equal(Yp.view(torch.int16), Y.view(torch.int16))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T,D,H,P", [(16, 256, 16, 4), (6, 12, 3, 3), (48, 768, 48, 2), (10, 40, 10, 5)])
def test_exchange_layouts_match_the_host_permutation(T, D, H, P, dtype):
    """tm_tp_exchange_layout in all four uses against the host permutation, bit for bit (16-byte
    pieces when a chunk row is a multiple of 16 bytes, single elements otherwise)."""
    from test_token_parallel import HostLayouts
    plan = TP.ShardPlan(T, D, H, P)
    B = 37
    g = torch.Generator().manual_seed(T * 1000 + D)
    x = torch.randn((B, plan.Tp, D), generator=g).to(dtype)
    r = torch.randn((B, T, plan.Dp), generator=g).to(dtype)
    e = torch.randn((P, B, plan.Tp, plan.Dp), generator=g).to(dtype)
    L = TP.LibraryLayouts
    for fn, arg in (("pack_for_heads", x), ("unpack_heads", e), ("pack_for_tokens", r), ("unpack_tokens", e)):
        want = getattr(HostLayouts, fn)(plan, arg)
        got = getattr(L, fn)(plan, arg.to(DEV))
        torch.cuda.synchronize()
        assert torch.equal(got.cpu(), want), fn


def test_rank_stage_runs_sample_chunks():
    """A rank's sub-layers on a chunk of its samples (the overlapped schedule's unit of work) give
    the bits of the same rows in the whole-batch call."""
    cfg = CASES[0]
    blocks = api.blocks_from_synth(cfg, DEV)
    sh = api.config_shape(cfg)
    plan = TP.ShardPlan(cfg.T, cfg.D, cfg.H, 2)
    st = TP.RankStage(blocks, plan, 1, sh, DEV)
    g = torch.Generator().manual_seed(5)
    G = torch.randn((cfg.B, plan.T, plan.Dp), generator=g).to(torch.bfloat16).to(DEV)
    Xr = torch.randn((cfg.B, plan.Tp, plan.D), generator=g).to(torch.bfloat16).to(DEV)
    x = torch.randn((cfg.B, plan.Tp, plan.D), generator=g).to(torch.bfloat16).to(DEV)
    R = st.mixing(0, G).clone()
    Y = st.reverting(0, Xr, x, None).clone()
    a, b = 37, 211
    Rc = st.mixing(0, G[a:b].contiguous())
    Yc = st.reverting(0, Xr[a:b].contiguous(), x[a:b].contiguous(), None)
    api.get_device_error()
    assert torch.equal(Rc.view(torch.int16), R[a:b].view(torch.int16))
    assert torch.equal(Yc.view(torch.int16), Y[a:b].view(torch.int16))

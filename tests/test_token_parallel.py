"""Token Parallel on the CPU: two or three gloo ranks exchange their shards with all_to_all_single.

Each rank holds its share of the tokens and of the heads of a small stack and runs the exchange
schedule and shard packing of token_sparse_moe_b200.token_parallel; the compute of each rank's
sub-layers is the float64 oracle here (this test has no GPU), with the model's bf16 storage
rounding.  Gathered over the ranks, the result must equal the oracle's unsharded stack exactly:
every row sees the same data and weights either way."""
import os

import numpy as np
import pytest
import torch

import oracle
import tm_synth as S
from oracle import tokenmixer as O
from tm_synth import FFNSpec
from token_sparse_moe_b200 import token_parallel as TP


class HostLayouts:
    """The four packing maps of the two exchanges as host permutations of CPU tensors (the ranks of
    this test compute on the CPU; the library's tm_tp_exchange_layout is the device form, checked
    against this one bit for bit in the GPU tests)."""

    @staticmethod
    def pack_for_heads(plan, x_local):
        B = x_local.shape[0]
        return x_local.reshape(B, plan.Tp, plan.P, plan.Dp).permute(2, 0, 1, 3).contiguous()

    @staticmethod
    def unpack_heads(plan, recv):
        B = recv.shape[1]
        return recv.permute(1, 0, 2, 3).reshape(B, plan.T, plan.Dp).contiguous()

    @staticmethod
    def pack_for_tokens(plan, r_local):
        B = r_local.shape[0]
        return r_local.reshape(B, plan.P, plan.Tp, plan.Dp).permute(1, 0, 2, 3).contiguous()

    @staticmethod
    def unpack_tokens(plan, recv):
        B = recv.shape[1]
        return recv.permute(1, 2, 0, 3).reshape(B, plan.Tp, plan.D).contiguous()


class OracleStage:
    """A rank's two sub-layer computations done by the oracle (float64 torch tensors in and out)."""

    def __init__(self, cfg, plan, rank):
        self.cfg, self.plan = cfg, plan
        self.h0, _ = plan.heads(rank)
        self.t0, _ = plan.tokens(rank)
        self.get = oracle.synth_banks(cfg)
        self.rnd = O.storage_round(cfg.dtype)

    def mixing(self, l, G):
        g = G.numpy()
        rows = O.mix(g, self.plan.Hp)
        out = O.sublayer(rows, lambda j: self.get(l, 0, self.h0 + j), self.cfg.mix, self.cfg.eps)["out"]
        return torch.from_numpy(self.rnd(O.revert(out + rows, self.plan.T)))

    def reverting(self, l, Xr, x, extra):
        out = O.sublayer(Xr.numpy(), lambda j: self.get(l, 1, self.t0 + j), self.cfg.rev, self.cfg.eps)["out"]
        y = out + x.numpy() + (extra.numpy() if extra is not None else 0.0)
        return torch.from_numpy(self.rnd(y))


def _cfg(kind):
    if kind == "moe3":
        # three ranks: 6 tokens and 6 heads, two of each per rank
        spec = FFNSpec("moe", E=3, k=2, hidden_e=16, hidden_s=16, alpha=1.5)
        return S.Config("tp_moe3", B=18, T=6, D=24, H=6, L=2, gap=1, dtype="bf16", mix=spec, rev=spec)
    if kind == "moe":
        spec = FFNSpec("moe", E=4, k=2, hidden_e=16, hidden_s=16, alpha=2.0)
        # 25 samples: the overlapped schedule's three chunks are ragged (8, 8, 9)
        return S.Config("tp_moe", B=25, T=4, D=32, H=4, L=3, gap=2, dtype="bf16", mix=spec, rev=spec)
    return S.Config("tp_dense", B=24, T=4, D=32, H=2, L=2, gap=1, dtype="bf16",
                    mix=FFNSpec("dense", hidden=32), rev=FFNSpec("dense", hidden=16))


def _rank(rank, world, kind, port, out_path, overlapped=False):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = _cfg(kind)
        plan = TP.ShardPlan(cfg.T, cfg.D, cfg.H, world)
        X = torch.from_numpy(S.to_f64(S.make_x(cfg)))
        t0, t1 = plan.tokens(rank)
        if overlapped:
            y = TP.forward_rank_overlapped(OracleStage(cfg, plan, rank), plan, X[:, t0:t1].contiguous(), cfg.L,
                                           cfg.gap, TP.torch_exchange_async(), chunks=3, layouts=HostLayouts)
        else:
            y = TP.forward_rank(OracleStage(cfg, plan, rank), plan, X[:, t0:t1].contiguous(), cfg.L, cfg.gap,
                                TP.torch_exchange(), layouts=HostLayouts)
        parts = [torch.empty_like(y) for _ in range(world)]
        dist.all_gather(parts, y)
        if rank == 0:
            torch.save(torch.cat(parts, dim=1), out_path)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("overlapped", [False, True], ids=["plain", "overlapped"])
@pytest.mark.parametrize("kind", ["moe", "dense", "moe3"])
def test_token_parallel_ranks_equal_the_unsharded_stack(kind, overlapped, tmp_path):
    """Also with the exchanges issued asynchronously in three sample chunks, each chunk's compute
    starting when its own exchange has landed (forward_rank_overlapped); moe3 runs three ranks."""
    import torch.multiprocessing as mp
    out = str(tmp_path / "y.pt")
    world = 3 if kind == "moe3" else 2
    port = 29600 + (os.getpid() % 200) + {"moe": 0, "dense": 1, "moe3": 4}[kind] + (2 if overlapped else 0) * 3
    mp.spawn(_rank, args=(world, kind, port, out, overlapped), nprocs=world, join=True)
    cfg = _cfg(kind)
    ref = oracle.run_stack(cfg, storage=cfg.dtype)["Y"]
    got = torch.load(out).numpy()
    assert got.shape == ref.shape
    assert np.array_equal(got, ref)


def test_shard_plan_and_packing_round_trip():
    """The two exchanges' packing is a pure permutation: packing a rank's data for every rank and
    unpacking what each rank receives moves every element to its place."""
    plan = TP.ShardPlan(T=6, D=12, H=3, P=3)
    B = 2
    X = torch.arange(B * 6 * 12, dtype=torch.float64).reshape(B, 6, 12)
    sends = [HostLayouts.pack_for_heads(plan, X[:, slice(*plan.tokens(q))]) for q in range(3)]
    for p in range(3):
        G = HostLayouts.unpack_heads(plan, torch.stack([sends[q][p] for q in range(3)]))
        c0, c1 = p * plan.Dp, (p + 1) * plan.Dp
        assert torch.equal(G, X[:, :, c0:c1])
    Rs = [X[:, :, p * plan.Dp:(p + 1) * plan.Dp] for p in range(3)]
    sends = [HostLayouts.pack_for_tokens(plan, Rs[q]) for q in range(3)]
    for p in range(3):
        Xr = HostLayouts.unpack_tokens(plan, torch.stack([sends[q][p] for q in range(3)]))
        assert torch.equal(Xr, X[:, slice(*plan.tokens(p))])
    with pytest.raises(ValueError):
        TP.ShardPlan(T=6, D=12, H=4, P=3)
    assert [TP.skip_index(l, 4, 2) for l in range(1, 5)] == [None, 0, None, None]

"""The multi-rank bookkeeping of bench.py on CPU: two gloo ranks, no GPU.

Each rank runs its own batch (weak scaling, no data-path collective); the only collectives are
the barriers around the timed region and the max-over-ranks reduction of the step time."""
import importlib.util
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b = _bench()
        step_ms = 1.0 + rank * 0.25                      # rank 1 is the slow one
        t = b.max_over_ranks(step_ms, world, torch.device("cpu"))
        dist.barrier()
        out[rank] = (t, b.job_throughput(4096, world, t))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(out)
    assert res[0][0] == res[1][0] == pytest.approx(1.25)  # both ranks see the slowest rank's time
    assert res[0][1] == pytest.approx(2 * 4096 / 1.25e-3)  # whole-job samples per second



def test_single_rank_needs_no_process_group():
    b = _bench()
    assert b.max_over_ranks(3.5, 1, None) == 3.5
    assert b.job_throughput(100, 1, 2.0) == pytest.approx(5e4)


def test_each_rank_draws_its_own_batch():
    import tm_synth as S
    b = _bench()
    cfg = S.CONFIGS["tiny_f32_dense"]
    x0 = S.make_x(b.rank_config(cfg, 0), np.arange(4))
    x1 = S.make_x(b.rank_config(cfg, 1), np.arange(4))
    assert not np.array_equal(x0, x1)
    assert np.array_equal(x0, S.make_x(cfg, np.arange(4)))   # rank 0 is the workload's own batch


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import argparse
    import tm_synth as S
    b = _bench()
    args = argparse.Namespace(steps_ref=1, warmup=1, ref_samples=2, gpus=2)
    b.run_reference(args, S.CONFIGS["tiny_f32_dense"], rank=1)
    assert capsys.readouterr().out == ""


def test_end_to_end_chunk_bounds():
    """The pipelined end-to-end call's chunks: every sample in exactly one chunk, in order; the ramp
    keeps the first and last chunks at 1/16 of the batch (the copy time left uncovered)."""
    from token_sparse_moe_b200 import api
    assert api.chunk_bounds(16384, api.RAMP_CHUNKS) == [0, 1024, 4096, 12288, 15360, 16384]
    assert api.chunk_bounds(8192, 8) == [1024 * i for i in range(9)]
    assert api.chunk_bounds(9, api.RAMP_CHUNKS) == [0, 9]            # too small to split
    assert api.chunk_bounds(4096, 1) == [0, 4096]
    for B in (13, 100, 333, 4097):
        b = api.chunk_bounds(B, api.RAMP_CHUNKS)
        assert b[0] == 0 and b[-1] == B and all(x < y for x, y in zip(b, b[1:]))

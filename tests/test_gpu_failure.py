"""Device-side failure detection, made to fire without faulting the GPU.

Every wait in the library's kernels is bounded by a wall-clock limit and every index read from
device data is bounds-checked; a failure is recorded in the device error word and the kernel
returns.  Here (a) the wait limit is shortened to 1 ms and the self-test kernel waits on a barrier
that nothing completes: it must come back with TM_ERR_DEVICE_TIMEOUT at its site, and a second wait
made after the abort flag is raised must return at once; (b) the bucketing scatter is given a
host-made table that under-counts the routed rows: the positions past the bucket array must be
reported as TM_ERR_DEVICE_BOUNDS and left unwritten (guard entries past the array keep their
values).  In both cases the context stays usable: an ordinary call afterwards succeeds.
"""

import numpy as np
import pytest
import torch

import tm_synth as S
from parity_util import check_buckets
from tm_synth import FFNSpec
from token_sparse_moe_b200 import api
from token_sparse_moe_b200 import _abi as A

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _ordinary_call_still_works():
    spec = FFNSpec("moe", E=4, k=2, hidden_e=64, hidden_s=64, alpha=2.0)
    cfg = S.Config("after", B=130, T=8, D=128, H=8, L=1, dtype="bf16", mix=spec, rev=spec)
    sw = api.sublayer_from_synth(cfg, 0, 1, DEV)
    r = api.route_topk(api.to_device(S.make_x(cfg), DEV), A.TM_LAYOUT_ROWS, api.config_shape(cfg), sw)
    api.get_device_error()
    idx = r["idx"].cpu().numpy()
    check_buckets(idx, r["offsets"].cpu().numpy(), r["rows"].cpu().numpy(), r["slot_of"].cpu().numpy(), spec.E)


def test_bounded_wait_runs_out_reports_its_site_and_returns():
    lib = api.lib()
    api.get_device_error()                                   # start from a clear error word
    res = torch.zeros(4, dtype=torch.int64, device=DEV)
    limit = 1_000_000                                        # 1 ms
    assert lib.tm_set_wait_limit_ns(limit) == A.TM_OK
    try:
        A.check(lib.tm_selftest_wait(api._p(res), api._s(None)), "tm_selftest_wait")
        st = lib.tm_get_device_error(api._s(None))
        assert st == A.TM_ERR_DEVICE_TIMEOUT
        assert lib.tm_last_device_error_site() == 0x7001
        assert b"0x7001" in lib.tm_last_cuda_error()
        t_wait, failed, t_abort, failed2 = res.cpu().tolist()
        assert failed == 1 and failed2 == 1
        assert limit <= t_wait < 100 * limit                 # it waited out the limit, no longer
        assert t_abort < limit                               # the raised abort flag ends a wait at once
        # the error word was cleared by the read
        assert lib.tm_get_device_error(api._s(None)) == A.TM_OK
        assert lib.tm_last_device_error_site() == 0
    finally:
        assert lib.tm_set_wait_limit_ns(2_000_000_000) == A.TM_OK
    _ordinary_call_still_works()


def test_wait_limit_is_validated_on_the_host():
    lib = api.lib()
    assert lib.tm_set_wait_limit_ns(10) == A.TM_ERR_INVALID_ARG
    assert lib.tm_set_wait_limit_ns(10 ** 12) == A.TM_ERR_INVALID_ARG


def _scatter_tables(B, banks, E, counted):
    """Every row of every bank chooses experts 0 and 1.  The chunk prefix is exact; the group offsets
    come from `counted` rows per (bank, expert) instead of the true ones."""
    nch = (B + 127) // 128
    idx = np.zeros((B, banks, 2), dtype=np.int32)
    idx[..., 1] = 1
    prefix = np.zeros((banks, nch, E), dtype=np.int32)
    for c in range(nch):
        prefix[:, c, :2] = 128 * c
    sizes = counted.reshape(-1)
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    return idx, prefix, offsets


def _run_scatter(idx, prefix, offsets, B, banks, E, capacity, guard=256):
    # the device copies stay referenced until the kernel has run (the caching allocator would hand a
    # freed temporary's memory to the next copy)
    dev = [torch.from_numpy(np.ascontiguousarray(a)).to(DEV) for a in (idx, prefix, offsets)]
    rows = torch.full((capacity + guard,), -7, dtype=torch.int32, device=DEV)
    slot = torch.full((B, banks, 2), -5, dtype=torch.int32, device=DEV)
    A.check(api.lib().tm_selftest_bucket_scatter(api._p(dev[0]), api._p(dev[1]), api._p(dev[2]), B, banks, E, 2,
                                                 api._p(rows), capacity, api._p(slot), api._s(None)),
            "tm_selftest_bucket_scatter")
    torch.cuda.synchronize()
    st = api.lib().tm_get_device_error(api._s(None))
    return st, rows.cpu().numpy(), slot.cpu().numpy()


def test_under_counted_bucket_table_is_reported_and_nothing_is_written_out_of_range():
    B, banks, E = 300, 2, 4
    api.get_device_error()
    true = np.zeros((banks, E), dtype=np.int64)
    true[:, :2] = B
    # the exact table: no error, and the buckets have the structure tm_route_topk guarantees
    idx, prefix, offsets = _scatter_tables(B, banks, E, true)
    cap = int(offsets[-1])
    st, rows, slot = _run_scatter(idx, prefix, offsets, B, banks, E, cap)
    assert st == A.TM_OK
    assert np.all(rows[cap:] == -7)
    check_buckets(idx, offsets, rows[:cap], slot, E)
    # the last non-empty group (bank 1, expert 1) under-counted by 100 rows: its last 100 positions
    # fall past the bucket array (sized by the table's own total)
    bad = true.copy()
    bad[1, 1] -= 100
    idx, prefix, offsets = _scatter_tables(B, banks, E, bad)
    cap = int(offsets[-1])
    assert cap == B * banks * 2 - 100
    st, rows, slot = _run_scatter(idx, prefix, offsets, B, banks, E, cap)
    assert st == A.TM_ERR_DEVICE_BOUNDS
    assert api.lib().tm_last_device_error_site() == 0x501
    assert np.all(rows[cap:] == -7), "a position past the bucket array was written"
    # every in-range position was written with its sample; the refused choices kept no slot
    assert np.all(rows[:cap] >= 0)
    assert np.all(slot[B - 100:, 1, 1] == -5)
    assert np.all(slot[:B - 100, 1, 1] >= 0) and np.all(slot[:, 0, :] >= 0) and np.all(slot[:, 1, 0] >= 0)
    _ordinary_call_still_works()

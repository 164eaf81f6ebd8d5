"""bench.py's multi-rank host logic on CPU with the gloo backend (world size 2):
each rank quantizes its own tables (seed = rank) and the reported time is the
max over ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime
    import torch
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        wl = bench.rank_workload("kaggle", rank)
        got = bench.max_over_ranks(10.0 + 5.0 * rank, torch.device("cpu"))
        q.put((rank, got, wl.rows[:3], wl.seed))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, m0, rows0, s0), (r1, m1, rows1, s1) = res
    assert m0 == m1 == 15.0          # max over ranks
    assert (s0, s1) == (0, 1)        # independent tables per rank
    assert rows0 != rows1


def test_single_process_is_a_noop():
    import torch
    import bench
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5


def _e2e_worker(rank, world, port, q):
    """run_e2e's decision to skip is taken by all ranks together: rank 1 sees no free host
    memory, rank 0 plenty; both must skip (and so take the same collectives)."""
    import datetime
    import types
    import psutil
    import torch
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        if rank == 1:
            psutil.virtual_memory = lambda: types.SimpleNamespace(available=1)
        wl = types.SimpleNamespace(d=16, n_tables=1)
        step = types.SimpleNamespace(cld=8, codes=[torch.zeros(4, 8, dtype=torch.uint8)],
                                     sbs=[torch.zeros(4, 2, dtype=torch.int16)])
        got = bench.run_e2e(None, wl, [torch.zeros(4, 16)], step, torch.device("cpu"), None, world)
        dist.barrier()
        q.put((rank, "skipped" in got))
    finally:
        dist.destroy_process_group()


def test_e2e_skip_is_one_decision_for_all_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_e2e_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(0, True), (1, True)]

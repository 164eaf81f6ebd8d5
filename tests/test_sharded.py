"""Table-wise sharded lookup with the all-to-all of pooled outputs ("Deep Learning
Recommendation Model for Personalization and Recommendation Systems", 提出的方法:
model-parallel tables, data-parallel ranks), as gloo ranks on CPU: every rank's slice
of the batch equals the single-process lookup over all tables, bit for bit. The
per-rank lookup is the oracle's (this host has no GPU); on GPUs it is
dq_embbag_int4_fwd and the exchange runs over NCCL; the GPU tests compare that path with
the oracle's lookup on the same packed tables."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from int4_row_wise_b200.sharded import plan_tables, sharded_embbag

D = 8


def _problem(T, B, seed, d=D, pool=(0, 4)):
    r = np.random.default_rng(seed)
    rows = [int(n) for n in r.integers(0, 400, T)]
    rows[0] = 0 if T > 3 else rows[0]  # an empty table when there are several
    tables = []
    for n in rows:
        x = r.standard_normal((max(n, 1), d)).astype(np.float32)[:n]
        c, sb, _, _ = oracle.quantize_rows(x) if n else (np.zeros((0, (d + 1) // 2), np.uint8),
                                                          np.zeros((0, 2), np.uint16), None, None)
        tables.append((c, sb))
    per_table = []
    for t, n in enumerate(rows):
        lens = r.integers(pool[0], pool[1] + 1, B)
        off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        idx = r.integers(-2, max(n, 1) + 3, off[-1]).astype(np.int32)  # some ids out of range
        per_table.append((idx, off))
    return rows, tables, per_table


def _batch_of(tables_sel, per_table):
    """Table-major indices/offsets over the selected tables."""
    idx, off = [], [0]
    for t in tables_sel:
        i, o = per_table[t]
        idx.append(i)
        off.extend((o[1:] + off[-1]).tolist())
    return (np.concatenate(idx) if idx else np.zeros(0, np.int32)).astype(np.int32), np.array(off, np.int32)


def _oracle_lookup(tables, d, indices, offsets, batch):
    out, _, _ = oracle.embbag([(c, s) for c, s in tables], d, indices.numpy(), offsets.numpy(), batch)
    return torch.from_numpy(out)


def _rank(rank, world, port, T, B, seed, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rows, tables, per_table = _problem(T, B, seed)
        owner = plan_tables(rows, world)
        mine = [t for t in range(T) if owner[t] == rank]
        idx, off = _batch_of(mine, per_table)
        out = sharded_embbag([tables[t] for t in mine], owner, D, torch.from_numpy(idx), torch.from_numpy(off), B,
                             lookup=_oracle_lookup)
        results[rank] = out.numpy().copy()
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,T,B,seed", [(2, 5, 6, 0), (3, 7, 9, 1), (3, 2, 3, 2), (2, 1, 4, 3)])
def test_sharded_lookup_equals_the_single_device_lookup(world, T, B, seed):
    rows, tables, per_table = _problem(T, B, seed)
    idx, off = _batch_of(list(range(T)), per_table)
    want = _oracle_lookup(tables, D, torch.from_numpy(idx), torch.from_numpy(off), B).numpy()
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_rank, args=(world, _free_port(), T, B, seed, results), nprocs=world, start_method="spawn")
    bl = B // world
    for r in range(world):
        assert np.array_equal(results[r].view(np.uint32), want[r * bl:(r + 1) * bl].view(np.uint32)), r


def test_plan_is_deterministic_and_balanced():
    r = np.random.default_rng(5)
    for world in (1, 2, 3, 8):
        rows = [int(n) for n in r.integers(1, 10 ** 6, 26)]
        a, b = plan_tables(rows, world), plan_tables(rows, world)
        assert a == b and set(a) <= set(range(world))
        load = [sum(n for n, o in zip(rows, a) if o == k) for k in range(world)]
        assert max(load) - min(load) <= max(rows)
    assert plan_tables([5, 5, 5], 2) == [0, 1, 0]  # equal loads go to the lower rank


@pytest.fixture(scope="module")
def nccl_one_rank(cuda_device):
    """A one-rank NCCL process group on cuda:0 (every run of this build has one GPU)."""
    import datetime
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    yield
    dist.destroy_process_group()


@pytest.mark.gpu
@pytest.mark.parametrize("d", [16, 64, 128])
@pytest.mark.parametrize("pool", [(1, 1), (4, 12)])
def test_sharded_lookup_on_the_gpu_against_the_oracle(nccl_one_rank, d, pool):
    # the default path on a B200: dq_embbag_int4_fwd (the vectorised embbag_kernel at these
    # widths, one-hot and pooled layouts) and the exchanges over NCCL, both from the global
    # per-table batch and from the rank's own samples routed to the owners; compared with
    # the oracle's lookup on the same packed tables, element by element within
    # 1e-5 * sum|xhat| and bit for bit on bags of one id
    import int4_row_wise_b200 as dq
    from int4_row_wise_b200.sharded import sharded_embbag_local
    from tests.gpu_util import bag_tolerance_check
    T, B = 5, 256
    rows, tables, per_table = _problem(T, B, 7 + d, d=d, pool=pool)
    owner = plan_tables(rows, 1)
    idx, off = _batch_of(list(range(T)), per_table)
    cld = dq._codes_ld(d)
    dt = []
    for c, sb in tables:
        cp = np.zeros((c.shape[0], cld), np.uint8)
        cp[:, :c.shape[1]] = c
        dt.append(dq.PackedTable(torch.from_numpy(cp).cuda(), torch.from_numpy(np.ascontiguousarray(sb).view(np.int16)).cuda()))
    got = sharded_embbag(dt, owner, d, torch.from_numpy(idx).cuda(), torch.from_numpy(off).cuda(), B)
    routed = sharded_embbag_local(dt, owner, d, [(torch.from_numpy(i).cuda(), torch.from_numpy(o).cuda())
                                                 for i, o in per_table], B)
    torch.cuda.synchronize()
    ref, mag, _ = oracle.embbag(tables, d, idx, off, B, with_abs_sum=True)
    lens = np.stack([o[1:] - o[:-1] for _, o in per_table], axis=1)          # [B, T]
    one = np.repeat(lens == 1, d, axis=1)                                      # elements of one-id bags
    # the direct form: the lookup stores every row straight into its owner's buffer
    from int4_row_wise_b200.sharded import OwnerBuffers, sharded_embbag_direct
    bufs = OwnerBuffers.create(B, T * d, torch.device("cuda", 0))
    direct = sharded_embbag_direct(dt, owner, d, torch.from_numpy(idx).cuda(), torch.from_numpy(off).cuda(), B, bufs)
    torch.cuda.synchronize()
    for out in (got, routed, direct):
        o = out.cpu().numpy()
        bag_tolerance_check(o, ref, mag)
        assert np.array_equal(o[one].view(np.uint32), ref[one].view(np.uint32))


def test_sharded_rejects_bad_shapes():
    # a one-rank gloo group: the checks run before any collective
    from int4_row_wise_b200.sharded import sharded_embbag_local
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        rows, tables, per_table = _problem(3, 4, 0)
        owner = plan_tables(rows, 1)
        bt = [(torch.from_numpy(i), torch.from_numpy(o)) for i, o in per_table]
        with pytest.raises(ValueError, match="local_batch"):
            sharded_embbag_local(tables, owner, D, bt, 5, lookup=_oracle_lookup)   # 4 bags, not 5
        with pytest.raises(ValueError, match="no tables"):
            sharded_embbag_local([], [], D, [], 4, lookup=_oracle_lookup)
        with pytest.raises(ValueError, match="batches"):
            sharded_embbag_local(tables, owner, D, bt[:2], 4, lookup=_oracle_lookup)
        idx, off = _batch_of([0, 1, 2], per_table)
        with pytest.raises(ValueError, match="offsets"):
            sharded_embbag(tables, owner, D, torch.from_numpy(idx), torch.from_numpy(off[:-1]), 4,
                           lookup=_oracle_lookup)
        with pytest.raises(ValueError, match="owner ranks"):
            sharded_embbag(tables, [0, 1, 0], D, torch.from_numpy(idx), torch.from_numpy(off), 4,
                           lookup=_oracle_lookup)
        # the direct form checks its buffers, tables and offsets before any barrier or launch
        from int4_row_wise_b200.sharded import OwnerBuffers, sharded_embbag_direct
        ti, to = torch.from_numpy(idx), torch.from_numpy(off)
        good = OwnerBuffers(torch.zeros((4, 3 * D)), [0], [])
        with pytest.raises(ValueError, match="owner buffers"):
            sharded_embbag_direct(tables, owner, D, ti, to, 4, OwnerBuffers(good.own, [0, 0], []))
        with pytest.raises(ValueError, match="own buffer"):
            sharded_embbag_direct(tables, owner, D, ti, to, 4, OwnerBuffers(torch.zeros((4, 2 * D)), [0], []))
        with pytest.raises(ValueError, match="owns 3 tables"):
            sharded_embbag_direct(tables[:2], owner, D, ti, to, 4, good)
        with pytest.raises(ValueError, match="offsets"):
            sharded_embbag_direct(tables, owner, D, ti, to[:-1], 4, good)
        with pytest.raises(ValueError, match="owner ranks"):
            sharded_embbag_direct(tables, [0, 1, 0], D, ti, to, 4, good)
    finally:
        dist.destroy_process_group()


def _local_problem(T, bl, rank, seed):
    """This rank's own bags for every table (its local samples)."""
    r = np.random.default_rng(seed * 1000 + rank)
    rows, tables, _ = _problem(T, 1, seed)
    batches = []
    for n in rows:
        lens = r.integers(0, 5, bl)
        off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        idx = r.integers(-1, max(n, 1) + 2, off[-1]).astype(np.int32)
        batches.append((idx, off))
    return rows, tables, batches


def _rank_local(rank, world, port, T, bl, seed, results):
    from int4_row_wise_b200.sharded import sharded_embbag_local
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rows, tables, batches = _local_problem(T, bl, rank, seed)
        owner = plan_tables(rows, world)
        mine = [t for t in range(T) if owner[t] == rank]
        out = sharded_embbag_local([tables[t] for t in mine], owner, D,
                                   [(torch.from_numpy(i), torch.from_numpy(o)) for i, o in batches], bl,
                                   lookup=_oracle_lookup)
        results[rank] = out.numpy().copy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,T,bl,seed", [(2, 5, 3, 0), (3, 6, 4, 1), (3, 2, 2, 2)])
def test_routed_lookup_from_local_batches(world, T, bl, seed):
    # every rank starts with its own samples' bags for all tables; the ids travel to the
    # owners and the pooled rows back: each rank gets the single-device lookup of its bags
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_rank_local, args=(world, _free_port(), T, bl, seed, results), nprocs=world,
                       start_method="spawn")
    for r in range(world):
        rows, tables, batches = _local_problem(T, bl, r, seed)
        idx, off = _batch_of(list(range(T)), batches)
        want = _oracle_lookup(tables, D, torch.from_numpy(idx), torch.from_numpy(off), bl).numpy()
        assert np.array_equal(results[r].view(np.uint32), want.view(np.uint32)), r


def _rank_bad_args(rank, world, port, which, results):
    import datetime
    from int4_row_wise_b200.sharded import sharded_embbag_local
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    # a short timeout: were the checks not collective, the good rank would wait in the
    # exchange until it ran out, and fail with a timeout instead of a ValueError
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        T, B = 4, 6
        rows, tables, per_table = _problem(T, B, 7)
        owner = plan_tables(rows, world)
        mine = [t for t in range(T) if owner[t] == rank]
        idx, off = _batch_of(mine, per_table)
        ti, to = torch.from_numpy(idx), torch.from_numpy(off)
        try:
            if which == "global":
                if rank == world - 1:
                    to = to[:-1]   # this rank's offsets are one short
                sharded_embbag([tables[t] for t in mine], owner, D, ti, to, B, lookup=_oracle_lookup)
            else:
                bt = [(torch.from_numpy(i), torch.from_numpy(o)) for i, o in per_table]
                lb = B if rank != world - 1 else B - 1   # this rank's batch size disagrees with its offsets
                sharded_embbag_local([tables[t] for t in mine], owner, D, bt, lb, lookup=_oracle_lookup)
            results[rank] = "no error"
        except ValueError as e:
            results[rank] = "ValueError: " + str(e)
        except Exception as e:   # e.g. a collective that timed out
            results[rank] = type(e).__name__ + ": " + str(e)[:200]
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("which", ["global", "local"])
def test_bad_arguments_on_one_rank_fail_every_rank(which):
    world = 2
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_rank_bad_args, args=(world, _free_port(), which, results), nprocs=world,
                       start_method="spawn")
    assert results[world - 1].startswith("ValueError: ") and "another rank" not in results[world - 1], results
    assert results[0] == "ValueError: another rank's arguments failed their checks", results

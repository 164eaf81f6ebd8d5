"""Table-wise sharded lookup: the hybrid parallelism of "Deep Learning Recommendation
Model for Personalization and Recommendation Systems" (section 提出的方法, proposed
method: embedding tables distributed across devices, model-parallel, while the rest
of the model runs data-parallel; the pooled embeddings reach every data-parallel
rank through an all-to-all exchange).

Each rank owns whole tables. For the global batch it looks up its own tables with
dq_embbag_int4_fwd (or an injected lookup), then one all-to-all sends every rank
the rows of its slice of the batch; each rank reassembles [batch / world, T * d] in
table order, exactly what a single device computes for those bags. The exchanges are
torch.distributed's all_to_all_single (NCCL between GPUs).

Host synchronisation: sharded_embbag needs none; sharded_embbag_local reads two small
count arrays back to the host (the all-to-all split sizes must be host integers):
every table's first and last offset before the exchange, and the received per-(source,
table) id counts after the bag lengths have been exchanged.

Direct form (OwnerBuffers): every rank maps all ranks' receive buffers into its address
space (CUDA IPC through torch's storage sharing) and one kernel,
dq_embbag_int4_fwd_to_owners, stores each pooled row straight into its owner's buffer
at its final place: no all-to-all, no reassembly copy. The ranks meet at a barrier
before each call (the owners have read the previous result) and after it (every row
has arrived).
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence

__all__ = ["plan_tables", "sharded_embbag", "sharded_embbag_local", "OwnerBuffers", "sharded_embbag_direct"]


def plan_tables(rows: Sequence[int], world: int) -> List[int]:
    """Owner rank of every table: the largest table first, each to the rank holding
    the fewest rows so far (ties to the lower rank). Deterministic, so every rank
    computes the same plan."""
    if world < 1:
        raise ValueError("world must be >= 1")
    load = [0] * world
    owner = [0] * len(rows)
    for t in sorted(range(len(rows)), key=lambda t: (-int(rows[t]), t)):
        r = min(range(world), key=lambda k: (load[k], k))
        owner[t] = r
        load[r] += int(rows[t])
    return owner


def _check_owner(owner: Sequence[int], world: int) -> None:
    if len(owner) == 0:
        raise ValueError("no tables: the plan is empty")
    bad = [r for r in owner if not 0 <= int(r) < world]
    if bad:
        raise ValueError(f"owner ranks {bad[:4]} outside [0, {world})")


def _agree(err: Optional[str], group, device) -> None:
    """Every rank learns, before any exchange, whether some rank's arguments failed its
    checks (one all-reduce of a flag), and then all of them raise: a rank with bad
    arguments cannot leave the others waiting in an exchange it never joins. Also a
    barrier: it returns once every rank has reached it."""
    import torch
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        if err:
            raise ValueError(err)
        return
    if dist.get_backend(group) != "nccl":
        device = torch.device("cpu")
    flag = torch.tensor([1 if err else 0], dtype=torch.int32, device=device)
    dist.all_reduce(flag, op=dist.ReduceOp.MAX, group=group)
    if err:
        raise ValueError(err)
    if int(flag.item()):
        raise ValueError("another rank's arguments failed their checks")


def _reassemble(recv, owner: Sequence[int], world: int, bl: int, d: int):
    """[bl, T * d] in global table order from the received buffer, which holds, source
    by source, [bl, tables of that source, d]. One concatenation kernel."""
    import torch
    T = len(owner)
    counts = [0] * world
    where = []                       # (source, slot within the source) of every global table
    for t in range(T):
        s = int(owner[t])
        where.append((s, counts[s]))
        counts[s] += 1
    base, at = [], 0
    for s in range(world):
        base.append(at)
        at += bl * counts[s] * d
    chunks = {s: recv[base[s]:base[s] + bl * counts[s] * d].view(bl, counts[s], d)
              for s in range(world) if counts[s]}
    parts = [chunks[s][:, k:k + 1, :] for s, k in where]
    return torch.cat(parts, dim=1).view(bl, T * d)


def sharded_embbag(local_tables: Sequence, owner: Sequence[int], d: int, indices, offsets, global_batch: int,
                   group=None, lookup: Optional[Callable] = None, _checked: bool = False):
    """Pooled outputs of this rank's slice of the global batch, over all tables.

    local_tables  the tables this rank owns, in ascending global table order
    owner         owner rank of every global table (plan_tables)
    indices, offsets   the lookup batch of this rank's tables for the whole global batch
                  (table-major over the owned tables, as dq_embbag_int4_fwd takes them);
                  tensors (a rank without tables passes empty ones on its device)
    global_batch  bags per table, divisible by the world size
    lookup        (tables, d, indices, offsets, batch) -> [batch, len(tables) * d];
                  dq.embbag by default
    Returns a [global_batch // world, T * d] tensor on the tables' device. The argument
    checks are collective: if any rank's fail, every rank raises ValueError."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    mine = [t for t, r in enumerate(owner) if r == rank]
    if not _checked:
        err = None
        try:
            _check_owner(owner, world)
            if global_batch % world:
                raise ValueError(f"global batch {global_batch} is not divisible by the world size {world}")
            if len(mine) != len(local_tables):
                raise ValueError(f"rank {rank} owns {len(mine)} tables by the plan but holds {len(local_tables)}")
            if mine and int(offsets.numel()) != len(mine) * global_batch + 1:
                raise ValueError(f"offsets hold {int(offsets.numel())} entries; {len(mine)} tables x "
                                 f"{global_batch} bags need {len(mine) * global_batch + 1}")
        except ValueError as e:
            err = str(e)
        _agree(err, group, offsets.device)
    if lookup is None:
        import int4_row_wise_b200 as dq
        lookup = dq.embbag
    T = len(owner)
    bl = global_batch // world
    counts = [sum(1 for r in owner if r == s) for s in range(world)]
    if mine:
        # [world * bl, T_own * d], row-major: already destination-major (rank s gets rows s*bl ..)
        send = lookup(local_tables, d, indices, offsets, global_batch).reshape(-1)
        dev, dt = send.device, send.dtype
    else:  # a rank without tables still takes part in the exchange
        dev, dt = offsets.device, torch.float32
        send = torch.empty(0, dtype=dt, device=dev)
    recv = torch.empty(bl * T * d, dtype=dt, device=dev)
    dist.all_to_all_single(recv, send, output_split_sizes=[bl * c * d for c in counts],
                           input_split_sizes=[bl * len(mine) * d] * world, group=group)
    return _reassemble(recv, owner, world, bl, d)


def sharded_embbag_local(local_tables: Sequence, owner: Sequence[int], d: int, batches: Sequence, local_batch: int,
                         group=None, lookup: Optional[Callable] = None):
    """The whole hybrid-parallel lookup from data-parallel inputs: every rank holds the
    bags of its own `local_batch` samples for every table (`batches[t] = (indices,
    offsets)`, offsets of length local_batch + 1, nondecreasing), and gets back
    [local_batch, T * d] for those samples.

    Steps: the bag lengths of every table travel to the table's owner (fixed-size
    all-to-all), then the ids (one all-to-all with the split sizes read back from the
    lengths); each owner lays out its tables' global batch in rank order (rank 0's bags
    first); sharded_embbag looks them up and returns every rank its slice."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    T = len(owner)
    err = None
    try:
        _check_owner(owner, world)
        if len(batches) != T:
            raise ValueError(f"{len(batches)} batches for {T} tables")
        for t, (_, off) in enumerate(batches):
            if int(off.numel()) != local_batch + 1:
                raise ValueError(f"table {t}: offsets hold {int(off.numel())} entries, local_batch + 1 = "
                                 f"{local_batch + 1} expected")
        mine_n = sum(1 for r in owner if r == rank)
        if mine_n != len(local_tables):
            raise ValueError(f"rank {rank} owns {mine_n} tables by the plan but holds {len(local_tables)}")
    except ValueError as e:
        err = str(e)
    _agree(err, group, batches[0][1].device if batches else torch.device("cpu"))
    dev = batches[0][1].device
    to = [[t for t in range(T) if owner[t] == s] for s in range(world)]
    mine = to[rank]
    dest_order = [t for s in range(world) for t in to[s]]          # tables by destination rank
    # host read 1: first and last offset of every table (the ids each table sends)
    offs = torch.stack([off.to(torch.int64) for _, off in batches])  # [T, local_batch + 1]
    ends = offs[:, [0, -1]].cpu().tolist()
    # the lengths, destination-major over tables
    lens_all = (offs[:, 1:] - offs[:, :-1]).to(torch.int32)          # [T, local_batch]
    lens_send = lens_all[torch.tensor(dest_order, device=dev)].reshape(-1)
    ids_parts, n_ids_out = [], []
    for s in range(world):
        n = 0
        for t in to[s]:
            a, b = ends[t]
            ids_parts.append(batches[t][0][a:b].to(torch.int32))
            n += b - a
        n_ids_out.append(n)
    ids_send = torch.cat(ids_parts) if ids_parts else torch.empty(0, dtype=torch.int32, device=dev)
    lens_recv = torch.empty(world * local_batch * len(mine), dtype=torch.int32, device=dev)
    dist.all_to_all_single(lens_recv, lens_send, output_split_sizes=[local_batch * len(mine)] * world,
                           input_split_sizes=[local_batch * len(to[s]) for s in range(world)], group=group)
    lens = lens_recv.view(world, len(mine), local_batch)             # [source, table, bag]
    # host read 2: ids per (source, table), which fixes the split sizes of the ids exchange
    per_src_tab = lens.sum(dim=2).cpu().tolist()
    n_ids_in = [int(sum(row)) for row in per_src_tab]
    ids_recv = torch.empty(sum(n_ids_in), dtype=torch.int32, device=dev)
    dist.all_to_all_single(ids_recv, ids_send, output_split_sizes=n_ids_in, input_split_sizes=n_ids_out,
                           group=group)
    # the owner's batch, table-major over its tables, rank-major within a table
    src_base = [0]
    for s in range(world):
        src_base.append(src_base[-1] + n_ids_in[s])
    parts = []
    for k in range(len(mine)):
        for s in range(world):
            start = src_base[s] + sum(per_src_tab[s][:k])
            parts.append(ids_recv[start:start + per_src_tab[s][k]])
    indices = torch.cat(parts) if parts else torch.empty(0, dtype=torch.int32, device=dev)
    offsets = torch.zeros(len(mine) * world * local_batch + 1, dtype=torch.int32, device=dev)
    offsets[1:] = torch.cumsum(lens.permute(1, 0, 2).reshape(-1), dim=0).to(torch.int32)
    return sharded_embbag(local_tables, owner, d, indices, offsets, world * local_batch, group=group,
                          lookup=lookup, _checked=True)


class OwnerBuffers:
    """Every rank's receive buffer [batch // world, T * d] binary32, as device addresses
    usable by this rank's kernels: this rank's own tensor, and the others' buffers opened
    from the CUDA IPC handles of their storages (exchanged once, at creation)."""

    def __init__(self, own, addresses: List[int], keep: list):
        self.own = own                # this rank's buffer (the rows it owns)
        self.addresses = addresses    # device address of rank r's buffer, r = 0 .. world-1
        self._keep = keep             # the opened storages of the other ranks

    @classmethod
    def create(cls, local_batch: int, width: int, device, group=None) -> "OwnerBuffers":
        import torch
        import torch.distributed as dist
        own = torch.zeros((local_batch, width), dtype=torch.float32, device=device)
        world = dist.get_world_size(group) if dist.is_initialized() else 1
        if world == 1:
            return cls(own, [own.data_ptr()], [])
        rank = dist.get_rank(group)
        storage = own.untyped_storage()
        handles = [None] * world
        dist.all_gather_object(handles, (storage._share_cuda_(), own.storage_offset() * own.element_size()),
                               group=group)
        addresses, keep = [], []
        for r, (h, off) in enumerate(handles):
            if r == rank:
                addresses.append(own.data_ptr())
                continue
            peer = torch.UntypedStorage._new_shared_cuda(*h)
            keep.append(peer)
            addresses.append(peer.data_ptr() + off)
        return cls(own, addresses, keep)


def sharded_embbag_direct(local_tables: Sequence, owner: Sequence[int], d: int, indices, offsets, global_batch: int,
                          buffers: OwnerBuffers, group=None):
    """sharded_embbag with the exchange folded into the lookup: this rank's tables' rows
    for the global batch are stored straight into the owners' buffers (buffers.addresses,
    one per rank, each [global_batch // world, T * d]) at the column block of their global
    table. Returns this rank's buffer (the rows of its samples, all tables) once every
    rank's rows have arrived."""
    import torch
    import torch.distributed as dist
    import int4_row_wise_b200 as dq

    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    T = len(owner)
    mine = [t for t, r in enumerate(owner) if r == rank]
    err = None
    try:
        _check_owner(owner, world)
        if global_batch % world:
            raise ValueError(f"global batch {global_batch} is not divisible by the world size {world}")
        if len(buffers.addresses) != world:
            raise ValueError(f"{len(buffers.addresses)} owner buffers for {world} ranks")
        if tuple(buffers.own.shape) != (global_batch // world, T * d):
            raise ValueError(f"own buffer {tuple(buffers.own.shape)}, expected {(global_batch // world, T * d)}")
        if len(mine) != len(local_tables):
            raise ValueError(f"rank {rank} owns {len(mine)} tables by the plan but holds {len(local_tables)}")
        if mine and int(offsets.numel()) != len(mine) * global_batch + 1:
            raise ValueError(f"offsets hold {int(offsets.numel())} entries; {len(mine)} tables x {global_batch} "
                             f"bags need {len(mine) * global_batch + 1}")
    except ValueError as e:
        err = str(e)
    if world > 1:   # the owners have read the previous result (the agreement is the barrier)
        torch.cuda.current_stream(buffers.own.device).synchronize()
    _agree(err, group, buffers.own.device)
    stream = torch.cuda.current_stream(buffers.own.device)
    if mine:
        dq.dq_embbag_int4_fwd_to_owners(local_tables, d, indices, offsets, global_batch, mine, T,
                                        buffers.addresses, None, stream)
    if world > 1:   # every rank's rows have arrived
        stream.synchronize()
        dist.barrier(group)
    return buffers.own

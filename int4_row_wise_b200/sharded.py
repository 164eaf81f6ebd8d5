"""Table-wise sharded lookup: the hybrid parallelism of "Deep Learning Recommendation
Model for Personalization and Recommendation Systems" (section 提出的方法, proposed
method: embedding tables distributed across devices, model-parallel, while the rest
of the model runs data-parallel; the pooled embeddings reach every data-parallel
rank through an all-to-all exchange).

Each rank owns whole tables. For the global batch it looks up its own tables with
dq_embbag_int4_fwd (or an injected lookup), then one all-to-all sends every rank
the rows of its slice of the batch; each rank reassembles [batch / world, T * d] in
table order, exactly what a single device computes for those bags. The exchange is
torch.distributed's all_to_all_single (NCCL between GPUs).
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence

__all__ = ["plan_tables", "sharded_embbag", "sharded_embbag_local"]


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


def sharded_embbag(local_tables: Sequence, owner: Sequence[int], d: int, indices, offsets, global_batch: int,
                   group=None, lookup: Optional[Callable] = None):
    """Pooled outputs of this rank's slice of the global batch, over all tables.

    local_tables  the tables this rank owns, in ascending global table order
    owner         owner rank of every global table (plan_tables)
    indices, offsets   the lookup batch of this rank's tables for the whole global batch
                  (table-major over the owned tables, as dq_embbag_int4_fwd takes them);
                  tensors (a rank without tables passes empty ones on its device)
    global_batch  bags per table, divisible by the world size
    lookup        (tables, d, indices, offsets, batch) -> [batch, len(tables) * d];
                  dq.embbag by default
    Returns a [global_batch // world, T * d] tensor on the tables' device."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if global_batch % world:
        raise ValueError(f"global batch {global_batch} is not divisible by the world size {world}")
    mine = [t for t, r in enumerate(owner) if r == rank]
    if len(mine) != len(local_tables):
        raise ValueError(f"rank {rank} owns {len(mine)} tables by the plan but holds {len(local_tables)}")
    if lookup is None:
        import int4_row_wise_b200 as dq
        lookup = dq.embbag
    T = len(owner)
    bl = global_batch // world
    counts = [sum(1 for r in owner if r == s) for s in range(world)]
    if mine:
        local = lookup(local_tables, d, indices, offsets, global_batch)       # [B, T_own * d]
        dev, dt = local.device, local.dtype
        send = local.reshape(world, bl, len(mine) * d).contiguous().reshape(-1)  # destination-major
    else:  # a rank without tables still takes part in the exchange
        dev, dt = offsets.device, torch.float32
        send = torch.empty(0, dtype=dt, device=dev)
    recv = torch.empty(bl * sum(counts) * d, dtype=dt, device=dev)
    dist.all_to_all_single(recv, send, output_split_sizes=[bl * c * d for c in counts],
                           input_split_sizes=[bl * len(mine) * d] * world, group=group)
    out = torch.empty((bl, T, d), dtype=dt, device=dev)
    at = 0
    for s in range(world):
        if counts[s] == 0:
            continue
        chunk = recv[at:at + bl * counts[s] * d].view(bl, counts[s], d)
        at += bl * counts[s] * d
        out[:, [t for t, r in enumerate(owner) if r == s], :] = chunk
    return out.view(bl, T * d)


def sharded_embbag_local(local_tables: Sequence, owner: Sequence[int], d: int, batches: Sequence, local_batch: int,
                         group=None, lookup: Optional[Callable] = None):
    """The whole hybrid-parallel lookup from data-parallel inputs: every rank holds the
    bags of its own `local_batch` samples for every table (`batches[t] = (indices,
    offsets)`, CSR per table), and gets back [local_batch, T * d] for those samples.

    Steps: the bag lengths and the ids of every table travel to the table's owner (two
    all-to-alls: per-destination id counts, then lengths and ids); each owner lays out
    its tables' global batch in rank order (rank 0's bags first); sharded_embbag looks
    them up and returns every rank its slice."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    T = len(owner)
    if len(batches) != T:
        raise ValueError(f"{len(batches)} batches for {T} tables")
    dev = batches[0][1].device
    to = [[t for t in range(T) if owner[t] == s] for s in range(world)]
    mine = to[rank]
    # what this rank sends to s: the lengths of its bags for s's tables, then their ids
    lens_out, ids_out, n_ids_out = [], [], []
    for s in range(world):
        ls, ids = [], []
        for t in to[s]:
            idx, off = batches[t]
            ls.append((off[1:] - off[:-1]).to(torch.int32))
            ids.append(idx[off[0]:off[-1]].to(torch.int32))
        lens_out.append(torch.cat(ls) if ls else torch.empty(0, dtype=torch.int32, device=dev))
        cat = torch.cat(ids) if ids else torch.empty(0, dtype=torch.int32, device=dev)
        ids_out.append(cat)
        n_ids_out.append(cat.numel())
    # id counts per destination
    cnt_send = torch.tensor(n_ids_out, dtype=torch.int64, device=dev)
    cnt_recv = torch.empty(world, dtype=torch.int64, device=dev)
    dist.all_to_all_single(cnt_recv, cnt_send, group=group)
    n_ids_in = [int(v) for v in cnt_recv.tolist()]
    # lengths: local_batch per table, fixed sizes
    lens_recv = torch.empty(world * local_batch * len(mine), dtype=torch.int32, device=dev)
    dist.all_to_all_single(lens_recv, torch.cat(lens_out), output_split_sizes=[local_batch * len(mine)] * world,
                           input_split_sizes=[local_batch * len(to[s]) for s in range(world)], group=group)
    ids_recv = torch.empty(sum(n_ids_in), dtype=torch.int32, device=dev)
    dist.all_to_all_single(ids_recv, torch.cat(ids_out), output_split_sizes=n_ids_in,
                           input_split_sizes=n_ids_out, group=group)
    # the owner's batch, table-major over its tables, rank-major within a table
    lens = lens_recv.view(world, len(mine), local_batch)           # [source, table, bag]
    per_src_tab = lens.sum(dim=2).tolist()                         # ids per (source, table)
    src_base = [0]
    for s in range(world):
        src_base.append(src_base[-1] + n_ids_in[s])
    ids_parts = []
    for k in range(len(mine)):
        for s in range(world):
            start = src_base[s] + sum(per_src_tab[s][:k])
            ids_parts.append(ids_recv[start:start + per_src_tab[s][k]])
    indices = torch.cat(ids_parts) if ids_parts else torch.empty(0, dtype=torch.int32, device=dev)
    offsets = torch.zeros(len(mine) * world * local_batch + 1, dtype=torch.int32, device=dev)
    offsets[1:] = torch.cumsum(lens.permute(1, 0, 2).reshape(-1), dim=0).to(torch.int32)
    return sharded_embbag(local_tables, owner, d, indices, offsets, world * local_batch, group=group,
                          lookup=lookup)

"""Seeded synthetic inputs for the quantizer and the INT4 embedding bag.

This module only draws random numbers. It holds none of the quantizer's or the
lookup's arithmetic, so the CPU oracle and the CUDA path can both be fed from it.

The five workloads stand in for data that is not available here: the Criteo
Kaggle and Terabyte click logs used by the DQRM repository page and by "Deep
Learning Recommendation Model for Personalization and Recommendation Systems"
(section 主要发现 / main findings), and the Facebook production embedding tables of
"Post-Training 4-bit Quantization on Embedding Tables" (section 主要发现 / main
findings). Only their shapes are reproduced:

  tiny        1 table x 1000 rows, d=16, N(0, 0.1^2); 64 bags of 4 uniform ids
  kaggle      26 tables, rows log-uniform in [10, 1e7], d=16, U(-1/sqrt(n), 1/sqrt(n));
              one-hot bags, batch 2048, Zipf(1.05) ids
  terabyte    26 tables, rows min(log-uniform[1e3, 4e7], 4e6), d=64, N(0, 0.05^2);
              one-hot bags, batch 65536, Zipf(1.05) ids through a per-table permutation
  production  8 tables x 10M rows, d=128, per-row scale log-normal(-3, 1) times
              Student-t(3) entries; bags of U[20, 80] ids, batch 16384, Zipf(1.2) ids
  sweep-<d>   1 table x 1M rows, d in {16, 32, 64, 128, 256}, Student-t(3) entries
              times a per-row log-normal(0, 1) scale, 1% of rows with one entry x50;
              bags of 32 uniform ids, batch 8192

Every draw comes from numpy's PCG64 seeded by a SeedSequence keyed on
(seed, workload, table, purpose, block). Table values are drawn in blocks of
BLOCK_ROWS rows, each with its own key, so any block (and so any sampled row)
can be regenerated on its own, in any order and in any process.
"""
from __future__ import annotations

import dataclasses
import functools
import math
from typing import List, Optional, Tuple

import numpy as np

BLOCK_ROWS = 1 << 16

# purpose keys of the seed tree
_P_ROWS, _P_VALUES, _P_POOLING, _P_INDICES, _P_PERM, _P_PACKED = 1, 2, 3, 4, 5, 6

_WORKLOAD_KEYS = {
    "tiny": 10, "kaggle": 11, "terabyte": 12, "production": 13,
    "sweep-16": 20, "sweep-32": 21, "sweep-64": 22, "sweep-128": 23, "sweep-256": 24,
}

WORKLOADS = tuple(_WORKLOAD_KEYS)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    d: int
    rows: Tuple[int, ...]          # rows per table
    values: str                    # value distribution name
    batch: int                     # bags per table per lookup call
    pooling: Tuple[int, int]       # bag length drawn uniformly from [lo, hi] (lo == hi: fixed)
    zipf_alpha: Optional[float]    # None: uniform ids
    permute_ids: bool              # apply a per-table random permutation to Zipf ranks

    @property
    def n_tables(self) -> int:
        return len(self.rows)

    @property
    def total_rows(self) -> int:
        return int(sum(self.rows))


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(k) for k in key])))


def workload(name: str, seed: int = 0) -> Workload:
    """The named synthetic workload, with its table sizes drawn from `seed`."""
    if name not in _WORKLOAD_KEYS:
        raise ValueError(f"unknown workload {name!r}; known: {', '.join(WORKLOADS)}")
    wk = _WORKLOAD_KEYS[name]
    if name == "tiny":
        return Workload(name, seed, 16, (1000,), "normal0.1", 64, (4, 4), None, False)
    if name == "kaggle":
        r = _rng(seed, wk, 0, _P_ROWS, 0)
        rows = tuple(int(round(10.0 ** e)) for e in r.uniform(1.0, 7.0, 26))
        return Workload(name, seed, 16, rows, "uniform_inv_sqrt_n", 2048, (1, 1), 1.05, False)
    if name == "terabyte":
        r = _rng(seed, wk, 0, _P_ROWS, 0)
        hi = math.log10(4e7)
        rows = tuple(min(int(round(10.0 ** e)), 4_000_000) for e in r.uniform(3.0, hi, 26))
        return Workload(name, seed, 64, rows, "normal0.05", 65536, (1, 1), 1.05, True)
    if name == "production":
        return Workload(name, seed, 128, (10_000_000,) * 8, "lognormal_t3", 16384, (20, 80), 1.2, False)
    d = int(name.split("-")[1])
    return Workload(name, seed, d, (1_000_000,), "t3_outliers", 8192, (32, 32), None, False)


def first_tables(wl: Workload, n: int) -> Workload:
    """The workload restricted to its first n tables (same draws for those tables)."""
    return dataclasses.replace(wl, rows=wl.rows[:max(1, n)])


def table_block(wl: Workload, t: int, block: int) -> np.ndarray:
    """Rows [block*BLOCK_ROWS, min((block+1)*BLOCK_ROWS, n)) of table t, float32 [rows, d]."""
    n = wl.rows[t]
    r0 = block * BLOCK_ROWS
    if r0 >= n or block < 0:
        raise IndexError("block out of range")
    m = min(BLOCK_ROWS, n - r0)
    d = wl.d
    r = _rng(wl.seed, _WORKLOAD_KEYS[wl.name], t, _P_VALUES, block)
    if wl.values == "normal0.1":
        return (r.standard_normal((m, d), dtype=np.float32) * np.float32(0.1)).astype(np.float32)
    if wl.values == "normal0.05":
        return (r.standard_normal((m, d), dtype=np.float32) * np.float32(0.05)).astype(np.float32)
    if wl.values == "uniform_inv_sqrt_n":
        a = 1.0 / math.sqrt(n)
        return r.uniform(-a, a, (m, d)).astype(np.float32)
    if wl.values == "lognormal_t3":
        scale = r.lognormal(-3.0, 1.0, (m, 1))
        return (r.standard_t(3.0, (m, d)) * scale).astype(np.float32)
    if wl.values == "t3_outliers":
        scale = r.lognormal(0.0, 1.0, (m, 1))
        x = r.standard_t(3.0, (m, d)) * scale
        hit = np.nonzero(r.random(m) < 0.01)[0]
        col = r.integers(0, d, hit.size)
        x[hit, col] *= 50.0
        return x.astype(np.float32)
    raise ValueError(wl.values)


def device_table(wl: Workload, t: int, device, rows_per_draw: int = 1 << 19):
    """Table t drawn on a CUDA device with torch's generator: float32 [n, d].

    For benches whose tables are too large to draw on the host in reasonable time
    (the production-shaped workload holds 10.24G values). The distributions are those
    of table_block; the random stream is torch's Philox keyed on (seed, workload,
    table), so the values differ from the host draws of the same table. Student-t(3)
    is drawn as z0 / sqrt((z1^2 + z2^2 + z3^2) / 3) from four standard normals."""
    import torch
    n, d = wl.rows[t], wl.d
    key = np.random.SeedSequence([wl.seed, _WORKLOAD_KEYS[wl.name], t, _P_VALUES, 1 << 20]).generate_state(1)[0]
    g = torch.Generator(device=device)
    g.manual_seed(int(key))
    out = torch.empty((n, d), dtype=torch.float32, device=device)

    def t3(m):
        z = torch.randn((4, m, d), generator=g, device=device)
        return z[0] * torch.rsqrt(z[1:].square().sum(0) / 3.0)

    for r0 in range(0, n, rows_per_draw):
        m = min(rows_per_draw, n - r0)
        o = out[r0:r0 + m]
        if wl.values == "normal0.1":
            torch.randn((m, d), generator=g, device=device, out=o).mul_(0.1)
        elif wl.values == "normal0.05":
            torch.randn((m, d), generator=g, device=device, out=o).mul_(0.05)
        elif wl.values == "uniform_inv_sqrt_n":
            a = 1.0 / math.sqrt(n)
            torch.rand((m, d), generator=g, device=device, out=o).mul_(2 * a).sub_(a)
        elif wl.values == "lognormal_t3":
            scale = torch.randn((m, 1), generator=g, device=device).sub_(3.0).exp_()
            o.copy_(t3(m) * scale)
        elif wl.values == "t3_outliers":
            scale = torch.randn((m, 1), generator=g, device=device).exp_()
            x = t3(m) * scale
            hit = torch.nonzero(torch.rand(m, generator=g, device=device) < 0.01).flatten()
            col = torch.randint(0, d, (hit.numel(),), generator=g, device=device)
            x[hit, col] *= 50.0
            o.copy_(x)
        else:
            raise ValueError(wl.values)
    return out


def n_blocks(wl: Workload, t: int) -> int:
    return (wl.rows[t] + BLOCK_ROWS - 1) // BLOCK_ROWS


def table_rows(wl: Workload, t: int, start: int = 0, stop: Optional[int] = None,
               out: Optional[np.ndarray] = None) -> np.ndarray:
    """Rows [start, stop) of table t as float32 [stop-start, d] (all rows by default)."""
    n = wl.rows[t]
    stop = n if stop is None else min(stop, n)
    if out is None:
        out = np.empty((max(stop - start, 0), wl.d), dtype=np.float32)
    pos = 0
    for b in range(start // BLOCK_ROWS, (stop + BLOCK_ROWS - 1) // BLOCK_ROWS):
        blk = table_block(wl, t, b)
        b0 = b * BLOCK_ROWS
        lo, hi = max(start, b0), min(stop, b0 + blk.shape[0])
        out[pos:pos + hi - lo] = blk[lo - b0:hi - b0]
        pos += hi - lo
    return out


def sample_rows(wl: Workload, t: int, rows: np.ndarray) -> np.ndarray:
    """The listed rows of table t (any order), regenerating only the blocks they fall in."""
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((rows.size, wl.d), dtype=np.float32)
    blocks = rows // BLOCK_ROWS
    for b in np.unique(blocks):
        blk = table_block(wl, t, int(b))
        sel = np.nonzero(blocks == b)[0]
        out[sel] = blk[rows[sel] - int(b) * BLOCK_ROWS]
    return out


@functools.lru_cache(maxsize=64)
def _zipf_cdf(n: int, alpha: float) -> np.ndarray:
    w = np.arange(1, n + 1, dtype=np.float64) ** (-alpha)
    c = np.cumsum(w)
    c /= c[-1]
    c.flags.writeable = False
    return c


@functools.lru_cache(maxsize=64)
def _permutation(seed: int, wk: int, t: int, n: int) -> np.ndarray:
    p = _rng(seed, wk, t, _P_PERM, 0).permutation(n)
    p.flags.writeable = False
    return p


def lookup_batch(wl: Workload, batch_id: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """One embedding-bag call: (indices int32 [sum L], offsets int32 [T*B + 1]).

    Bags are table-major: bag (t, b) is indices[offsets[t*B + b] : offsets[t*B + b + 1]]
    and holds row ids of table t.
    """
    wk = _WORKLOAD_KEYS[wl.name]
    B = wl.batch
    lens, ids = [], []
    for t, n in enumerate(wl.rows):
        lo, hi = wl.pooling
        if lo == hi:
            ln = np.full(B, lo, dtype=np.int64)
        else:
            ln = _rng(wl.seed, wk, t, _P_POOLING, batch_id).integers(lo, hi + 1, B)
        m = int(ln.sum())
        r = _rng(wl.seed, wk, t, _P_INDICES, batch_id)
        if wl.zipf_alpha is None:
            v = r.integers(0, n, m)
        else:
            v = np.searchsorted(_zipf_cdf(n, wl.zipf_alpha), r.random(m), side="right")
            v = np.minimum(v, n - 1)
            if wl.permute_ids:
                v = _permutation(wl.seed, wk, t, n)[v]
        lens.append(ln)
        ids.append(v)
    lens = np.concatenate(lens)
    offsets = np.zeros(lens.size + 1, dtype=np.int64)
    np.cumsum(lens, out=offsets[1:])
    if offsets[-1] >= 2 ** 31:
        raise OverflowError("lookup batch exceeds int32 offsets")
    return np.concatenate(ids).astype(np.int32), offsets.astype(np.int32)


def random_packed_table(n_rows: int, d: int, seed: int, codes_ld: Optional[int] = None
                        ) -> Tuple[np.ndarray, np.ndarray]:
    """A packed table with random bytes as codes and random binary16 scale/bias.

    For lookup tests at sizes where quantizing real rows first is not the point:
    codes uint8 [n_rows, codes_ld], scale_bias uint16 [n_rows, 2] (bit patterns).
    Odd d gets its unused high nibble cleared.
    """
    cb = (d + 1) // 2
    codes_ld = cb if codes_ld is None else codes_ld
    r = _rng(seed, 99, n_rows, _P_PACKED, d)
    raw = r.bit_generator.random_raw((n_rows * cb + 7) // 8).view(np.uint8)[:n_rows * cb].reshape(n_rows, cb)
    if codes_ld == cb:
        codes = raw.copy()
    else:
        codes = np.zeros((n_rows, codes_ld), dtype=np.uint8)
        codes[:, :cb] = raw
    if d % 2:
        codes[:, cb - 1] &= 0x0F
    scale = r.uniform(1e-3, 2e-2, n_rows).astype(np.float16)
    bias = r.uniform(-0.2, 0.05, n_rows).astype(np.float16)
    sb = np.stack([scale.view(np.uint16), bias.view(np.uint16)], axis=1)
    return codes, np.ascontiguousarray(sb)


# ---------------------------------------------------------------------------
# parallel generation of large tables (identical values: same per-block keys)
# ---------------------------------------------------------------------------
def _fill_blocks(args):
    from multiprocessing import shared_memory
    name, shape, wl, t, blocks = args
    shm = shared_memory.SharedMemory(name=name)
    try:
        out = np.ndarray(shape, dtype=np.float32, buffer=shm.buf)
        for b in blocks:
            blk = table_block(wl, t, b)
            out[b * BLOCK_ROWS:b * BLOCK_ROWS + blk.shape[0]] = blk
    finally:
        del out
        shm.close()
    return len(blocks)


class SharedTable:
    """A table generated by a pool of processes into shared memory. `array` is
    valid until close()."""

    def __init__(self, wl: Workload, t: int, procs: Optional[int] = None):
        import multiprocessing as mp
        import os as _os
        from multiprocessing import shared_memory
        n, d = wl.rows[t], wl.d
        self.shm = shared_memory.SharedMemory(create=True, size=max(n * d * 4, 4))
        self.array = np.ndarray((n, d), dtype=np.float32, buffer=self.shm.buf)
        nb = n_blocks(wl, t)
        procs = procs or min(len(_os.sched_getaffinity(0)), 32)
        chunks = [list(range(i, nb, procs)) for i in range(procs) if i < nb]
        with mp.get_context("spawn").Pool(len(chunks)) as pool:
            pool.map(_fill_blocks, [(self.shm.name, (n, d), wl, t, c) for c in chunks])

    def close(self):
        self.array = None
        self.shm.close()
        self.shm.unlink()

"""Bench: quantized rows/s of the row-wise INT4 path on B200, with the lookup's GB/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload production] [--impl reference]

One step is one pass of the whole path over the workload: quantize every table
(greedy search, FP16 scale/bias, packed codes), one sum-pooled embedding-bag call
over the packed tables, and dequantization of every packed row. `value` is rows
quantized per second of step time, all ranks together. The default workload is
the production-shaped one (8 tables x 10M rows x d=128), the largest that fits one
GPU; `per_workload` repeats the measurement, with fewer steps, for the tiny,
Kaggle-, Terabyte-shaped and sweep workloads.

The lookup's own throughput (`embbag`) is measured apart from the step: K_b
distinct pre-generated lookup batches on the device, L2 flushed once, one CUDA
graph of the K_b back-to-back calls, bytes = the sum of every call's unique
algorithmic bytes (cross-call L2 reuse of hot Zipf rows is included).

Multi-GPU (torchrun, one process per GPU): every rank quantizes an independent
set of tables (the workload drawn with seed = rank), with no collective on the
data path; timing is the max over ranks (weak scaling).

--impl reference times the CPU oracle on the same workload, on rank 0 only: every
step quantizes and dequantizes a bounded sample of rows and makes one full lookup
call; `ms_per_step` is the time of those steps as timed, `value` the sampled rows
per second of them, and the whole-table step time is extrapolated in a field of
its own.

After the timed region the line also reports, on rank 0: the pages' quality measure
(`quality`, `l2_eval`), the codebook quantizer and the bag backward + SGD +
re-quantization on the step's own tables (`next_rows`; --no-next-rows skips them),
the end-to-end leg from pinned host memory (`e2e`), the CPU oracle (`cpu_baseline`)
and the other workloads (`per_workload`; --no-per-workload skips them).
Other modes, one JSON line each: --lookup-only (the lookup alone), --bwd (the bag
backward + SGD + re-quantization), --codebook (the codebook quantizer and its
lookup), --sharded (the table-wise sharded lookup with its all-to-all exchanges).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from int4_row_wise_b200 import workloads as W  # noqa: E402

METRIC = "quantized rows/s and INT4 embedding-bag GB/s (fraction of B200 HBM roofline)"
FLOPS_PER_ELEMENT_EVAL = 10      # sub, div, rint, 2 clamps, mul, add, sub, mul, add
EVALS_PER_ROW = 1 + 2 * 168      # initial clip + two candidates per move
FP32_LANES_PER_SM = 128
SM_MHZ_MAX = 1965.0
DEVICE_DRAWN = ("production",)   # workloads whose fp32 tables are drawn on the device
HOST_PARALLEL_BYTES = 256 << 20  # host-drawn workloads above this use a process pool
HBM_FALLBACK_GBS = 6650.0
OTHER_WORKLOADS = ("tiny", "kaggle", "terabyte", "sweep-16", "sweep-32", "sweep-64", "sweep-128", "sweep-256")
# dram bytes read + written per quantized row, by row width d, from ncu captures of the
# quantizer (`ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum -k regex:quantize_rows
# -s 3 -c 1` around `bench.py --workload W --steps 1 --warmup 3 --no-per-workload --no-e2e
# --no-cpu-baseline --no-next-rows`): d=16, a Kaggle-shaped table of 3,097,041 rows, 199.1 MB
# read + 25.6 MB written; d=128, the sweep d=128 table of 1,000,000 rows, 514.8 MB read +
# 61.6 MB written. A launch's traffic scales with its rows at a fixed d; it is reported only
# for a captured d and while the kernel source still has the recorded sha256 prefix.
NCU_QUANT_TRAFFIC = {"kernel_sha": "b1b4606e303e4827", "bytes_per_row": {16: 72.56, 128: 576.39}}


# ---------------------------------------------------------------------------
# descriptions, peaks, algorithmic bytes
# ---------------------------------------------------------------------------
def _workload_desc(wl: W.Workload) -> str:
    pool = wl.pooling[0] if wl.pooling[0] == wl.pooling[1] else f"U[{wl.pooling[0]},{wl.pooling[1]}]"
    ids = "uniform" if wl.zipf_alpha is None else f"Zipf({wl.zipf_alpha})" + (" permuted" if wl.permute_ids else "")
    return (f"{wl.name}: {wl.n_tables} fp32 tables, d={wl.d}, {wl.total_rows} rows ({wl.values}); "
            f"embedding bag batch {wl.batch} x {wl.n_tables} tables, pooling {pool}, {ids} ids")


def _config(wl: W.Workload, n_gpus: int) -> dict:
    mb = wl.total_rows * wl.d * 4 / 1e6
    return {"workload": _workload_desc(wl), "tables": wl.n_tables, "d": wl.d, "rows_per_rank": wl.total_rows,
            "batch": wl.batch, "pooling": list(wl.pooling), "seed": "rank", "parallelism": f"dp{n_gpus}",
            "inputs": ("fp32 tables drawn on the device (torch Philox, the workload's distributions)"
                       if wl.name in DEVICE_DRAWN else "fp32 tables drawn on the host (numpy PCG64), uploaded"),
            "l2": ("inputs larger than L2 (fp32 tables %.0f MB > 126 MB)" % mb) if mb > 126 else
                  "inputs smaller than L2 (%.1f MB): the step re-reads them from L2" % mb}


def _kernel_sha() -> str:
    p = os.path.join(ROOT, "int4_row_wise_b200", "csrc", "dq_quantize.cu")
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:16]


def hbm_peak():
    """(GB/s, source) of the HBM roofline: the measured copy bandwidth when present."""
    try:
        return float(json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["hbm_gbs"]), \
            "MEASURED_PEAKS.json hbm_gbs (of measured)"
    except Exception:
        return HBM_FALLBACK_GBS, "6.65 TB/s earlier measurement on this pool (of fallback: MEASURED_PEAKS.json absent)"


def fp32_peak(sms: int) -> float:
    """FP32 peak in TFLOP/s: 2 x 128 lanes x SMs x 1965 MHz (FMA = 2 flops)."""
    return 2 * FP32_LANES_PER_SM * sms * SM_MHZ_MAX * 1e6 / 1e12


def _unique_bag_bytes(wl: W.Workload, idx: np.ndarray, off: np.ndarray, row_bytes=None) -> int:
    """Algorithmic bytes of one lookup call: unique packed rows touched per table,
    the ids, the offsets and the output."""
    rb = row_bytes or (wl.d + 1) // 2 + 4
    B = wl.batch
    uniq = 0
    for t in range(wl.n_tables):
        uniq += np.unique(idx[off[t * B]:off[(t + 1) * B]]).size
    return uniq * rb + idx.nbytes + off.nbytes + B * wl.n_tables * wl.d * 4


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        try:
            import torch
            p = torch.cuda.get_device_properties(device_index)
            self.sel = "%08X:%02X:%02X.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
        except Exception:
            self.sel = None

    def __enter__(self):
        if self.sel is None:
            return self
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self) -> dict:
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [v.strip() for v in l.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx.append(float(f[1]))
            except ValueError:
                continue
            for name, v in zip(names, f[4:8]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# the CPU oracle as baseline (and as the reference arm)
# ---------------------------------------------------------------------------
class OracleBench:
    """Times the CPU oracle on bounded samples of a workload: one oracle step quantizes
    and dequantizes a sample of rows (drawn from a pool of at most one block of 65,536
    rows per table, in proportion to the table sizes) and makes one full lookup call
    over packed tables of the workload's sizes."""

    def __init__(self, wl: W.Workload, tables=None):
        import oracle
        self.oracle = oracle
        self.wl = wl
        self.cores = len(os.sched_getaffinity(0))
        self.pool = [W.table_block(wl, t, 0) if n else np.zeros((0, wl.d), np.float32) for t, n in enumerate(wl.rows)]
        big = int(np.argmax(wl.rows))
        cal = self.pool[big][:256]
        t0 = time.perf_counter()
        oracle.quantize_rows(cal, nthreads=1)
        self.per_row_core = (time.perf_counter() - t0) / cal.shape[0]
        self.bag = W.lookup_batch(wl)
        self.tabs = tables if tables is not None else [W.random_packed_table(n, wl.d, 77 + t)
                                                       for t, n in enumerate(wl.rows)]
        self.tables_kind = "the GPU's packed tables" if tables is not None else \
            "random packed tables of the workload's sizes"

    def step(self, target_s: float, seed: int = 0) -> dict:
        """One oracle step sized for about target_s seconds."""
        wl, oracle = self.wl, self.oracle
        rng = np.random.default_rng(1234 + seed)
        n_sample = int(max(self.cores * 16, min(wl.total_rows, target_s * self.cores / self.per_row_core * 0.8)))
        share = np.array(wl.rows, dtype=np.float64) / wl.total_rows
        per_table = np.maximum(np.round(share * n_sample).astype(np.int64), (np.array(wl.rows) > 0).astype(np.int64))
        xs = []
        for t, k in enumerate(per_table):
            if k and self.pool[t].shape[0]:
                m = self.pool[t].shape[0]
                xs.append(self.pool[t][rng.choice(m, int(k), replace=int(k) > m)])
        x = np.ascontiguousarray(np.concatenate(xs))
        t0 = time.perf_counter()
        codes, sb, _, _ = oracle.quantize_rows(x, nthreads=self.cores)
        tq = time.perf_counter() - t0
        t0 = time.perf_counter()
        oracle.dequantize_rows(codes, sb, wl.d)
        tdq = time.perf_counter() - t0
        t0 = time.perf_counter()
        oracle.embbag(self.tabs, wl.d, self.bag[0], self.bag[1], wl.batch, nthreads=self.cores)
        tbag = time.perf_counter() - t0
        n = x.shape[0]
        return {"rows": n, "step_s": tq + tdq + tbag, "quantize_s": tq, "dequantize_s": tdq, "lookup_s": tbag,
                "full_step_s": (tq + tdq) * wl.total_rows / n + tbag}

    def describe(self, r: dict) -> str:
        return (f"{r['rows']} rows sampled across the {self.wl.n_tables} tables in proportion to their sizes "
                f"(from the first {W.BLOCK_ROWS} rows of each table), quantized ({r['quantize_s']:.2f} s) and "
                f"dequantized ({r['dequantize_s']:.3f} s), plus one full lookup call over {self.tables_kind} "
                f"({r['lookup_s']:.3f} s)")

    def single_core(self, n: int = 10_000) -> dict:
        """The oracle quantizer alone on one thread, over the first n rows of the largest table."""
        x = self.pool[int(np.argmax(self.wl.rows))][:n]
        t0 = time.perf_counter()
        self.oracle.quantize_rows(x, nthreads=1)
        dt = time.perf_counter() - t0
        return {"value": x.shape[0] / dt, "unit": "rows/s", "cores": 1, "rows": int(x.shape[0]),
                "what": "the oracle's greedy quantizer on one thread, first rows of the largest table"}

    def baseline(self, target_s: float) -> dict:
        r = self.step(target_s)
        return {"value": r["rows"] / r["step_s"], "unit": "rows/s", "cores": self.cores, "kind": "oracle",
                "sample": self.describe(r), "timed_s": r["step_s"],
                "extrapolated_full_step_s": r["full_step_s"], "single_core": self.single_core()}


def run_reference(args, wl: W.Workload) -> None:
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    ob = OracleBench(wl)
    per_step = max(1.0, min(6.0, args.ref_budget_s / (args.warmup + args.steps)))
    res = []
    for i in range(args.warmup + args.steps):
        r = ob.step(per_step, seed=i)
        if i >= args.warmup:
            res.append(r)
    rows = sum(r["rows"] for r in res)
    secs = sum(r["step_s"] for r in res)
    value = rows / secs
    line = {"metric": METRIC, "value": value, "unit": "rows/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / len(res) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": _config(wl, 1),
            "rows_per_step": rows / len(res),
            "extrapolated_full_step_ms": float(np.mean([r["full_step_s"] for r in res])) * 1e3,
            "cpu_baseline": {"value": value, "unit": "rows/s", "cores": ob.cores, "kind": "oracle",
                             "sample": "per step: " + ob.describe(res[-1])},
            "e2e": {"value": value, "unit": "rows/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# inputs
# ---------------------------------------------------------------------------
def _fill_table_blocks(task):
    from multiprocessing import shared_memory
    name, shape, wl, t, blocks = task
    shm = shared_memory.SharedMemory(name=name)
    try:
        out = np.ndarray(shape, dtype=np.float32, buffer=shm.buf)
        for b in blocks:
            blk = W.table_block(wl, t, b)
            out[b * W.BLOCK_ROWS:b * W.BLOCK_ROWS + blk.shape[0]] = blk
        del out
    finally:
        shm.close()
    return len(blocks)


class HostTables:
    """All tables of a host-drawn workload: serially when small, else by one pool of
    processes into shared memory. `arrays` is valid until close()."""

    def __init__(self, wl: W.Workload):
        self.shms = []
        if wl.total_rows * wl.d * 4 <= HOST_PARALLEL_BYTES:
            self.arrays = [W.table_rows(wl, t) for t in range(wl.n_tables)]
            return
        import multiprocessing as mp
        from multiprocessing import shared_memory
        procs = min(len(os.sched_getaffinity(0)), 32)
        self.arrays, tasks = [], []
        for t, n in enumerate(wl.rows):
            shm = shared_memory.SharedMemory(create=True, size=max(n * wl.d * 4, 4))
            self.shms.append(shm)
            self.arrays.append(np.ndarray((n, wl.d), dtype=np.float32, buffer=shm.buf))
            nb = W.n_blocks(wl, t)
            step = max(1, nb // procs)
            tasks += [(shm.name, (n, wl.d), wl, t, list(range(b, min(b + step, nb)))) for b in range(0, nb, step)]
        with mp.get_context("spawn").Pool(procs) as pool:
            for _ in pool.imap_unordered(_fill_table_blocks, tasks):
                pass

    def close(self):
        self.arrays = None
        for shm in self.shms:
            shm.close()
            shm.unlink()
        self.shms = []


def device_tables(wl: W.Workload, dev):
    """The workload's fp32 tables on the device: drawn there for the production-shaped
    workload, drawn on the host and uploaded otherwise."""
    import torch
    if wl.name in DEVICE_DRAWN:
        return [W.device_table(wl, t, dev) for t in range(wl.n_tables)]
    ht = HostTables(wl)
    try:
        return [torch.from_numpy(a).to(dev) for a in ht.arrays]
    finally:
        ht.close()


def rank_workload(name: str, rank: int) -> W.Workload:
    """Rank r quantizes its own independent set of tables: the workload drawn with seed r."""
    return W.workload(name, seed=rank)


def max_over_ranks(value: float, device) -> float:
    """The max of a per-rank device time over all ranks (a no-op without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# the device step
# ---------------------------------------------------------------------------
class Step:
    """Device buffers of one workload and its step: quantize every table (spread over
    side streams, largest first, each to the least loaded stream, so the partly idle
    last wave of one table overlaps the next), one lookup call (rotating over
    n_batches lookup batches), dequantize every row."""

    def __init__(self, dq, wl: W.Workload, xs, dev, n_streams: int = 4, n_batches: int = 4):
        import torch
        self.dq, self.wl, self.xs, self.dev = dq, wl, xs, dev
        d = wl.d
        self.cld = dq._codes_ld(d)
        self.codes = [torch.empty((n, self.cld), dtype=torch.uint8, device=dev) for n in wl.rows]
        self.sbs = [torch.empty((n, 2), dtype=torch.int16, device=dev) for n in wl.rows]
        self.deq = [torch.empty((n, d), dtype=torch.float32, device=dev) for n in wl.rows]
        self.tables = [dq.PackedTable(c, s) for c, s in zip(self.codes, self.sbs)]
        self.batches_h = [W.lookup_batch(wl, batch_id=i) for i in range(n_batches)]
        self.batches = [(torch.from_numpy(i).to(dev), torch.from_numpy(o).to(dev)) for i, o in self.batches_h]
        self.out = torch.empty((wl.batch, wl.n_tables * d), dtype=torch.float32, device=dev)
        self.stream = torch.cuda.current_stream(dev)
        self.side = [torch.cuda.Stream(dev) for _ in range(max(1, n_streams))]
        load = [0] * len(self.side)
        self.owner = [0] * wl.n_tables
        for t in sorted(range(wl.n_tables), key=lambda t: -wl.rows[t]):
            k = min(range(len(self.side)), key=lambda i: load[i])
            self.owner[t] = k
            load[k] += wl.rows[t]
        self.fork = torch.cuda.Event()
        self.joins = [torch.cuda.Event() for _ in self.side]
        self.launches = sum(1 for n in wl.rows if n > 0) * 2 + 1

    def run(self, k: int, ev=None):
        dq, wl, d, s = self.dq, self.wl, self.wl.d, self.stream
        if ev:
            ev[0].record(s)
        self.fork.record(s)
        for sst in self.side:
            sst.wait_event(self.fork)
        for t in range(wl.n_tables):
            dq.dq_quantize_rows_int4(self.xs[t], wl.rows[t], d, d, self.codes[t], self.cld, self.sbs[t], None, None,
                                     dq.DQ_MODE_GREEDY, None, self.side[self.owner[t]])
        for sst, j in zip(self.side, self.joins):
            j.record(sst)
            s.wait_event(j)
        if ev:
            ev[1].record(s)
        bi, bo = self.batches[k % len(self.batches)]
        dq.dq_embbag_int4_fwd(self.tables, d, bi, bo, wl.batch, self.out, None, s)
        if ev:
            ev[2].record(s)
        for c, sb, o in zip(self.codes, self.sbs, self.deq):
            dq.dq_dequantize_rows(c, self.cld, sb, c.shape[0], d, o, d, s)
        if ev:
            ev[3].record(s)

    def timed(self, steps: int, warmup: int, barrier, sampler=None):
        """Runs warm-up steps, then `steps` timed ones; returns the event times (ms):
        total, quantize, lookup, dequantize, and the sampler's clock summary."""
        import torch
        for k in range(warmup):
            self.run(k)
        barrier()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if sampler is not None:
            sampler.__enter__()
        try:
            t0.record(self.stream)
            for k in range(steps):
                self.run(k, ev[k])
            t1.record(self.stream)
            barrier()
        finally:
            if sampler is not None:
                sampler.__exit__(None, None, None)
        return {"total": t0.elapsed_time(t1),
                "quantize": sum(e[0].elapsed_time(e[1]) for e in ev),
                "lookup": sum(e[1].elapsed_time(e[2]) for e in ev),
                "dequantize": sum(e[2].elapsed_time(e[3]) for e in ev),
                "clocks": sampler.summary() if sampler is not None else None}


def lookup_graph(dq, wl: W.Workload, tables, dev, reps: int = 5, kb: int = 0, row_bytes=None, fwd=None) -> dict:
    """The lookup's throughput: K_b distinct lookup batches pre-generated on the device
    (64 when a call moves under 32 MB, else 8, enough to exceed L2 either way), each
    call with its own output buffer; L2 flushed once (a write of 2 x L2), then one CUDA
    graph of the K_b back-to-back calls; bytes = the sum of every call's unique
    algorithmic bytes. Median of `reps` flushed replays."""
    import torch
    fwd = fwd or dq.dq_embbag_int4_fwd
    b0 = W.lookup_batch(wl, batch_id=1000)
    bytes0 = _unique_bag_bytes(wl, *b0, row_bytes=row_bytes)
    kb = kb or (64 if bytes0 < (32 << 20) else 8)
    bh = [b0] + [W.lookup_batch(wl, batch_id=1000 + i) for i in range(1, kb)]
    nbytes = [bytes0] + [_unique_bag_bytes(wl, i, o, row_bytes=row_bytes) for i, o in bh[1:]]
    bd = [(torch.from_numpy(i).to(dev), torch.from_numpy(o).to(dev)) for i, o in bh]
    outs = [torch.empty((wl.batch, wl.n_tables * wl.d), dtype=torch.float32, device=dev) for _ in range(kb)]
    l2 = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 0) or (126 << 20)
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        for (i, o), out in zip(bd, outs):     # eager warm-up (device attributes cached before capture)
            fwd(tables, wl.d, i, o, wl.batch, out, None, side)
    side.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for (i, o), out in zip(bd, outs):
            fwd(tables, wl.d, i, o, wl.batch, out, None, side)
    torch.cuda.synchronize(dev)
    s = torch.cuda.current_stream(dev)
    ms = []
    for _ in range(reps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        g.replay()
        e1.record(s)
        torch.cuda.synchronize(dev)
        ms.append(e0.elapsed_time(e1))
    del g
    t = statistics.median(ms)
    peak, src = hbm_peak()
    gbs = sum(nbytes) / (t / 1e3) / 1e9
    return {"value": gbs, "unit": "GB/s", "peak": peak, "frac": gbs / peak, "peak_source": src,
            "calls_per_graph": kb, "bytes_per_call": int(np.mean(nbytes)), "us_per_call": t * 1e3 / kb,
            "method": f"CUDA graph of {kb} back-to-back calls over distinct batches, L2 flushed once before it; "
                      "sum of per-call unique bytes (cross-call L2 reuse of hot Zipf rows included); "
                      f"median of {reps} replays"}


# ---------------------------------------------------------------------------
# the CUDA path: the default line
# ---------------------------------------------------------------------------
def run_gpu(args, wl: W.Workload) -> None:
    import torch
    import torch.distributed as dist

    import int4_row_wise_b200 as dq

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    dq.load()

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    wlr = rank_workload(wl.name, rank)
    xs = device_tables(wlr, dev)
    step = Step(dq, wlr, xs, dev, n_streams=args.streams)
    tm = step.timed(args.steps, args.warmup, barrier, ClockSampler(dev.index))
    total_ms = max_over_ranks(tm["total"], dev)
    value = wlr.total_rows * world * args.steps / (total_ms / 1e3)

    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    peak_tf = fp32_peak(sms)
    q_flops = float(FLOPS_PER_ELEMENT_EVAL * EVALS_PER_ROW * wlr.d) * wlr.total_rows * args.steps
    achieved = q_flops / (tm["quantize"] / 1e3) / 1e12
    traffic = None  # bytes per average quantize launch (one launch per table)
    per_row = NCU_QUANT_TRAFFIC["bytes_per_row"].get(wlr.d)
    if per_row is not None and NCU_QUANT_TRAFFIC["kernel_sha"] == _kernel_sha():
        traffic = per_row * wlr.total_rows / max(1, sum(1 for n in wlr.rows if n))

    line = None
    if rank == 0:
        stream = step.stream
        hbm, hbm_src = hbm_peak()
        bag_in_step = sum(_unique_bag_bytes(wlr, *step.batches_h[k % len(step.batches_h)])
                          for k in range(args.steps)) / (tm["lookup"] / 1e3) / 1e9
        embbag = lookup_graph(dq, wlr, step.tables, dev)
        embbag["in_step"] = {"value": bag_in_step, "unit": "GB/s", "frac": bag_in_step / hbm,
                             "us_per_call": tm["lookup"] / args.steps * 1e3,
                             "method": "one call per bench step, rotating 4 batches, event-timed in the step"}
        quality, l2_eval = _quality(dq, wlr, xs, step, dev, stream)
        line = {
            "metric": METRIC, "value": value, "unit": "rows/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": _config(wlr, world),
            "roofline": {"bound": "alu", "kernel": "quantize_rows_kernel", "achieved": achieved,
                         "peak": peak_tf, "unit": "TFLOP/s", "frac": achieved / peak_tf, "traffic": traffic,
                         "peak_source": f"2 x {FP32_LANES_PER_SM} FP32 lanes x {sms} SMs x 1965 MHz (FMA = 2 flops), "
                                        "derived from unit counts and the max clock",
                         "work": f"{FLOPS_PER_ELEMENT_EVAL} flops x {EVALS_PER_ROW} evaluations x d per row"},
            "embbag": embbag,
            "quality": quality, "l2_eval": l2_eval,
            "phases_ms_per_step": {k: tm[k] / args.steps for k in ("quantize", "lookup", "dequantize")},
            "gpu_launches": step.launches * args.steps,
            "clocks": tm["clocks"],
        }
    if world > 1:
        dist.barrier()
    # the dequantized rows are not needed after the timed region: room for the other legs
    step.deq = None
    torch.cuda.empty_cache()
    if rank == 0 and not args.no_next_rows:
        line["next_rows"] = _next_rows(wlr, xs, step, dev, dq)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        host_tabs = [(c.cpu().numpy()[:, :(wlr.d + 1) // 2], s.cpu().numpy().view(np.uint16))
                     for c, s in zip(step.codes, step.sbs)]
        line["cpu_baseline"] = OracleBench(wlr, host_tabs).baseline(args.ref_seconds)
        del host_tabs
    if not args.no_e2e:   # every rank: the same end-to-end step at N GPUs, max over ranks
        e2e = run_e2e(args, wlr, xs, step, dev, dq, world)
        if rank == 0:
            line["e2e"] = e2e
    del step, xs
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_per_workload:
        pw = {}
        for name in OTHER_WORKLOADS:
            if name != wlr.name:
                pw[name] = _workload_entry(args, W.workload(name), dev, dq)
        pw[wlr.name] = {"value": line["value"], "ms_per_step": line["ms_per_step"],
                        "fp32_frac": line["roofline"]["frac"], "embbag": _brief(line["embbag"]),
                        "cpu_baseline": line.get("cpu_baseline"), "rows": wlr.total_rows, "steps": args.steps,
                        "note": "the default line's own numbers"}
        line["per_workload"] = pw
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def _brief(e: dict) -> dict:
    return {k: e[k] for k in ("value", "unit", "frac", "us_per_call", "bytes_per_call", "calls_per_graph") if k in e}


def _quality(dq, wl, xs, step, dev, stream):
    """The pages' quality measure (normalized l2 error, greedy vs plain min/max) and
    the evaluator's own rate."""
    import torch
    d, cld = wl.d, step.cld
    err_g = torch.zeros(1, dtype=torch.float64, device=dev)
    err_m = torch.zeros(1, dtype=torch.float64, device=dev)
    l0, l1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for x, c, sb in zip(xs, step.codes, step.sbs):   # warm-up of the evaluator
        dq.dq_row_l2_error(x, x.shape[0], d, d, c, cld, sb, None, None, stream)
    l0.record(stream)
    for x, c, sb in zip(xs, step.codes, step.sbs):
        dq.dq_row_l2_error(x, x.shape[0], d, d, c, cld, sb, None, err_g, stream)
    l1.record(stream)
    mc = torch.empty((max(wl.rows), cld), dtype=torch.uint8, device=dev)
    ms = torch.empty((max(wl.rows), 2), dtype=torch.int16, device=dev)
    for x in xs:
        n = x.shape[0]
        dq.dq_quantize_rows_int4(x, n, d, d, mc, cld, ms, None, None, dq.DQ_MODE_MINMAX, None, stream)
        dq.dq_row_l2_error(x, n, d, d, mc, cld, ms, None, err_m, stream)
    torch.cuda.synchronize(dev)
    del mc, ms
    l2_bytes = wl.total_rows * (4 * d + (d + 1) // 2 + 4)
    l2_ms = l0.elapsed_time(l1)
    hbm, _ = hbm_peak()
    quality = {"normalized_l2_greedy": float(err_g.item()) / wl.total_rows,
               "normalized_l2_minmax": float(err_m.item()) / wl.total_rows,
               "definition": "mean over rows of ||x - xhat||_2 / ||x||_2 (binary64)",
               "context": "pages: greedy 0.03889-0.06221 across dims on Facebook production tables"}
    l2_eval = {"value": l2_bytes / (l2_ms / 1e3) / 1e9, "unit": "GB/s", "ms": l2_ms,
               "frac": l2_bytes / (l2_ms / 1e3) / 1e9 / hbm, "launches": len(xs)}
    return quality, l2_eval


def _workload_entry(args, wl: W.Workload, dev, dq) -> dict:
    """One other workload: a few steps on the device, its lookup by the graph method, and
    the oracle on a short bounded sample."""
    import torch
    xs = device_tables(wl, dev)
    step = Step(dq, wl, xs, dev, n_streams=args.streams)
    steps = 20 if wl.total_rows < 100_000 else 5
    tm = step.timed(steps, 3, lambda: torch.cuda.synchronize(dev))
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    flops = float(FLOPS_PER_ELEMENT_EVAL * EVALS_PER_ROW * wl.d) * wl.total_rows * steps
    entry = {"value": wl.total_rows * steps / (tm["total"] / 1e3), "unit": "rows/s",
             "ms_per_step": tm["total"] / steps, "steps": steps, "warmup": 3, "rows": wl.total_rows,
             "fp32_frac": flops / (tm["quantize"] / 1e3) / 1e12 / fp32_peak(sms),
             "embbag": _brief(lookup_graph(dq, wl, step.tables, dev)),
             "workload": _workload_desc(wl)}
    if not args.no_cpu_baseline:
        host_tabs = [(c.cpu().numpy()[:, :(wl.d + 1) // 2], s.cpu().numpy().view(np.uint16))
                     for c, s in zip(step.codes, step.sbs)]
        entry["cpu_baseline"] = OracleBench(wl, host_tabs).baseline(args.ref_seconds_other)
    del step, xs
    torch.cuda.empty_cache()
    return entry


def _kmeans_ops(d: int, iters: int, row_iters) -> tuple:
    """ALU ops the codebook quantizer executed over rows whose per-row Lloyd iteration
    counts (the kernel's row_iters output) are given: per element and centroid update 16
    distances (subtract, compare) and one add into its own cluster (33); the assignment
    that found the repeat (32) for rows that stopped early; the final 16 distances and the
    loss terms (35). Returns (ops, centroid updates run per row)."""
    ran = sum(int(r.sum()) for r in row_iters)
    stopped = sum(int((r < iters).sum()) for r in row_iters)
    rows = sum(int(r.numel()) for r in row_iters)
    return float(d) * (33 * ran + 32 * stopped + 35 * rows), ran / max(rows, 1)


def _next_rows(wl, xs, step, dev, dq) -> dict:
    """The codebook quantizer (all tables, 3 steps, then one codebook lookup per step) and
    the bag backward + SGD + re-quantization (10 calls over the step's lookup batches,
    each with its own seeded output gradient), timed with CUDA events after the bench's
    timed region. The codebook leg runs first, on the untouched tables; the backward then
    updates the tables in place."""
    import torch
    d = wl.d
    cld = step.cld
    stream = step.stream
    T, B = wl.n_tables, wl.batch
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    out = {}
    kc = [torch.empty((n, cld), dtype=torch.uint8, device=dev) for n in wl.rows]
    kcb = [torch.empty((n, 16), dtype=torch.int16, device=dev) for n in wl.rows]
    kt = [dq.KmeansTable(c, b) for c, b in zip(kc, kcb)]
    kit = [torch.empty(n, dtype=torch.int32, device=dev) for n in wl.rows]
    bag_out = torch.empty((B, T * d), dtype=torch.float32, device=dev)
    iters = dq.KMEANS_ITERS

    def cb_step(k):
        for t, x in enumerate(xs):
            if wl.rows[t]:
                dq.dq_quantize_rows_kmeans4(x, wl.rows[t], d, d, kc[t], cld, kcb[t], None, iters, None, stream,
                                            row_iters=kit[t])
        i, o = step.batches[k % len(step.batches)]
        dq.dq_embbag_kmeans4_fwd(kt, d, i, o, B, bag_out, None, stream)

    cb_step(0)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for k in range(3):
        cb_step(k)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    cb_ms = e0.elapsed_time(e1) / 3
    t = int(np.argmax(wl.rows))
    n_q = min(wl.rows[t], 200000)
    x64 = xs[t][:n_q].double()
    xk = dq.dequantize_rows_kmeans(kc[t][:n_q], kcb[t][:n_q], d).double()
    xu = dq.dequantize_rows(step.codes[t][:n_q], step.sbs[t][:n_q], d).double()
    nrm = x64.norm(dim=1)
    ok = nrm > 0
    cb_flops, cb_iters_run = _kmeans_ops(d, iters, [r for r, n in zip(kit, wl.rows) if n])
    cb_peak = FP32_LANES_PER_SM * sms * SM_MHZ_MAX * 1e6 / 1e12
    out["codebook"] = {
        "what": "codebook 4-bit quantization (per-row k-means, 16 binary16 centroids, "
                f"{iters} Lloyd iterations) of all tables + one codebook lookup call",
        "rows_per_s": wl.total_rows / (cb_ms / 1e3), "ms_per_step": cb_ms,
        "lloyd_updates_run_per_row": cb_iters_run,
        "alu_frac_upper": cb_flops / (cb_ms / 1e3) / 1e12 / cb_peak, "alu_peak_tops": cb_peak,
        "normalized_l2_codebook": float(((x64 - xk).norm(dim=1)[ok] / nrm[ok]).mean()),
        "normalized_l2_greedy": float(((x64 - xu).norm(dim=1)[ok] / nrm[ok]).mean()),
        "bytes_per_row": {"codebook": (d + 1) // 2 + 32, "greedy": (d + 1) // 2 + 4}}
    del kc, kcb, kt, kit, xk, xu, x64
    torch.cuda.empty_cache()
    gen = torch.Generator(device=dev)
    gen.manual_seed(4321)
    grads = [torch.randn((B, T * d), generator=gen, device=dev) * 1e-2 for _ in step.batches]
    n_ids = [int(i.size) for i, _ in step.batches_h]
    touched = [_touched_rows(wl, i, o) for i, o in step.batches_h]
    ws = torch.empty(max(dq.dq_embbag_int4_bwd_workspace_bytes(d, max(n_ids)), 256), dtype=torch.uint8,
                     device=dev)
    mt = [dq.MasterTable(x_, c_, s_) for x_, c_, s_ in zip(xs, step.codes, step.sbs)]

    def bwd(k):
        i, o = step.batches[k % len(step.batches)]
        dq.dq_embbag_int4_bwd_sgd(mt, d, i, o, B, n_ids[k % len(step.batches)], grads[k % len(step.batches)], 0.05,
                                  dq.DQ_MODE_GREEDY, ws, ws.numel(), None, stream)

    bwd(0)
    e0.record(stream)
    K = 10
    for k in range(K):
        bwd(k)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    b_ms = e0.elapsed_time(e1)
    ids = sum(n_ids[k % len(step.batches)] for k in range(K))
    rows = sum(touched[k % len(step.batches)] for k in range(K))
    out["bwd"] = {
        "what": "bag backward + SGD on the binary32 tables + greedy re-quantization of the touched rows, "
                "one call per lookup batch",
        "ids_per_s": ids / (b_ms / 1e3), "touched_rows_per_s": rows / (b_ms / 1e3), "ms_per_call": b_ms / K,
        "requant_alu_frac_over_call": rows * EVALS_PER_ROW * FLOPS_PER_ELEMENT_EVAL * d / (b_ms / 1e3) / 1e12
        / fp32_peak(sms)}
    del ws, grads
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------------------
# end to end through the public API, pinned host memory <-> device
# ---------------------------------------------------------------------------
def run_e2e(args, wl, xs, step, dev, dq, world) -> dict:
    """The same step through the Python binding, from and to pinned host memory. The
    host tables are a pinned copy of the step's inputs; every step uploads each table
    (one cudaMemcpyAsync per table), quantizes and dequantizes it, and downloads its
    codes, scale/bias and dequantized rows (those through a ring of pinned chunks, one
    cudaMemcpyAsync per chunk), then makes the lookup call and downloads its output.
    Uploads, kernels and downloads run on three streams over pieces of at most 1M rows, so
    piece p's upload overlaps piece p-1's kernels and piece p-2's downloads."""
    import psutil
    import torch
    d, T = wl.d, wl.n_tables
    cld = step.cld
    in_bytes = sum(x.numel() * 4 for x in xs)
    code_bytes = sum(c.numel() + s.numel() * 2 for c, s in zip(step.codes, step.sbs))
    ring_chunk = 64 << 20
    need = in_bytes + code_bytes + 4 * ring_chunk + (1 << 30)
    avail = psutil.virtual_memory().available
    fits = need * world <= 0.8 * avail
    if world > 1:   # one decision for all ranks, so that they take the same collectives
        import torch.distributed as dist
        f = torch.tensor([1 if fits else 0], dtype=torch.int32, device=dev)
        dist.all_reduce(f, op=dist.ReduceOp.MIN)
        fits = bool(f.item())
    if not fits:
        return {"skipped": f"pinned host copies of {need / 1e9:.1f} GB per rank x {world} ranks exceed 80 % of the "
                           f"free host memory ({avail / 1e9:.0f} GB on rank's node)"}
    stream = step.stream
    host_x = [torch.empty(x.shape, dtype=torch.float32, pin_memory=True) for x in xs]
    for h, x in zip(host_x, xs):
        h.copy_(x)
    pin_b = [(torch.from_numpy(i).pin_memory(), torch.from_numpy(o).pin_memory()) for i, o in step.batches_h]
    h_codes = [torch.empty(c.shape, dtype=torch.uint8, pin_memory=True) for c in step.codes]
    h_sb = [torch.empty(s.shape, dtype=torch.int16, pin_memory=True) for s in step.sbs]
    h_out = torch.empty((wl.batch, T * d), dtype=torch.float32, pin_memory=True)
    ring = [torch.empty(ring_chunk // 4, dtype=torch.float32, pin_memory=True) for _ in range(4)]
    deq = [torch.empty((n, d), dtype=torch.float32, device=dev) for n in wl.rows]
    out = torch.empty((wl.batch, T * d), dtype=torch.float32, device=dev)
    bi_d = torch.empty(max(i.numel() for i, _ in pin_b), dtype=torch.int32, device=dev)
    bo_d = torch.empty(pin_b[0][1].numel(), dtype=torch.int32, device=dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    # pieces of at most 1M rows: piece p's upload overlaps piece p-1's kernels and piece p-2's
    # downloads, so the pipeline fills and drains in one piece rather than one table
    piece_rows = 1 << 20
    pieces = [(t, r0, min(r0 + piece_rows, wl.rows[t])) for t in range(T) for r0 in range(0, wl.rows[t], piece_rows)]
    done = [torch.cuda.Event() for _ in pieces]
    for e in done:
        e.record(stream)
    tables = [dq.PackedTable(c, s_) for c, s_ in zip(step.codes, step.sbs)]
    per_chunk = ring_chunk // 4
    deq_bytes = sum(q.numel() * 4 for q in deq)
    h2d = in_bytes + pin_b[0][0].numel() * 4 + pin_b[0][1].numel() * 4
    d2h = code_bytes + deq_bytes + h_out.numel() * 4

    def one(k):
        bi, bo = pin_b[k % len(pin_b)]
        n_ids = bi.numel()
        prev = torch.cuda.Event()
        prev.record(stream)
        s_in.wait_event(prev)       # the previous step's lookup has read the batch buffers
        with torch.cuda.stream(s_in):
            bi_d[:n_ids].copy_(bi, non_blocking=True)
            bo_d.copy_(bo, non_blocking=True)
        slot = 0
        for pi, (t, r0, r1) in enumerate(pieces):
            n = r1 - r0
            s_in.wait_event(done[pi])   # the previous step's kernels of this piece have read its input
            with torch.cuda.stream(s_in):
                xs[t][r0:r1].copy_(host_x[t][r0:r1], non_blocking=True)
                up = torch.cuda.Event()
                up.record(s_in)
            stream.wait_event(up)
            codes_p, sbs_p, deq_p = step.codes[t][r0:r1], step.sbs[t][r0:r1], deq[t][r0:r1]
            dq.dq_quantize_rows_int4(xs[t][r0:r1], n, d, d, codes_p, cld, sbs_p, None, None,
                                     dq.DQ_MODE_GREEDY, None, stream)
            dq.dq_dequantize_rows(codes_p, cld, sbs_p, n, d, deq_p, d, stream)
            done[pi].record(stream)
            s_out.wait_event(done[pi])
            with torch.cuda.stream(s_out):
                h_codes[t][r0:r1].copy_(codes_p, non_blocking=True)
                h_sb[t][r0:r1].copy_(sbs_p, non_blocking=True)
                flat = deq_p.reshape(-1)
                for c0 in range(0, flat.numel(), per_chunk):
                    c1 = min(flat.numel(), c0 + per_chunk)
                    ring[slot % len(ring)][:c1 - c0].copy_(flat[c0:c1], non_blocking=True)
                    slot += 1
        in_done = torch.cuda.Event()
        in_done.record(s_in)
        stream.wait_event(in_done)
        dq.dq_embbag_int4_fwd(tables, d, bi_d[:n_ids], bo_d, wl.batch, out, None, stream)
        bag = torch.cuda.Event()
        bag.record(stream)
        s_out.wait_event(bag)
        with torch.cuda.stream(s_out):
            h_out.copy_(out, non_blocking=True)
        fin = torch.cuda.Event()
        fin.record(s_out)
        stream.wait_event(fin)

    steps = 3
    for k in range(2):
        one(k)
    torch.cuda.synchronize(dev)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for k in range(steps):
        one(k)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, dev) if world > 1 else e0.elapsed_time(e1) / steps
    del host_x, h_codes, h_sb, ring, deq
    torch.cuda.empty_cache()
    return {"value": wl.total_rows * world / (ms / 1e3), "unit": "rows/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": ms, "steps": steps,
            "api": "int4_row_wise_b200.dq_* from pinned host buffers, in pieces of at most 1M rows; one "
                   "cudaMemcpyAsync per piece upload and per 64 MB chunk of dequantized rows; upload / kernels / "
                   "download on 3 streams"}


# ---------------------------------------------------------------------------
# other modes
# ---------------------------------------------------------------------------
def run_lookup_only(args, wl: W.Workload) -> None:
    """The lookup alone over random packed tables of the workload's sizes (a few GB on the
    device at most, e.g. for profiling), by the graph method of lookup_graph, plus
    `single`: K single calls, each after an L2 flush, event-timed one by one."""
    import torch
    import int4_row_wise_b200 as dq
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    dq.load()
    if args.tables:
        wl = W.first_tables(wl, args.tables)
    d = wl.d
    cld = dq._codes_ld(d)
    tables = []
    for t, n in enumerate(wl.rows):
        c, sb = W.random_packed_table(n, d, 500 + t, cld)
        tables.append(dq.PackedTable(torch.from_numpy(c).to(dev), torch.from_numpy(sb.view(np.int16)).to(dev)))
    n_batches = 4
    bh = [W.lookup_batch(wl, batch_id=i) for i in range(n_batches)]
    bd = [(torch.from_numpy(i).to(dev), torch.from_numpy(o).to(dev)) for i, o in bh]
    nbytes = [_unique_bag_bytes(wl, i, o) for i, o in bh]
    out = torch.empty((wl.batch, wl.n_tables * d), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for k in range(args.warmup):
        dq.dq_embbag_int4_fwd(tables, d, bd[k % n_batches][0], bd[k % n_batches][1], wl.batch, out, None, stream)
    torch.cuda.synchronize(dev)
    for k in range(args.steps):
        flush.zero_()
        evs[k][0].record(stream)
        dq.dq_embbag_int4_fwd(tables, d, bd[k % n_batches][0], bd[k % n_batches][1], wl.batch, out, None, stream)
        evs[k][1].record(stream)
    torch.cuda.synchronize(dev)
    ms = [a.elapsed_time(b) for a, b in evs]
    single = sum(nbytes[k % n_batches] for k in range(args.steps)) / (sum(ms) / 1e3) / 1e9
    graph = lookup_graph(dq, wl, tables, dev) if not args.no_graph else None
    head = graph or {"value": single, "peak": hbm_peak()[0], "frac": single / hbm_peak()[0],
                     "bytes_per_call": int(np.mean(nbytes)), "peak_source": hbm_peak()[1],
                     "us_per_call": sum(ms) / len(ms) * 1e3, "calls_per_graph": 0}
    print(json.dumps({
        "metric": "INT4 embedding-bag GB/s (unique algorithmic bytes)", "value": head["value"], "unit": "GB/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["us_per_call"] / 1e3,
        "higher_is_better": True, "dtype": "f32", "data": "synthetic",
        "config": {"workload": _workload_desc(wl), "tables": "random packed codes of the workload's table sizes"},
        "roofline": {"bound": "hbm", "achieved": head["value"], "peak": head["peak"], "unit": "GB/s",
                     "frac": head["frac"], "bytes_per_call": head["bytes_per_call"],
                     "peak_source": head["peak_source"]},
        "graph": graph,
        "single": {"value": single, "unit": "GB/s", "us_per_call": sum(ms) / len(ms) * 1e3,
                   "method": "one call after each 256 MB L2 flush, CUDA events around the call (includes the "
                             "host's launch latency through the binding)"},
        "gpu_launches": head["calls_per_graph"] * 6 + args.steps + args.warmup}), flush=True)


def _touched_rows(wl: W.Workload, idx: np.ndarray, off: np.ndarray) -> int:
    """Distinct (table, row) pairs of one lookup batch: the rows its backward updates."""
    B = wl.batch
    return int(sum(np.unique(idx[off[t * B]:off[(t + 1) * B]]).size for t in range(wl.n_tables)))


def run_bwd(args, wl: W.Workload) -> None:
    """Times the training step after the lookup (dq_embbag_int4_bwd_sgd): the bag
    backward, the SGD step on binary32 masters of the workload's table sizes and the
    re-quantization of the touched rows, over 4 distinct lookup batches, each with its
    own output gradient. Masters and gradients are seeded normal draws on the device."""
    import torch
    import int4_row_wise_b200 as dq
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    dq.load()
    d = wl.d
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234)
    tables = []
    for n in wl.rows:
        m = torch.randn((n, d), generator=gen, device=dev)
        c, sb, _, _ = dq.quantize_rows(m, with_loss=False)
        tables.append(dq.MasterTable(m, c, sb))
    n_batches = 4
    bh = [W.lookup_batch(wl, batch_id=i) for i in range(n_batches)]
    bd = [(torch.from_numpy(i).to(dev), torch.from_numpy(o).to(dev)) for i, o in bh]
    grads = [torch.randn((wl.batch, wl.n_tables * d), generator=gen, device=dev) * 1e-2 for _ in range(n_batches)]
    touched = [_touched_rows(wl, i, o) for i, o in bh]
    n_ids = [int(i.size) for i, _ in bh]
    ws = torch.empty(max(dq.dq_embbag_int4_bwd_workspace_bytes(d, max(n_ids)), 256), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    lr = 0.05

    def call(k):
        i, o = bd[k % n_batches]
        dq.dq_embbag_int4_bwd_sgd(tables, d, i, o, wl.batch, n_ids[k % n_batches], grads[k % n_batches], lr,
                                  dq.DQ_MODE_GREEDY, ws, ws.numel(), None, stream)

    for k in range(args.warmup):
        call(k)
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(0) as clocks:
        for k in range(args.steps):
            flush.zero_()
            evs[k][0].record(stream)
            call(k)
            evs[k][1].record(stream)
        torch.cuda.synchronize(dev)
    clk = clocks.summary()
    ms = [a.elapsed_time(b) for a, b in evs]
    tot_ms = sum(ms)
    ids = sum(n_ids[k % n_batches] for k in range(args.steps))
    rows = sum(touched[k % n_batches] for k in range(args.steps))
    # the re-quantization's FP32 work (3370 d flops per touched row) against the FP32 peak,
    # over the whole call: a lower bound for requant_rows_kernel, which is most of it
    flops = rows * EVALS_PER_ROW * 10 * d
    peak = fp32_peak(torch.cuda.get_device_properties(dev).multi_processor_count)
    tflops = flops / (tot_ms / 1e3) / 1e12
    bits = max(1, int(sum(wl.rows)).bit_length())
    launches = 1 + 3 * ((bits + 7) // 8) + 3  # keys, sort passes, window, span, re-quantization
    print(json.dumps({
        "metric": "INT4 bag backward + SGD on binary32 masters + greedy re-quantization of touched rows: ids/s",
        "value": ids / (tot_ms / 1e3), "unit": "ids/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot_ms / len(ms), "higher_is_better": True, "dtype": "f32 (f64 gradient sums)",
        "data": "synthetic",
        "config": {"workload": _workload_desc(wl), "ids_per_call": int(np.mean(n_ids)),
                   "touched_rows_per_call": int(np.mean(touched)), "lr": lr,
                   "masters": "seeded normal draws of the workload's table sizes",
                   "l2": "256 MB flush written before every call"},
        "touched_rows_per_s": rows / (tot_ms / 1e3),
        "roofline": {"bound": "alu", "achieved": tflops, "peak": peak, "unit": "TFLOP/s", "frac": tflops / peak,
                     "over": "the whole call (re-quantization flops only)"},
        "clocks": clk, "gpu_launches": launches * args.steps}), flush=True)


def run_codebook(args, wl: W.Workload) -> None:
    """Times the codebook quantizer (per-row k-means, 16 binary16 centroids): one step =
    quantize every table of the workload + one codebook lookup call, inputs resident in
    HBM. Reports rows/s, the quantizer's ALU roofline, the lookup's unique bytes/s (graph
    method), and the normalized l2 error of the codebook and the greedy uniform quantizer
    on the first rows of the largest table."""
    import torch
    import int4_row_wise_b200 as dq
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    dq.load()
    xs = device_tables(wl, dev)
    d = wl.d
    cld = dq._codes_ld(d)
    iters = dq.KMEANS_ITERS
    codes = [torch.empty((n, cld), dtype=torch.uint8, device=dev) for n in wl.rows]
    cbs = [torch.empty((n, 16), dtype=torch.int16, device=dev) for n in wl.rows]
    tables = [dq.KmeansTable(c, b) for c, b in zip(codes, cbs)]
    its = [torch.empty(n, dtype=torch.int32, device=dev) for n in wl.rows]
    n_batches = 4
    bh = [W.lookup_batch(wl, batch_id=i) for i in range(n_batches)]
    bd = [(torch.from_numpy(i).to(dev), torch.from_numpy(o).to(dev)) for i, o in bh]
    rb = (d + 1) // 2 + 32
    out = torch.empty((wl.batch, wl.n_tables * d), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(k, ev=None):
        if ev:
            ev[0].record(stream)
        for t, x in enumerate(xs):
            if wl.rows[t]:
                dq.dq_quantize_rows_kmeans4(x, wl.rows[t], d, d, codes[t], cld, cbs[t], None, iters, None, stream,
                                            row_iters=its[t])
        if ev:
            ev[1].record(stream)
        i, o = bd[k % n_batches]
        dq.dq_embbag_kmeans4_fwd(tables, d, i, o, wl.batch, out, None, stream)
        if ev:
            ev[2].record(stream)

    for k in range(args.warmup):
        step(k)
    torch.cuda.synchronize(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    with ClockSampler(0) as clocks:
        for k in range(args.steps):
            step(k, evs[k])
        torch.cuda.synchronize(dev)
    clk = clocks.summary()
    q_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    tot_ms = sum(e[0].elapsed_time(e[2]) for e in evs)
    rows = wl.total_rows * args.steps
    # ALU work the kernel executed (every step quantizes the same tables: the same
    # iteration counts)
    ops_step, iters_run = _kmeans_ops(d, iters, [r for r, n in zip(its, wl.rows) if n])
    flops = ops_step * args.steps
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    peak = FP32_LANES_PER_SM * sms * SM_MHZ_MAX * 1e6 / 1e12  # one FP32 op per lane per clock (no FMA here)
    achieved = flops / (q_ms / 1e3) / 1e12
    bag = lookup_graph(dq, wl, tables, dev, row_bytes=rb, fwd=dq.dq_embbag_kmeans4_fwd)
    t = int(np.argmax(wl.rows))
    n_q = min(wl.rows[t], 200000)
    x = xs[t][:n_q]
    xk = dq.dequantize_rows_kmeans(codes[t][:n_q], cbs[t][:n_q], d)
    uc, usb, _, _ = dq.quantize_rows(x, with_loss=False)
    xu = dq.dequantize_rows(uc, usb, d)
    x64 = x.double()
    nrm = x64.norm(dim=1)
    ok = nrm > 0
    l2k = float(((x64 - xk.double()).norm(dim=1)[ok] / nrm[ok]).mean())
    l2u = float(((x64 - xu.double()).norm(dim=1)[ok] / nrm[ok]).mean())
    print(json.dumps({
        "metric": "codebook (k-means, 16 binary16 centroids) 4-bit quantization rows/s, step = quantize all tables "
                  "+ one codebook lookup call",
        "value": rows / (tot_ms / 1e3), "unit": "rows/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot_ms / args.steps, "higher_is_better": True, "dtype": "f32", "data": "synthetic",
        "config": {"workload": _workload_desc(wl), "lloyd_iterations": iters},
        "roofline": {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": f"{FP32_LANES_PER_SM} FP32 lanes x {sms} SMs x 1965 MHz, one op per lane-clock",
                     "ops_per_element": "33 per centroid update run + 32 for the repeat check of a row that "
                                        "stopped early + 35 (final assignment and loss)",
                     "lloyd_updates_run_per_row": iters_run},
        "embbag": _brief(bag),
        "quality": {"normalized_l2_codebook": l2k, "normalized_l2_greedy_uniform": l2u, "rows": n_q,
                    "bytes_per_row_codebook": rb, "bytes_per_row_uniform": (d + 1) // 2 + 4},
        "clocks": clk, "gpu_launches": (sum(1 for n in wl.rows if n) + 1) * args.steps}), flush=True)


def run_sharded(args, wl: W.Workload) -> None:
    """The table-wise sharded lookup (int4_row_wise_b200.sharded.sharded_embbag_local):
    tables planned over the ranks, every rank holding the bags of its own `batch`
    samples for every table; per call the bag lengths and ids travel to the owners,
    the owners look up the global batch and one all-to-all returns the pooled rows.
    Weak scaling: `batch` samples per rank. Tables are random packed codes of the
    workload's sizes. At one rank the exchanges are local copies through NCCL."""
    import datetime
    import torch
    import torch.distributed as dist
    import int4_row_wise_b200 as dq
    from int4_row_wise_b200.sharded import plan_tables, sharded_embbag_local

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world == 1:
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        if "MASTER_PORT" not in os.environ:
            import socket
            with socket.socket() as sk:
                sk.bind(("127.0.0.1", 0))
                os.environ["MASTER_PORT"] = str(sk.getsockname()[1])
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dist.init_process_group("nccl", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=300),
                            device_id=dev)
    dq.load()
    d = wl.d
    cld = dq._codes_ld(d)
    owner = plan_tables(wl.rows, world)
    mine = [t for t in range(wl.n_tables) if owner[t] == rank]
    tables = []
    for t in mine:
        c, sb = W.random_packed_table(wl.rows[t], d, 500 + t, cld)
        tables.append(dq.PackedTable(torch.from_numpy(c).to(dev), torch.from_numpy(sb.view(np.int16)).to(dev)))
    n_batches = 4
    B = wl.batch
    batches = []
    mywl = W.workload(wl.name, seed=rank)
    for k in range(n_batches):
        idx, off = W.lookup_batch(mywl, batch_id=k)  # this rank's samples, every table
        per_t = []
        for t in range(wl.n_tables):
            o = off[t * B:(t + 1) * B + 1].astype(np.int64)
            per_t.append((torch.from_numpy(idx[o[0]:o[-1]]).to(dev),
                          torch.from_numpy((o - o[0]).astype(np.int32)).to(dev)))
        batches.append((per_t, int(idx.size)))
    stream = torch.cuda.current_stream(dev)
    for k in range(args.warmup):
        sharded_embbag_local(tables, owner, d, batches[k % n_batches][0], B)
    torch.cuda.synchronize(dev)
    dist.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        e0.record(stream)
        for k in range(args.steps):
            sharded_embbag_local(tables, owner, d, batches[k % n_batches][0], B)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        dist.barrier()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dev)

    # the lookup and the exchange alone, from each owner's global batch of its tables:
    # through NCCL (sharded_embbag: lookup, all-to-all, reassembly) and folded into the
    # lookup (sharded_embbag_direct: one kernel stores every row in its owner's buffer)
    from int4_row_wise_b200.sharded import OwnerBuffers, sharded_embbag, sharded_embbag_direct
    gwl = W.dataclasses.replace(W.workload(wl.name, seed=100 + rank), batch=world * B)
    gidx, goff = W.lookup_batch(gwl, batch_id=0)
    GB = world * B
    parts, lens = [], []
    for t in mine:
        o = goff[t * GB:(t + 1) * GB + 1].astype(np.int64)
        parts.append(gidx[o[0]:o[-1]])
        lens.append(np.diff(o))
    g_idx = torch.from_numpy(np.concatenate(parts) if parts else np.zeros(1, np.int32)).to(dev)
    g_off = torch.from_numpy(np.concatenate([[0], np.cumsum(np.concatenate(lens))]).astype(np.int32)
                             if lens else np.zeros(1, np.int32)).to(dev)
    bufs = OwnerBuffers.create(B, wl.n_tables * d, dev)
    legs = {}
    for name, fn in (("nccl", lambda: sharded_embbag(tables, owner, d, g_idx, g_off, GB)),
                     ("direct", lambda: sharded_embbag_direct(tables, owner, d, g_idx, g_off, GB, bufs))):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(dev)
        dist.barrier()
        torch.cuda.synchronize(dev)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.steps):
            fn()
        f1.record(stream)
        torch.cuda.synchronize(dev)
        dist.barrier()
        legs[name] = max_over_ranks(f0.elapsed_time(f1) / args.steps, dev)
    del bufs
    ids_local = float(np.mean([n for _, n in batches]))
    bytes_ids = ids_local * 4 + wl.n_tables * B * 4          # ids + bag lengths each rank sends per call
    bytes_out = B * wl.n_tables * d * 4                        # pooled rows each rank receives per call
    cross = (world - 1) / world
    dist.barrier()
    if rank == 0:
        bags = world * B * wl.n_tables
        print(json.dumps({
            "metric": "table-wise sharded INT4 embedding-bag lookup (ids to the table owners, lookup, all-to-all of "
                      "pooled rows): bags/s", "value": bags / (ms / 1e3), "unit": "bags/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "dtype": "f32", "data": "synthetic",
            "config": {"workload": _workload_desc(wl), "local_batch": B, "global_batch": world * B,
                       "tables_per_rank": [sum(1 for o in owner if o == r) for r in range(world)],
                       "tables": "random packed codes of the workload's table sizes"},
            "exchange": {"bytes_per_rank_per_call": int(bytes_ids + bytes_out),
                         "cross_rank_bytes_per_rank_per_call": int((bytes_ids + bytes_out) * cross),
                         "parts": {"ids_and_lengths": int(bytes_ids), "pooled_rows": int(bytes_out)},
                         "note": "at one rank every exchange is a local copy"},
            "lookup_and_exchange": {
                "what": "from each owner's global batch of its tables: the lookup and the delivery of every "
                        "pooled row to its owner's [batch, T*d] rows",
                "nccl_ms": legs["nccl"], "direct_ms": legs["direct"],
                "nccl": "dq_embbag_int4_fwd, all_to_all_single, reassembly in table order",
                "direct": "dq_embbag_int4_fwd_to_owners storing into every owner's buffer (CUDA IPC across ranks), "
                          "a barrier before and after"},
            "clocks": clocks.summary()}), flush=True)
    dist.barrier()
    dist.destroy_process_group()


def main(argv=None) -> None:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=None, choices=W.WORKLOADS,
                    help="default: production (terabyte for --sharded)")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--ref-seconds", type=float, default=12.0, help="seconds of oracle work in the CPU baseline")
    ap.add_argument("--ref-seconds-other", type=float, default=3.0,
                    help="seconds of oracle work in each per_workload CPU baseline")
    ap.add_argument("--ref-budget-s", type=float, default=120.0,
                    help="--impl reference: seconds of oracle work over all warm-up and timed steps")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg (profiling runs)")
    ap.add_argument("--no-per-workload", action="store_true", help="skip the other workloads")
    ap.add_argument("--no-graph", action="store_true", help="--lookup-only: skip the CUDA-graph timing")
    ap.add_argument("--lookup-only", action="store_true",
                    help="time only the lookup, over random packed tables of the workload's sizes")
    ap.add_argument("--tables", type=int, default=0,
                    help="--lookup-only: only the workload's first N tables (a smaller case for profiling)")
    ap.add_argument("--streams", type=int, default=4, help="streams the per-table quantize launches spread over")
    ap.add_argument("--no-next-rows", action="store_true",
                    help="skip the codebook and backward legs that follow the timed region")
    ap.add_argument("--codebook", action="store_true",
                    help="time the codebook (k-means) quantizer and its lookup on the workload's tables")
    ap.add_argument("--bwd", action="store_true",
                    help="time the bag backward + SGD + re-quantization over masters of the workload's sizes")
    ap.add_argument("--sharded", action="store_true",
                    help="time the table-wise sharded lookup with its all-to-all exchanges")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    name = args.workload or ("terabyte" if args.sharded else "production")
    wl = W.workload(name, seed=0)
    if args.impl == "reference":
        run_reference(args, wl)
    elif args.lookup_only:
        run_lookup_only(args, wl)
    elif args.bwd:
        run_bwd(args, wl)
    elif args.codebook:
        run_codebook(args, wl)
    elif args.sharded:
        run_sharded(args, wl)
    else:
        run_gpu(args, wl)


if __name__ == "__main__":
    main()

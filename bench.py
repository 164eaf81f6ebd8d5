"""Bench: quantized rows/s of the row-wise INT4 path on B200, with the lookup's GB/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload kaggle] [--impl reference]

One step is one pass of the whole path over the workload: quantize every table
(greedy search, FP16 scale/bias, packed codes), one sum-pooled embedding-bag call
over the packed tables, and dequantization of every packed row. `value` is rows
quantized per second of step time, all ranks together; the lookup's throughput
is reported beside it in `embbag`.

Multi-GPU (torchrun, one process per GPU): every rank quantizes an independent
set of tables (the workload drawn with seed = rank), with no collective on the
data path; timing is the max over ranks (weak scaling).

--impl reference times the CPU oracle on the same workload (a bounded sample of
rows per step, extrapolated to the whole step), on rank 0 only.

After the timed region the line also reports, on rank 0: the pages' quality measure
(`quality`, `l2_eval`), the codebook quantizer and the bag backward + SGD +
re-quantization on the step's own tables (`next_rows`; --no-next-rows skips them),
the end-to-end leg from pinned host memory (`e2e`) and the CPU oracle (`cpu_baseline`).
Other modes, one JSON line each: --lookup-only (the lookup alone), --bwd (the bag
backward + SGD + re-quantization), --codebook (the codebook quantizer and its lookup).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from int4_row_wise_b200 import workloads as W  # noqa: E402

LARGE_BYTES = 8 << 30  # fp32 tables above this are generated in parallel and skip the e2e leg
METRIC = "quantized rows/s and INT4 embedding-bag GB/s (fraction of B200 HBM roofline)"
FLOPS_PER_ELEMENT_EVAL = 10      # sub, div, rint, 2 clamps, mul, add, sub, mul, add
EVALS_PER_ROW = 1 + 2 * 168      # initial clip + two candidates per move
SM_COUNT_NOMINAL = 148
FP32_LANES_PER_SM = 128
# dram bytes read + written per quantized row, from the ncu capture of the quantizer on
# the largest Kaggle-shaped table (304.1 MB read + 47.4 MB written for 4,742,154 rows);
# reported only while the kernel source still has the sha256 prefix recorded with it.
NCU_QUANT_TRAFFIC = {"kernel_sha": "b26922f6dcea3bc2", "bytes_per_row": 74.12}


def _workload_desc(wl: W.Workload) -> str:
    pool = wl.pooling[0] if wl.pooling[0] == wl.pooling[1] else f"U[{wl.pooling[0]},{wl.pooling[1]}]"
    ids = "uniform" if wl.zipf_alpha is None else f"Zipf({wl.zipf_alpha})" + (" permuted" if wl.permute_ids else "")
    return (f"{wl.name}: {wl.n_tables} fp32 tables, d={wl.d}, {wl.total_rows} rows ({wl.values}); "
            f"embedding bag batch {wl.batch} x {wl.n_tables} tables, pooling {pool}, {ids} ids")


def _config(wl: W.Workload, n_gpus: int) -> dict:
    return {"workload": _workload_desc(wl), "tables": wl.n_tables, "d": wl.d, "rows_per_rank": wl.total_rows,
            "batch": wl.batch, "pooling": list(wl.pooling), "seed": "rank", "parallelism": f"dp{n_gpus}",
            "l2": "inputs larger than L2 (fp32 tables %.0f MB > 126 MB)" % (wl.total_rows * wl.d * 4 / 1e6)}


def _kernel_sha() -> str:
    p = os.path.join(ROOT, "int4_row_wise_b200", "csrc", "dq_quantize.cu")
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:16]


def _unique_bag_bytes(wl: W.Workload, idx: np.ndarray, off: np.ndarray) -> int:
    """Algorithmic bytes of one lookup call: unique packed rows touched per table,
    the ids, the offsets and the output."""
    rb = (wl.d + 1) // 2 + 4
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
        self.sel = None
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
        self.lines = []
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
        for l in getattr(self, "lines", []):
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
# the CPU oracle as baseline
# ---------------------------------------------------------------------------
class OracleBench:
    """Times the CPU oracle on bounded samples of a workload and extrapolates one
    step (quantize + dequantize every row, one lookup call)."""

    def __init__(self, wl: W.Workload):
        import oracle
        self.oracle = oracle
        self.wl = wl
        self.cores = len(os.sched_getaffinity(0))
        big = int(np.argmax(wl.rows))
        cal = W.table_rows(wl, big, 0, min(256, wl.rows[big]))
        t0 = time.perf_counter()
        oracle.quantize_rows(cal, nthreads=1)
        self.per_row_core = (time.perf_counter() - t0) / cal.shape[0]
        self.bag = W.lookup_batch(wl)
        self.tabs = [W.random_packed_table(n, wl.d, 77 + t) for t, n in enumerate(wl.rows)]

    def step(self, target_s: float, seed: int = 0):
        """Returns (rows/s, seconds per step, sample description)."""
        wl, oracle = self.wl, self.oracle
        rng = np.random.default_rng(1234 + seed)
        n_sample = int(max(self.cores * 16, min(wl.total_rows, target_s * self.cores / self.per_row_core * 0.8)))
        share = np.array(wl.rows, dtype=np.float64) / wl.total_rows
        per_table = np.minimum(np.maximum(1, np.round(share * n_sample).astype(np.int64)), np.array(wl.rows))
        xs = []
        for t, k in enumerate(per_table):
            # rows drawn from at most 4 random blocks of the table (cheap to regenerate)
            nb = W.n_blocks(wl, t)
            blocks = rng.choice(nb, min(nb, 4), replace=False)
            cand = np.concatenate([np.arange(b * W.BLOCK_ROWS, min((b + 1) * W.BLOCK_ROWS, wl.rows[t]))
                                   for b in blocks])
            xs.append(W.sample_rows(wl, t, np.sort(rng.choice(cand, min(int(k), cand.size), replace=False))))
        x = np.concatenate(xs)
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
        step_s = (tq + tdq) * wl.total_rows / n + tbag
        sample = (f"{n} rows sampled across all {wl.n_tables} tables in proportion to their sizes (from <= 4 blocks "
                  f"of {W.BLOCK_ROWS} rows per table) "
                  f"(quantize {tq:.2f} s + dequantize {tdq:.3f} s, scaled to {wl.total_rows} rows) "
                  f"+ one full lookup call ({tbag:.3f} s)")
        return wl.total_rows / step_s, step_s, sample


def run_reference(args, wl: W.Workload) -> None:
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    ob = OracleBench(wl)
    per_step = max(1.0, args.ref_seconds * 10 / (args.warmup + args.steps))
    steps, sample = [], ""
    for i in range(args.warmup + args.steps):
        rate, step_s, sample = ob.step(per_step, seed=i)
        if i >= args.warmup:
            steps.append(step_s)
    step_s = float(np.mean(steps))
    value = wl.total_rows / step_s
    line = {"metric": METRIC, "value": value, "unit": "rows/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": _config(wl, 1),
            "cpu_baseline": {"value": value, "unit": "rows/s", "cores": ob.cores, "kind": "oracle",
                             "sample": f"per step: {sample}"},
            "e2e": {"value": value, "unit": "rows/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# multi-rank host logic (weak scaling, no collective on the data path)
# ---------------------------------------------------------------------------
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
# the CUDA path
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
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    dq.load()

    # --- inputs, generated on the host (seeded per rank) and made resident in HBM
    wlr = rank_workload(wl.name, rank)
    big = wlr.total_rows * wlr.d * 4 > LARGE_BYTES
    host_tables, xs = [], []
    for t in range(wlr.n_tables):
        if big:  # generated block-parallel into shared memory, uploaded, released
            st = W.SharedTable(wlr, t)
            xs.append(torch.from_numpy(st.array).to(dev))
            st.close()
        else:
            host_tables.append(W.table_rows(wlr, t))
            xs.append(torch.from_numpy(host_tables[-1]).to(dev))
    d = wlr.d
    cld = dq._codes_ld(d)
    codes = [torch.empty((n, cld), dtype=torch.uint8, device=dev) for n in wlr.rows]
    sbs = [torch.empty((n, 2), dtype=torch.int16, device=dev) for n in wlr.rows]
    deq = [torch.empty((n, d), dtype=torch.float32, device=dev) for n in wlr.rows]
    n_batches = 4
    batches_h = [W.lookup_batch(wlr, batch_id=i) for i in range(n_batches)]
    batches = [(torch.from_numpy(i).to(dev), torch.from_numpy(o).to(dev)) for i, o in batches_h]
    bag_bytes = [_unique_bag_bytes(wlr, i, o) for i, o in batches_h]
    out = torch.empty((wlr.batch, wlr.n_tables * d), dtype=torch.float32, device=dev)
    tables = [dq.PackedTable(c, s) for c, s in zip(codes, sbs)]
    stream = torch.cuda.current_stream(dev)
    launches_per_step = sum(1 for n in wlr.rows if n > 0) * 2 + 1

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    # Tables are spread over side streams (largest first, each to the least loaded
    # stream) so the partly idle last wave of one table overlaps the next table.
    side = [torch.cuda.Stream(dev) for _ in range(max(1, args.streams))]
    load = [0] * len(side)
    owner = [0] * wlr.n_tables
    for t in sorted(range(wlr.n_tables), key=lambda t: -wlr.rows[t]):
        k = min(range(len(side)), key=lambda i: load[i])
        owner[t] = k
        load[k] += wlr.rows[t]
    fork = torch.cuda.Event()
    joins = [torch.cuda.Event() for _ in side]

    def step(k: int, timed: bool):
        e = ev[k] if timed else None
        if e:
            e[0].record(stream)
        fork.record(stream)
        for sst in side:
            sst.wait_event(fork)
        for t in range(wlr.n_tables):
            sst = side[owner[t]]
            dq.dq_quantize_rows_int4(xs[t], xs[t].shape[0], d, d, codes[t], cld, sbs[t], None, None,
                                     dq.DQ_MODE_GREEDY, None, sst)
        for sst, j in zip(side, joins):
            j.record(sst)
            stream.wait_event(j)
        if e:
            e[1].record(stream)
        bi, bo = batches[k % n_batches]
        dq.dq_embbag_int4_fwd(tables, d, bi, bo, wlr.batch, out, None, stream)
        if e:
            e[2].record(stream)
        for c, s, o in zip(codes, sbs, deq):
            dq.dq_dequantize_rows(c, cld, s, c.shape[0], d, o, d, stream)
        if e:
            e[3].record(stream)

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for k in range(args.warmup):
        step(k, False)
    barrier()
    sampler = ClockSampler(dev.index)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with sampler:
        t_start.record(stream)
        for k in range(args.steps):
            step(k, True)
        t_end.record(stream)
        barrier()
    total_ms = t_start.elapsed_time(t_end)
    q_ms = sum(e[0].elapsed_time(e[1]) for e in ev)
    bag_ms = sum(e[1].elapsed_time(e[2]) for e in ev)
    dq_ms = sum(e[2].elapsed_time(e[3]) for e in ev)
    clocks = sampler.summary()

    total_ms = max_over_ranks(total_ms, dev)

    rows_all = wlr.total_rows * world * args.steps
    value = rows_all / (total_ms / 1e3)

    # --- roofline of the dominant kernel (the quantizer: FP32-ALU bound)
    props = torch.cuda.get_device_properties(dev)
    sms = props.multi_processor_count
    peak_tflops = 2 * FP32_LANES_PER_SM * sms * 1965e6 / 1e12
    q_flops = float(FLOPS_PER_ELEMENT_EVAL * EVALS_PER_ROW * d) * wlr.total_rows * args.steps
    achieved = q_flops / (q_ms / 1e3) / 1e12
    traffic = None  # bytes per average quantize launch (the launches differ in size: one per table)
    if NCU_QUANT_TRAFFIC["kernel_sha"] == _kernel_sha() and NCU_QUANT_TRAFFIC["bytes_per_row"]:
        traffic = NCU_QUANT_TRAFFIC["bytes_per_row"] * wlr.total_rows / max(1, sum(1 for n in wlr.rows if n))

    # --- quality (normalized l2 error, greedy vs plain min/max) and the evaluator's rate
    quality, l2_eval = None, None
    if rank == 0:
        err_g = torch.zeros(1, dtype=torch.float64, device=dev)
        err_m = torch.zeros(1, dtype=torch.float64, device=dev)
        l0, l1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for x, c, sb in zip(xs, codes, sbs):   # warm-up of the evaluator
            dq.dq_row_l2_error(x, x.shape[0], d, d, c, cld, sb, None, None, stream)
        l0.record(stream)
        for x, c, sb in zip(xs, codes, sbs):
            dq.dq_row_l2_error(x, x.shape[0], d, d, c, cld, sb, None, err_g, stream)
        l1.record(stream)
        for x in xs:
            mc = torch.empty((x.shape[0], cld), dtype=torch.uint8, device=dev)
            ms = torch.empty((x.shape[0], 2), dtype=torch.int16, device=dev)
            dq.dq_quantize_rows_int4(x, x.shape[0], d, d, mc, cld, ms, None, None, dq.DQ_MODE_MINMAX, None, stream)
            dq.dq_row_l2_error(x, x.shape[0], d, d, mc, cld, ms, None, err_m, stream)
            del mc, ms
        torch.cuda.synchronize(dev)
        l2_bytes = wlr.total_rows * (4 * d + (d + 1) // 2 + 4)
        l2_ms = l0.elapsed_time(l1)
        quality = {"normalized_l2_greedy": float(err_g.item()) / wlr.total_rows,
                   "normalized_l2_minmax": float(err_m.item()) / wlr.total_rows,
                   "definition": "mean over rows of ||x - xhat||_2 / ||x||_2 (binary64)",
                   "context": "pages: greedy 0.03889-0.06221 across dims on Facebook production tables"}
        l2_eval = {"value": l2_bytes / (l2_ms / 1e3) / 1e9, "unit": "GB/s", "ms": l2_ms,
                   "frac": l2_bytes / (l2_ms / 1e3) / 1e9 / _measured_hbm(), "launches": len(xs)}

    # --- the lookup's own throughput (unique algorithmic bytes per call)
    bag_gbs = sum(bag_bytes[k % n_batches] for k in range(args.steps)) / (bag_ms / 1e3) / 1e9
    hbm = _measured_hbm()

    # --- the widened rows, after the timed region, on the same device tables
    next_rows = None
    if rank == 0 and not args.no_next_rows:
        next_rows = _next_rows(wlr, xs, codes, sbs, batches_h, batches, dev, stream, dq)

    # --- end to end through the public API with pinned host buffers
    e2e = None
    if rank == 0 and not args.no_e2e:
        e2e = (run_e2e(args, wlr, host_tables, batches_h, dev, stream, dq) if not big else
               {"skipped": f"fp32 tables of {wlr.total_rows * wlr.d * 4 / 1e9:.0f} GB exceed the pinned-host budget"})

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ob = OracleBench(wlr)
        rate, step_s, sample = ob.step(args.ref_seconds)
        cpu = {"value": rate, "unit": "rows/s", "cores": ob.cores, "kind": "oracle", "sample": sample}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "rows/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": _config(wlr, world),
            "roofline": {"bound": "alu", "kernel": "quantize_rows_kernel", "achieved": achieved,
                         "peak": peak_tflops, "unit": "TFLOP/s", "frac": achieved / peak_tflops,
                         "traffic": traffic,
                         "peak_source": f"2 x {FP32_LANES_PER_SM} FP32 lanes x {sms} SMs x 1965 MHz (FMA = 2 flops)",
                         "work": f"{FLOPS_PER_ELEMENT_EVAL} flops x {EVALS_PER_ROW} evaluations x d per row"},
            "embbag": {"value": bag_gbs, "unit": "GB/s", "peak": hbm, "frac": bag_gbs / hbm,
                       "bytes_per_call": int(np.mean(bag_bytes)), "us_per_call": bag_ms / args.steps * 1e3,
                       "peak_source": "MEASURED_PEAKS.json hbm_gbs (of measured)"},
            "quality": quality,
            "l2_eval": l2_eval,
            "next_rows": next_rows,
            "phases_ms_per_step": {"quantize": q_ms / args.steps, "embbag": bag_ms / args.steps,
                                   "dequantize": dq_ms / args.steps},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def _next_rows(wl, xs, codes, sbs, batches_h, batches, dev, stream, dq) -> dict:
    """The codebook quantizer (all tables, 3 steps, then one codebook lookup per step) and
    the bag backward + SGD + re-quantization (10 calls over the step's lookup batches,
    each with its own seeded output gradient), timed with CUDA events after the bench's
    timed region. The codebook leg runs first, on the untouched tables; the backward then
    updates the tables in place (nothing after it reads them)."""
    import torch
    d = wl.d
    cld = dq._codes_ld(d)
    T, B = wl.n_tables, wl.batch
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    out = {}
    # codebook quantizer + its lookup
    kc = [torch.empty((n, cld), dtype=torch.uint8, device=dev) for n in wl.rows]
    kcb = [torch.empty((n, 16), dtype=torch.int16, device=dev) for n in wl.rows]
    kt = [dq.KmeansTable(c, b) for c, b in zip(kc, kcb)]
    bag_out = torch.empty((B, T * d), dtype=torch.float32, device=dev)
    iters = dq.KMEANS_ITERS

    def cb_step(k):
        for t, x in enumerate(xs):
            if wl.rows[t]:
                dq.dq_quantize_rows_kmeans4(x, wl.rows[t], d, d, kc[t], cld, kcb[t], None, iters, None, stream)
        i, o = batches[k % len(batches)]
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
    x = xs[t][:n_q]
    xk = dq.dequantize_rows_kmeans(kc[t][:n_q], kcb[t][:n_q], d).double()
    xu = dq.dequantize_rows(codes[t][:n_q], sbs[t][:n_q], d).double()
    x64 = x.double()
    nrm = x64.norm(dim=1)
    ok = nrm > 0
    cb_flops = wl.total_rows * d * (iters * 33 + 35)
    cb_peak = FP32_LANES_PER_SM * sms * 1965e6 / 1e12
    out["codebook"] = {
        "what": "codebook 4-bit quantization (per-row k-means, 16 binary16 centroids, "
                f"{iters} Lloyd iterations) of all tables + one codebook lookup call",
        "rows_per_s": wl.total_rows / (cb_ms / 1e3), "ms_per_step": cb_ms,
        "alu_frac_upper": cb_flops / (cb_ms / 1e3) / 1e12 / cb_peak,
        "alu_peak_tops": cb_peak,
        "normalized_l2_codebook": float(((x64 - xk).norm(dim=1)[ok] / nrm[ok]).mean()),
        "normalized_l2_greedy": float(((x64 - xu).norm(dim=1)[ok] / nrm[ok]).mean()),
        "bytes_per_row": {"codebook": (d + 1) // 2 + 32, "greedy": (d + 1) // 2 + 4}}
    del kc, kcb, kt, xk, xu, x64
    # bag backward + SGD on the tables as binary32 masters + re-quantization of touched rows
    gen = torch.Generator(device=dev)
    gen.manual_seed(4321)
    grads = [torch.randn((B, T * d), generator=gen, device=dev) * 1e-2 for _ in batches]
    n_ids = [int(i.size) for i, _ in batches_h]
    touched = [_touched_rows(wl, i, o) for i, o in batches_h]
    ws = torch.empty(max(dq.dq_embbag_int4_bwd_workspace_bytes(d, max(n_ids)), 256), dtype=torch.uint8,
                     device=dev)
    mt = [dq.MasterTable(x_, c_, s_) for x_, c_, s_ in zip(xs, codes, sbs)]

    def bwd(k):
        i, o = batches[k % len(batches)]
        dq.dq_embbag_int4_bwd_sgd(mt, d, i, o, B, n_ids[k % len(batches)], grads[k % len(batches)], 0.05,
                                  dq.DQ_MODE_GREEDY, ws, ws.numel(), None, stream)

    bwd(0)
    e0.record(stream)
    K = 10
    for k in range(K):
        bwd(k)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    b_ms = e0.elapsed_time(e1)
    ids = sum(n_ids[k % len(batches)] for k in range(K))
    rows = sum(touched[k % len(batches)] for k in range(K))
    out["bwd"] = {
        "what": "bag backward + SGD on the binary32 tables + greedy re-quantization of the touched rows, "
                "one call per lookup batch",
        "ids_per_s": ids / (b_ms / 1e3), "touched_rows_per_s": rows / (b_ms / 1e3), "ms_per_call": b_ms / K,
        "requant_alu_frac_over_call": rows * EVALS_PER_ROW * FLOPS_PER_ELEMENT_EVAL * d / (b_ms / 1e3) / 1e12
        / (2 * FP32_LANES_PER_SM * sms * 1965e6 / 1e12)}
    return out


def run_lookup_only(args, wl: W.Workload) -> None:
    """Times the lookup alone over random packed tables of the workload's sizes
    (a few GB on the device at most, e.g. for profiling): K calls over n distinct
    batches, each call's unique algorithmic bytes against the HBM peak."""
    import torch
    import int4_row_wise_b200 as dq
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    dq.load()
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
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # 256 MB > L2: cold start per call
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
    tot_bytes = sum(nbytes[k % n_batches] for k in range(args.steps))
    gbs = tot_bytes / (sum(ms) / 1e3) / 1e9
    hbm = _measured_hbm()
    print(json.dumps({
        "metric": "INT4 embedding-bag GB/s (unique algorithmic bytes, L2 flushed before each call)",
        "value": gbs, "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sum(ms) / len(ms), "higher_is_better": True, "dtype": "f32", "data": "synthetic",
        "config": {"workload": _workload_desc(wl), "tables": "random packed codes of the workload's table sizes",
                   "l2": "256 MB flush written before every call"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                     "bytes_per_call": int(np.mean(nbytes))},
        "gpu_launches": args.steps}), flush=True)


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
    cld = dq._codes_ld(d)
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
    peak = 2 * FP32_LANES_PER_SM * torch.cuda.get_device_properties(dev).multi_processor_count * 1965e6 / 1e12
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
    HBM. Reports rows/s, the quantizer's ALU roofline, the lookup's unique bytes/s, and
    the normalized l2 error of the codebook and the greedy uniform quantizer on the first
    rows of the largest table."""
    import torch
    import int4_row_wise_b200 as dq
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    dq.load()
    big = wl.total_rows * wl.d * 4 > LARGE_BYTES
    xs = []
    for t in range(wl.n_tables):
        if big:
            st = W.SharedTable(wl, t)
            xs.append(torch.from_numpy(st.array).to(dev))
            st.close()
        else:
            xs.append(torch.from_numpy(W.table_rows(wl, t)).to(dev))
    d = wl.d
    cld = dq._codes_ld(d)
    iters = dq.KMEANS_ITERS
    codes = [torch.empty((n, cld), dtype=torch.uint8, device=dev) for n in wl.rows]
    cbs = [torch.empty((n, 16), dtype=torch.int16, device=dev) for n in wl.rows]
    tables = [dq.KmeansTable(c, b) for c, b in zip(codes, cbs)]
    n_batches = 4
    bh = [W.lookup_batch(wl, batch_id=i) for i in range(n_batches)]
    bd = [(torch.from_numpy(i).to(dev), torch.from_numpy(o).to(dev)) for i, o in bh]
    rb = (d + 1) // 2 + 32
    nbytes = []
    for i, o in bh:
        uniq = sum(np.unique(i[o[t * wl.batch]:o[(t + 1) * wl.batch]]).size for t in range(wl.n_tables))
        nbytes.append(uniq * rb + i.nbytes + o.nbytes + wl.batch * wl.n_tables * d * 4)
    out = torch.empty((wl.batch, wl.n_tables * d), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(k, ev=None):
        if ev:
            ev[0].record(stream)
        for t, x in enumerate(xs):
            if wl.rows[t]:
                dq.dq_quantize_rows_kmeans4(x, wl.rows[t], d, d, codes[t], cld, cbs[t], None, iters, None, stream)
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
    b_ms = sum(e[1].elapsed_time(e[2]) for e in evs)
    tot_ms = sum(e[0].elapsed_time(e[2]) for e in evs)
    rows = wl.total_rows * args.steps
    # algorithmic work per element: per iteration 16 distances (subtract, compare) and one
    # add into the element's own cluster; then the final 16 distances and the loss terms
    flops = wl.total_rows * d * (iters * 33 + 35) * args.steps
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    peak = FP32_LANES_PER_SM * sms * 1965e6 / 1e12  # one FP32 op per lane per clock (no FMA here)
    achieved = flops / (q_ms / 1e3) / 1e12
    bag_gbs = sum(nbytes[k % n_batches] for k in range(args.steps)) / (b_ms / 1e3) / 1e9
    # quality on the first rows of the largest table
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
        "config": {"workload": _workload_desc(wl), "lloyd_iterations": iters,
                   "l2": "inputs larger than L2 (fp32 tables %.0f MB > 126 MB)" % (wl.total_rows * d * 4 / 1e6)},
        "roofline": {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": f"{FP32_LANES_PER_SM} FP32 lanes x {sms} SMs x 1965 MHz, one op per lane-clock",
                     "flops_per_element": iters * 33 + 35},
        "embbag": {"achieved": bag_gbs, "unit": "GB/s", "peak": _measured_hbm(), "frac": bag_gbs / _measured_hbm(),
                   "ms_per_call": b_ms / args.steps},
        "quality": {"normalized_l2_codebook": l2k, "normalized_l2_greedy_uniform": l2u, "rows": n_q,
                    "bytes_per_row_codebook": rb, "bytes_per_row_uniform": (d + 1) // 2 + 4},
        "clocks": clk, "gpu_launches": (sum(1 for n in wl.rows if n) + 1) * args.steps}), flush=True)


def _measured_hbm() -> float:
    try:
        return float(json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["hbm_gbs"])
    except Exception:
        return 6650.0  # fallback figure for this pool


def run_e2e(args, wl, host_tables, batches_h, dev, stream, dq) -> dict:
    """Same step through the public Python API, from and to pinned host memory:
    H2D of the tables and the lookup batch, quantize, look up, dequantize, and D2H
    of the packed tables, the pooled output and the dequantized rows. Table t's
    upload, compute and download run on three streams, so they overlap with
    table t-1's and t+1's."""
    import torch
    pin_x = [torch.from_numpy(h).pin_memory() for h in host_tables]
    pin_b = [(torch.from_numpy(i).pin_memory(), torch.from_numpy(o).pin_memory()) for i, o in batches_h]
    d = wl.d
    cld = dq._codes_ld(d)
    xs = [torch.empty_like(p, device=dev) for p in pin_x]
    codes = [torch.empty((n, cld), dtype=torch.uint8, device=dev) for n in wl.rows]
    sbs = [torch.empty((n, 2), dtype=torch.int16, device=dev) for n in wl.rows]
    deqs = [torch.empty((n, d), dtype=torch.float32, device=dev) for n in wl.rows]
    h_codes = [torch.empty((n, cld), dtype=torch.uint8).pin_memory() for n in wl.rows]
    h_sb = [torch.empty((n, 2), dtype=torch.int16).pin_memory() for n in wl.rows]
    h_deq = [torch.empty((n, d), dtype=torch.float32).pin_memory() for n in wl.rows]
    h_out = torch.empty((wl.batch, wl.n_tables * d), dtype=torch.float32).pin_memory()
    out = torch.empty((wl.batch, wl.n_tables * d), dtype=torch.float32, device=dev)
    bi_d = torch.empty_like(pin_b[0][0], device=dev)
    bo_d = torch.empty_like(pin_b[0][1], device=dev)
    h2d = sum(p.numel() * 4 for p in pin_x) + pin_b[0][0].numel() * 4 + pin_b[0][1].numel() * 4
    d2h = sum(c.numel() + s_.numel() * 2 + q.numel() * 4 for c, s_, q in zip(h_codes, h_sb, h_deq)) + h_out.numel() * 4
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    order = sorted(range(wl.n_tables), key=lambda t: wl.rows[t])  # small tables first: short pipeline fill

    def step(k):
        bi, bo = pin_b[k % len(pin_b)]
        prev = torch.cuda.Event()
        prev.record(stream)      # the previous step's kernels and downloads are ordered before this
        s_in.wait_event(prev)    # so uploads never overwrite buffers still being read
        with torch.cuda.stream(s_in):
            bi_d.copy_(bi, non_blocking=True)
            bo_d.copy_(bo, non_blocking=True)
        for t in order:
            with torch.cuda.stream(s_in):
                xs[t].copy_(pin_x[t], non_blocking=True)
                up = torch.cuda.Event()
                up.record(s_in)
            stream.wait_event(up)
            dq.dq_quantize_rows_int4(xs[t], xs[t].shape[0], d, d, codes[t], cld, sbs[t], None, None,
                                     dq.DQ_MODE_GREEDY, None, stream)
            dq.dq_dequantize_rows(codes[t], cld, sbs[t], codes[t].shape[0], d, deqs[t], d, stream)
            done = torch.cuda.Event()
            done.record(stream)
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                h_codes[t].copy_(codes[t], non_blocking=True)
                h_sb[t].copy_(sbs[t], non_blocking=True)
                h_deq[t].copy_(deqs[t], non_blocking=True)
        dq.dq_embbag_int4_fwd([dq.PackedTable(c, s_) for c, s_ in zip(codes, sbs)], d, bi_d, bo_d,
                              wl.batch, out, None, stream)
        done = torch.cuda.Event()
        done.record(stream)
        s_out.wait_event(done)
        with torch.cuda.stream(s_out):
            h_out.copy_(out, non_blocking=True)
        fin = torch.cuda.Event()
        fin.record(s_out)
        stream.wait_event(fin)

    steps = max(3, min(args.steps, 10))
    for k in range(2):
        step(k)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for k in range(steps):
        step(k)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    return {"value": wl.total_rows / (ms / 1e3), "unit": "rows/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": ms, "steps": steps,
            "api": "int4_row_wise_b200.dq_* from pinned host buffers, upload/compute/download on 3 streams"}


def main(argv=None) -> None:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="kaggle", choices=W.WORKLOADS)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--ref-seconds", type=float, default=12.0,
                    help="seconds of oracle work in the CPU baseline (the reference arm spends ~10x this in all)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg (profiling runs)")
    ap.add_argument("--lookup-only", action="store_true",
                    help="time only the lookup, over random packed tables of the workload's sizes")
    ap.add_argument("--streams", type=int, default=4, help="streams the per-table quantize launches spread over")
    ap.add_argument("--no-next-rows", action="store_true",
                    help="skip the codebook and backward legs that follow the timed region")
    ap.add_argument("--codebook", action="store_true",
                    help="time the codebook (k-means) quantizer and its lookup on the workload's tables")
    ap.add_argument("--bwd", action="store_true",
                    help="time the bag backward + SGD + re-quantization over masters of the workload's sizes")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = W.workload(args.workload, seed=0)
    if args.impl == "reference":
        run_reference(args, wl)
    elif args.lookup_only:
        run_lookup_only(args, wl)
    elif args.bwd:
        run_bwd(args, wl)
    elif args.codebook:
        run_codebook(args, wl)
    else:
        run_gpu(args, wl)


if __name__ == "__main__":
    main()

"""bench.py's host-side pieces on CPU: the pooled table generation matches the serial
one, the oracle baseline reports what it timed, the lookup's algorithmic bytes count
each table's distinct rows once, and the codebook quantizer's work counts the updates
it ran."""
import numpy as np

import bench
from int4_row_wise_b200 import workloads as W


def test_host_tables_pool_matches_serial(monkeypatch):
    wl = W.workload("kaggle")
    wl = W.dataclasses.replace(wl, rows=(70_000, 5, 0, 131_073))
    monkeypatch.setattr(bench, "HOST_PARALLEL_BYTES", 1)
    ht = bench.HostTables(wl)
    try:
        for t in range(wl.n_tables):
            assert np.array_equal(ht.arrays[t], W.table_rows(wl, t))
    finally:
        ht.close()


def test_unique_bag_bytes_counts_distinct_rows_per_table():
    wl = W.dataclasses.replace(W.workload("tiny"), rows=(10, 10), batch=2, pooling=(2, 2))
    idx = np.array([3, 3, 4, 3, 3, 3, 9, 9], np.int32)   # table 0: {3, 4}; table 1: {3, 9}
    off = np.array([0, 2, 4, 6, 8], np.int32)
    rb = (wl.d + 1) // 2 + 4
    assert bench._unique_bag_bytes(wl, idx, off) == 4 * rb + idx.nbytes + off.nbytes + 2 * 2 * wl.d * 4


def test_oracle_baseline_reports_the_timed_sample():
    ob = bench.OracleBench(W.workload("kaggle"))
    r = ob.baseline(0.5)
    assert r["kind"] == "oracle" and r["cores"] >= 1 and r["unit"] == "rows/s"
    rows = int(r["sample"].split()[0])
    assert abs(r["value"] - rows / r["timed_s"]) < 1e-9 * r["value"]
    assert r["extrapolated_full_step_s"] > r["timed_s"]
    sc = r["single_core"]
    assert sc["cores"] == 1 and 0 < sc["rows"] <= 10_000 and sc["value"] > 0


def test_kmeans_ops_count_the_updates_run():
    import torch
    # per element: 33 ops per update run, 32 more for a row that stopped before `iters`
    # (the assignment that found the repeat), 35 for the final assignment and loss
    its = [torch.tensor([10, 3, 0], dtype=torch.int32), torch.tensor([2], dtype=torch.int32)]
    ops, per_row = bench._kmeans_ops(64, 10, its)
    assert ops == 64 * (33 * (10 + 3 + 0 + 2) + 32 * 3 + 35 * 4)
    assert per_row == (10 + 3 + 0 + 2) / 4
    ops, per_row = bench._kmeans_ops(16, 10, [])
    assert ops == 0 and per_row == 0

"""The seeded input generators: deterministic, block-addressable, and shaped
like the workloads they stand in for."""
import numpy as np
import pytest

from int4_row_wise_b200 import workloads as W


def test_blocks_regenerate_identically():
    wl = W.workload("sweep-32")
    full = W.table_rows(wl, 0, 0, 3 * W.BLOCK_ROWS + 5)
    rows = np.array([5, W.BLOCK_ROWS - 1, W.BLOCK_ROWS, 3 * W.BLOCK_ROWS + 4, 17])
    assert np.array_equal(W.sample_rows(wl, 0, rows), full[rows])
    assert np.array_equal(W.table_rows(wl, 0, 70000, 70010), full[70000:70010])


@pytest.mark.parametrize("name", W.WORKLOADS)
def test_shapes(name):
    wl = W.workload(name)
    assert wl.d in (16, 32, 64, 128, 256)
    x = W.table_rows(wl, 0, 0, 100)
    assert x.dtype == np.float32 and x.shape == (min(100, wl.rows[0]), wl.d)
    assert np.all(np.isfinite(x))


def test_workload_table_sizes():
    k = W.workload("kaggle")
    assert k.n_tables == 26 and all(10 <= n <= 10 ** 7 for n in k.rows)
    t = W.workload("terabyte")
    assert t.n_tables == 26 and all(1000 <= n <= 4_000_000 for n in t.rows)
    p = W.workload("production")
    assert p.rows == (10_000_000,) * 8 and p.d == 128
    assert W.workload("kaggle") == W.workload("kaggle")


@pytest.mark.parametrize("name", ["tiny", "kaggle", "sweep-64"])
def test_lookup_batches(name):
    wl = W.workload(name)
    idx, off = W.lookup_batch(wl)
    T, B = wl.n_tables, wl.batch
    assert off.shape == (T * B + 1,) and off[0] == 0 and off[-1] == idx.size
    lens = np.diff(off)
    assert lens.min() >= wl.pooling[0] and lens.max() <= wl.pooling[1]
    for t in range(T):
        ids = idx[off[t * B]:off[(t + 1) * B]]
        assert ids.min() >= 0 and ids.max() < wl.rows[t]
    idx2, off2 = W.lookup_batch(wl)
    assert np.array_equal(idx, idx2) and np.array_equal(off, off2)


def test_production_pooling_and_zipf_head():
    wl = W.workload("production")
    import dataclasses
    small = dataclasses.replace(wl, rows=(100_000,), batch=4096)
    idx, off = W.lookup_batch(small)
    lens = np.diff(off)
    assert lens.min() >= 20 and lens.max() <= 80
    # Zipf(1.2): id 0 is the most frequent
    assert np.bincount(idx).argmax() == 0


def test_shared_table_matches_serial_generation():
    # the block-parallel generator (spawned processes) draws exactly the serial values
    wl = W.workload("sweep-16")
    st = W.SharedTable(wl, 0, procs=3)
    try:
        assert np.array_equal(st.array, W.table_rows(wl, 0))
    finally:
        st.close()


def test_random_packed_table_layout():
    codes, sb = W.random_packed_table(1000, 7, seed=1, codes_ld=16)
    assert codes.shape == (1000, 16) and sb.shape == (1000, 2)
    assert np.all(codes[:, 4:] == 0) and np.all(codes[:, 3] >> 4 == 0)
    s = sb[:, 0].view(np.float16).astype(np.float32)
    assert np.all(s > 0) and np.all(np.isfinite(sb.view(np.float16)))

"""GPU parity of the codebook quantizer (per-row k-means, 16 binary16 centroids), its
dequantization and its bag against the oracle: codes, codebooks and row losses
bit-identical on every row; dequantization bit-exact; bags within 1e-5 of the summed
magnitudes (bit-exact for one-hot bags).

"Post-Training 4-bit Quantization on Embedding Tables", section 提出的方法 (proposed
method), bullet 3 (codebook quantization by k-means clustering)."""
import numpy as np
import pytest
import torch

import int4_row_wise_b200 as dq
import oracle
from int4_row_wise_b200 import workloads as W
from tests.gpu_util import bag_tolerance_check, to_dev

pytestmark = pytest.mark.gpu


def _gpu_kmeans(x, iters, x_ld=None, codes_ld=None, flags=False):
    n, d = x.shape
    ld = d if x_ld is None else x_ld
    buf = np.zeros((max(n, 1), ld), np.float32)
    buf[:n, :d] = x
    xd = to_dev(buf)
    cld = (d + 1) // 2 if codes_ld is None else codes_ld
    codes = torch.full((max(n, 1), cld), 0xAB, dtype=torch.uint8, device="cuda")
    cb = torch.zeros((max(n, 1), 16), dtype=torch.int16, device="cuda")
    loss = torch.zeros(max(n, 1), dtype=torch.float32, device="cuda")
    fl = torch.zeros(1, dtype=torch.int32, device="cuda") if flags else None
    dq.dq_quantize_rows_kmeans4(xd, n, d, ld, codes, cld, cb, loss, iters, fl)
    torch.cuda.synchronize()
    c = codes.cpu().numpy()
    assert np.all(c[:n, (d + 1) // 2:] == 0xAB)
    return (c[:n, :(d + 1) // 2], cb.cpu().numpy().view(np.uint16)[:n], loss.cpu().numpy()[:n],
            int(fl.item()) if flags else None)


def _assert_same(x, iters, **kw):
    gc, gcb, gl, _ = _gpu_kmeans(x, iters, **kw)
    oc, ocb, ol = oracle.quantize_rows_kmeans(x, iters=iters)
    bad = np.nonzero(~(np.all(gc == oc, axis=1) & np.all(gcb == ocb, axis=1) &
                       (gl.view(np.uint32) == ol.view(np.uint32))))[0]
    assert bad.size == 0, f"{bad.size}/{len(x)} rows differ, first {bad[:5]}"


def _rows(n, d, seed, kind="normal"):
    r = np.random.default_rng(seed)
    if kind == "normal":
        return r.standard_normal((n, d)).astype(np.float32)
    if kind == "heavy":
        return (r.standard_t(3, (n, d)) * np.exp(r.normal(0, 1, (n, 1)))).astype(np.float32)
    if kind == "offset":
        return (1000 + r.standard_normal((n, d))).astype(np.float32)
    if kind == "few":
        return r.choice(np.float32([-1.5, 0.25, 3.0, 7.75]), (n, d)).astype(np.float32)
    raise ValueError(kind)


@pytest.mark.parametrize("d", [1, 2, 5, 16, 17, 32, 48, 64, 100, 128, 256, 512, 1024])
def test_kmeans_widths(cuda_device, d):
    n = 3001 if d <= 128 else 701
    _assert_same(_rows(n, d, d), 10)


@pytest.mark.parametrize("iters", [0, 1, 3, 30, 64])
@pytest.mark.parametrize("kind", ["normal", "heavy", "offset", "few"])
def test_kmeans_iterations_and_values(cuda_device, iters, kind):
    _assert_same(_rows(1500, 64, iters + 7, kind), iters)


@pytest.mark.parametrize("d,kind", [(16, "normal"), (64, "heavy"), (128, "offset"), (48, "few"), (1024, "normal")])
def test_kmeans_stops_at_a_fixed_point(cuda_device, d, kind):
    # the kernel stops a row once its assignment repeats; row_iters says after how many
    # centroid updates. The oracle run for exactly that many iterations must give the
    # outputs of all 64, and so must the GPU (with or without the counts requested).
    n, iters = (257 if d == 1024 else 1200), 64
    x = _rows(n, d, d + 11, kind)
    xd = to_dev(x)
    cld = (d + 1) // 2
    got = []
    for want_iters in (True, False):
        codes = torch.zeros((n, cld), dtype=torch.uint8, device="cuda")
        cb = torch.zeros((n, 16), dtype=torch.int16, device="cuda")
        loss = torch.zeros(n, dtype=torch.float32, device="cuda")
        its = torch.full((n,), -1, dtype=torch.int32, device="cuda") if want_iters else None
        dq.dq_quantize_rows_kmeans4(xd, n, d, d, codes, cld, cb, loss, iters, None, None, row_iters=its)
        got.append((codes.cpu().numpy(), cb.cpu().numpy().view(np.uint16), loss.cpu().numpy().view(np.uint32),
                    its.cpu().numpy() if want_iters else None))
    (gc, gcb, gl, it), (gc2, gcb2, gl2, _) = got
    assert np.array_equal(gc, gc2) and np.array_equal(gcb, gcb2) and np.array_equal(gl, gl2)
    oc, ocb, ol = oracle.quantize_rows_kmeans(x, iters=iters)
    assert np.array_equal(gc, oc) and np.array_equal(gcb, ocb) and np.array_equal(gl, ol.view(np.uint32))
    assert it.min() >= 0 and it.max() <= iters
    assert it.mean() < iters / 2, it.mean()   # Lloyd's iteration settles long before 64 updates
    for k in np.unique(it):
        rows = np.nonzero(it == k)[0]
        kc, kcb, kl = oracle.quantize_rows_kmeans(x[rows], iters=int(k))
        assert np.array_equal(kc, oc[rows]) and np.array_equal(kcb, ocb[rows]), k
        assert np.array_equal(kl.view(np.uint32), ol.view(np.uint32)[rows]), k


@pytest.mark.parametrize("d", [3, 16, 64, 128, 1024])
def test_kmeans_exact_and_sequential_updates(cuda_device, d):
    # a row whose nonzero values span more binades than binary64 sums hold exactly is
    # updated in index order by one lane; the others add each element into its own
    # cluster in any order. Rows of both kinds share warps and blocks here.
    r = np.random.default_rng(d + 40)
    n = 300 if d == 1024 else 3000
    x = r.standard_normal((n, d)).astype(np.float32)
    wide = r.random(n) < 0.1
    for i in np.nonzero(wide)[0]:
        k = r.integers(0, d, 3 if d > 3 else 1)
        x[i, k] = np.float32(r.choice([1e-12, -3e-15, 2e-39, 1e-30]))
    # cancellation inside a cluster: values around 0 at scales 2^-40 apart
    for i in np.nonzero(r.random(n) < 0.05)[0]:
        k = r.integers(0, d, 4 if d >= 4 else d)
        x[i, k] = np.float32([1e-3, 1e-3 * 2.0 ** -40, -1e-3, 1e-3 * 2.0 ** -41])[:k.size]
    _assert_same(x, 10)
    _assert_same(x, 64)


def test_kmeans_special_rows_and_strides(cuda_device):
    x = _rows(600, 16, 3)
    x[0] = 0.0
    x[1] = 2.5
    x[2, :8] = 1e-30
    x[3] = np.linspace(-8, 8, 16)
    _assert_same(x, 10)
    _assert_same(_rows(300, 40, 4), 10, x_ld=43, codes_ld=23)


def test_kmeans_workload_rows(cuda_device):
    for name in ("kaggle", "terabyte", "production", "sweep-128"):
        wl = W.workload(name)
        t = int(np.argmax(wl.rows))
        x = W.sample_rows(wl, t, np.arange(2000))
        _assert_same(x, 10)


def test_kmeans_beats_uniform_on_normalized_l2(cuda_device):
    # the pages' finding: the codebook gives a lower normalized l2 loss than the uniform
    # quantizer; checked on the stored reconstructions of sampled workload rows
    for name in ("terabyte", "sweep-64"):
        wl = W.workload(name)
        x = W.sample_rows(wl, int(np.argmax(wl.rows)), np.arange(4000))
        xd = to_dev(x)
        codes, cb, _ = dq.quantize_rows_kmeans(xd)
        xk = dq.dequantize_rows_kmeans(codes, cb, x.shape[1]).cpu().numpy().astype(np.float64)
        uc, usb, _, _ = dq.quantize_rows(xd)
        xu = dq.dequantize_rows(uc, usb, x.shape[1]).cpu().numpy().astype(np.float64)
        x64 = x.astype(np.float64)
        nrm = np.linalg.norm(x64, axis=1)
        ek = np.mean(np.linalg.norm(x64 - xk, axis=1) / nrm)
        eu = np.mean(np.linalg.norm(x64 - xu, axis=1) / nrm)
        assert ek < eu, (name, ek, eu)


def test_kmeans_dequantize_bit_exact(cuda_device):
    r = np.random.default_rng(5)
    for d, cld in ((16, 8), (7, 5), (128, 64), (33, 17)):
        n = 2001
        codes = r.integers(0, 256, (n, cld), dtype=np.uint8)
        cb = r.integers(0, 0x7bff, (n, 16), dtype=np.uint16)
        out = torch.full((n, d + 2), -3.0, dtype=torch.float32, device="cuda")
        dq.dq_dequantize_rows_kmeans4(to_dev(codes), cld, to_dev(cb.view(np.int16)), n, d, out, d + 2)
        got = out.cpu().numpy()
        want = oracle.dequantize_rows_kmeans(codes, cb, d)
        assert np.array_equal(got[:, :d].view(np.uint32), want.view(np.uint32))
        assert np.all(got[:, d:] == -3.0)


def _kmeans_tables(rows, d, seed):
    r = np.random.default_rng(seed)
    out = []
    for n in rows:
        x = r.standard_normal((max(n, 1), d)).astype(np.float32)[:n]
        c, cb, _ = oracle.quantize_rows_kmeans(x, iters=5, codes_ld=dq._codes_ld(d)) if n else (
            np.zeros((0, dq._codes_ld(d)), np.uint8), np.zeros((0, 16), np.uint16), None)
        out.append((c, cb))
    return out


@pytest.mark.parametrize("d,pool", [(16, (1, 1)), (16, (0, 10)), (64, (20, 80)), (128, (1, 1)), (37, (0, 5)),
                                    (256, (3, 9)), (512, (0, 3)), (1024, (1, 1)), (1000, (1, 4)), (64, (0, 2)),
                                    (5, (0, 3)), (1, (1, 1))])
def test_kmeans_bag(cuda_device, d, pool):
    rows = [500, 0, 1300] if pool != (1, 1) else [800, 1200]
    T, B = len(rows), 300
    tabs = _kmeans_tables(rows, d, d)
    r = np.random.default_rng(d + pool[1])
    lens = r.integers(pool[0], pool[1] + 1, T * B)
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    idx = np.concatenate([r.integers(0, max(rows[g // B], 1), lens[g]) if rows[g // B] else np.full(lens[g], 3)
                          for g in range(T * B)]).astype(np.int32)
    fl = torch.zeros(1, dtype=torch.int32, device="cuda")
    dt = [dq.KmeansTable(to_dev(c), to_dev(cb.view(np.int16))) for c, cb in tabs]
    got = dq.embbag_kmeans(dt, d, to_dev(idx), to_dev(off), B, d_flags=fl).cpu().numpy()
    want, mag, skipped = oracle.embbag(tabs, d, idx, off, B, with_abs_sum=True, codebook=True)
    bag_tolerance_check(got, want, mag)
    if pool == (1, 1):
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    assert bool(fl.item() & dq.DQ_FLAG_BAD_INDEX) == (skipped > 0)


@pytest.mark.parametrize("d,pool", [(16, (1, 1)), (64, (1, 1)), (64, (0, 2)), (33, (0, 3)), (48, (1, 2)),
                                    (64, (2, 6)), (16, (3, 5))])
def test_kmeans_bag_many_bags(cuda_device, d, pool):
    # 81,000 bags at d <= 64: under two ids on average they take the 32-bags-per-warp layout
    # (one lane per bag for the bookkeeping, eight bags' rows loaded together), otherwise one
    # warp per bag; empty bags, invalid ids (the empty middle table) and bags of two or more
    # ids mixed in
    rows = [700, 0, 1500]
    T, B = len(rows), 27000
    tabs = _kmeans_tables(rows, d, d + 5)
    r = np.random.default_rng(d * 7 + pool[1])
    lens = r.integers(pool[0], pool[1] + 1, T * B)
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    idx = np.concatenate([r.integers(0, max(rows[g // B], 1), lens[g]) if rows[g // B] else np.full(lens[g], 3)
                          for g in range(T * B)]).astype(np.int32)
    fl = torch.zeros(1, dtype=torch.int32, device="cuda")
    dt = [dq.KmeansTable(to_dev(c), to_dev(cb.view(np.int16))) for c, cb in tabs]
    got = dq.embbag_kmeans(dt, d, to_dev(idx), to_dev(off), B, d_flags=fl).cpu().numpy()
    want, mag, skipped = oracle.embbag(tabs, d, idx, off, B, with_abs_sum=True, codebook=True)
    bag_tolerance_check(got, want, mag)
    one = np.repeat(np.diff(off.astype(np.int64)).reshape(T, B).T == 1, d, axis=1)
    assert np.array_equal(got[one].view(np.uint32), want[one].view(np.uint32))
    assert bool(fl.item() & dq.DQ_FLAG_BAD_INDEX) == (skipped > 0)

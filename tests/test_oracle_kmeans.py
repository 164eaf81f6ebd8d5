"""Pins the oracle's codebook quantizer (per-row k-means, 16 binary16 centroids) and
its dequantization and bag ("Post-Training 4-bit Quantization on Embedding Tables",
section 提出的方法 (proposed method), bullet 3: codebook quantization by k-means
clustering; 主要发现 (main findings), bullet 3).

Reading: centroids start at the 16 levels of the min/max quantizer; `iters` Lloyd
iterations in binary32 (nearest centroid by |x - c|, ties to the lower index; the mean
of a cluster = the binary64 sum of its members in index order / their count in
binary64, rounded once to binary32; empty clusters keep their centroid); stored as
binary16; final codes = nearest stored centroid."""
from fractions import Fraction

import numpy as np
import pytest
from sklearn.cluster import KMeans

import oracle
from tests.exact import F, round_to_f32


def _levels(x):
    lo, hi = np.float32(x.min()), np.float32(x.max())
    step = np.float32(np.float32(hi - lo) / np.float32(15))
    # fma(j, step, lo) rounded once
    return np.array([round_to_f32(F(j) * F(step) + F(lo)) for j in range(16)], np.float32)


def _nearest(x, c):
    dist = np.abs(x[:, None].astype(np.float32) - c[None, :].astype(np.float32))
    return np.argmin(dist, axis=1)  # first minimum: ties to the lower index


def _unpack(codes, d):
    q = np.zeros(d, np.int64)
    for k in range(d):
        q[k] = (codes[k // 2] >> (4 * (k % 2))) & 15
    return q


def test_zero_iterations_are_the_min_max_levels():
    r = np.random.default_rng(0)
    for d in (3, 16, 37, 128):
        x = r.standard_normal((1, d)).astype(np.float32)
        codes, cb, loss = oracle.quantize_rows_kmeans(x, iters=0)
        lev = _levels(x[0])
        assert np.array_equal(cb[0], lev.astype(np.float16).view(np.uint16))
        C = cb[0].view(np.float16).astype(np.float32)
        assert np.array_equal(_unpack(codes[0], d), _nearest(x[0], C))


def _grouped_row(r, lo, hi, per_group, jitter, grid=None):
    """Values in 16 groups around the uniform levels of [lo, hi] (jitter as a fraction of
    the level spacing, < 1/2, so each initial level is nearest to its own group only);
    lo and hi themselves are members, so they are the row's min and max."""
    sp = (hi - lo) / 15
    vals = [lo, hi]
    for j in range(16):
        n = per_group[j] - (1 if j in (0, 15) else 0)
        v = lo + j * sp + r.uniform(-jitter, jitter, n) * sp
        vals.append(np.clip(v, lo, hi))
    x = np.concatenate([np.atleast_1d(np.asarray(v, np.float64)) for v in vals])
    if grid:
        x = np.round(x / grid) * grid
    return r.permutation(x).astype(np.float32)


def test_lloyd_iterations_match_scikit_learn():
    # scikit-learn's Lloyd k-means in binary64 from the same initial centroids; no cluster
    # ever empties (scikit-learn would relocate an empty one), and the groups are far
    # enough apart that binary32 rounding cannot move a value across a boundary
    r = np.random.default_rng(1)
    for trial in range(20):
        per = r.integers(1, 7, 16)
        x = _grouped_row(r, r.uniform(-4, -1), r.uniform(1, 4), per, jitter=0.3)
        d = x.size
        iters = int(r.integers(1, 12))
        codes, cb, loss = oracle.quantize_rows_kmeans(x[None, :], iters=iters)
        km = KMeans(n_clusters=16, init=_levels(x).astype(np.float64)[:, None], n_init=1, max_iter=iters,
                    tol=0.0, algorithm="lloyd").fit(x.astype(np.float64)[:, None])
        want = km.cluster_centers_[:, 0]
        got = cb[0].view(np.float16).astype(np.float64)
        # stored centroids are the binary16 roundings of the means
        assert np.all(np.abs(got - want) <= np.abs(want) * 2.0 ** -11 + 1e-7), (trial, got, want)
        C = cb[0].view(np.float16).astype(np.float32)
        assert np.array_equal(_unpack(codes[0], d), _nearest(x, C))


def test_rows_on_binary16_levels_are_exact():
    # groups of equal values on a 1/64 grid near the uniform levels of [-8, 8]: one
    # iteration moves every centroid onto its group's value (the mean of equal values is
    # exact here), which binary16 holds exactly, so the row is reproduced with loss 0
    r = np.random.default_rng(2)
    for d_extra in (0, 40, 100):
        per = 1 + r.multinomial(d_extra, np.ones(16) / 16) + np.isin(np.arange(16), [0, 15])
        sp = 16 / 15
        lev = np.round((-8 + np.arange(16) * sp + r.uniform(-0.2, 0.2, 16) * sp) * 64) / 64
        lev[0], lev[15] = -8.0, 8.0
        x = r.permutation(np.repeat(lev, per)).astype(np.float32)
        codes, cb, loss = oracle.quantize_rows_kmeans(x[None, :], iters=3)
        C = cb[0].view(np.float16).astype(np.float32)
        xhat = C[_unpack(codes[0], x.size)]
        assert loss[0] == 0 and np.array_equal(xhat, x)
        assert np.array_equal(np.sort(C), lev.astype(np.float32))


def test_constant_and_two_value_rows():
    x = np.full((1, 8), 0.375, np.float32)
    codes, cb, loss = oracle.quantize_rows_kmeans(x)
    assert loss[0] == 0 and not codes.any()
    assert cb[0, 0] == np.float16(0.375).view(np.uint16)
    x = np.array([[1.0, -1.0, 1.0, -1.0, 1.0]], np.float32)
    codes, cb, loss = oracle.quantize_rows_kmeans(x)
    q = _unpack(codes[0], 5)
    assert list(q) == [15, 0, 15, 0, 15] and loss[0] == 0


def test_dequantize_is_a_table_lookup():
    r = np.random.default_rng(3)
    n, d = 50, 21
    codes = r.integers(0, 256, (n, 11), dtype=np.uint8)
    cb = r.integers(0, 0x7bff, (n, 16), dtype=np.uint16)
    out = oracle.dequantize_rows_kmeans(codes, cb, d)
    for i in range(n):
        want = cb[i].view(np.float16).astype(np.float32)[_unpack(codes[i], d)]
        assert np.array_equal(out[i], want)


def test_codebook_bag_sums_exactly():
    r = np.random.default_rng(4)
    n, d, B = 30, 6, 9
    codes = r.integers(0, 256, (n, 3), dtype=np.uint8)
    cb = (r.integers(-64, 64, (n, 16)).astype(np.float16) / np.float16(8)).view(np.uint16)
    lens = r.integers(0, 5, B)
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    idx = r.integers(0, n, off[-1]).astype(np.int32)
    out, mag, skipped = oracle.embbag([(codes, cb)], d, idx, off, B, with_abs_sum=True, codebook=True)
    deq = oracle.dequantize_rows_kmeans(codes, cb, d)
    for b in range(B):
        exact = [sum((Fraction(float(deq[i, k])) for i in idx[off[b]:off[b + 1]]), Fraction(0)) for k in range(d)]
        assert [float(v) for v in out[b]] == [float(round_to_f32(e)) for e in exact]
    assert skipped == 0


def test_mean_sums_members_in_index_order():
    # t = 2^-60 vanishes when added to 1 in binary64. Members [1, t, -1, t]: one addition
    # after the other gives ((1 + t) - 1) + t = t, so the mean is t / 4 = 2^-62; a pairwise
    # order would give (1 + t) + (-1 + t) = 0 and the exact mean is 2^-61
    c0 = np.arange(16, dtype=np.float32)
    a = np.full(4, 5, np.int32)
    t = np.float32(2.0 ** -60)
    got = oracle.kmeans_means(np.array([1.0, t, -1.0, t], np.float32), a, c0)
    assert got[5] == np.float32(2.0 ** -62)
    # [1, t, -1]: (1 + t) - 1 = 0, a +0 mean
    got = oracle.kmeans_means(np.array([1.0, t, -1.0], np.float32), a[:3], c0)
    assert got[5] == 0.0 and not np.signbit(got[5])
    # the other clusters have no members and keep their centroids
    assert np.array_equal(np.delete(got, 5), np.delete(c0, 5))


def test_mean_of_exactly_summed_members_is_the_rounded_exact_mean():
    # members on a 2^-20 grid below 2^10: every binary64 partial sum is exact, so the
    # centroid is the exact mean rounded to binary32 -- once when the count is a power
    # of two (the binary64 quotient is then exact too), and within binary32's half ulp
    # plus binary64's quotient rounding otherwise
    r = np.random.default_rng(7)
    for trial in range(300):
        d = int(r.integers(1, 200))
        x = (r.integers(-2 ** 30, 2 ** 30, d) * 2.0 ** -20).astype(np.float32)
        a = r.integers(0, 16, d).astype(np.int32)
        c0 = r.standard_normal(16).astype(np.float32)
        got = oracle.kmeans_means(x, a, c0)
        for j in range(16):
            m = a == j
            n = int(m.sum())
            if n == 0:
                assert got[j] == c0[j]
                continue
            exact = sum((F(v) for v in x[m]), Fraction(0)) / n
            want = round_to_f32(exact)
            if n & (n - 1) == 0:
                assert got[j] == want, (trial, j)
            else:
                assert abs(F(got[j]) - exact) <= abs(F(want) - exact) + abs(exact) * Fraction(1, 2 ** 52), (trial, j)


def test_mean_step_keeps_empty_clusters_and_counts_every_member():
    x = np.array([3.0, 5.0, -2.0, 7.0], np.float32)
    a = np.array([2, 2, 9, 2], np.int32)
    c0 = np.full(16, -1.0, np.float32)
    got = oracle.kmeans_means(x, a, c0)
    assert got[2] == np.float32(5.0) and got[9] == np.float32(-2.0)
    assert np.all(np.delete(got, [2, 9]) == -1.0)

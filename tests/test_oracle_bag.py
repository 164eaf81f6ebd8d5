"""Pins the oracle's dequantizer and sum-pooled INT4 embedding bag.

Lookup: "Deep Learning Recommendation Model for Personalization and
Recommendation Systems", section 提出的方法 (proposed method), bullet 1 (sparse
categorical features are mapped to dense vectors by embedding-table lookups);
sum pooling over a bag of ids. Row format: 4-bit codes with an FP16 scale and
bias per row ("Post-Training 4-bit Quantization on Embedding Tables", section
提出的方法 / proposed method, bullet 2).
"""
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from int4_row_wise_b200 import workloads as W
from tests.exact import F, round_to_f32


def _unpack(codes, d):
    q = np.zeros((codes.shape[0], 2 * codes.shape[1]), np.int64)
    q[:, 0::2] = codes & 15
    q[:, 1::2] = codes >> 4
    return q[:, :d]


@pytest.mark.parametrize("d", [1, 7, 16, 128])
def test_dequantize_is_exact_fma(d):
    """xhat = q*S + B rounded once: q*S + B is exact in binary64 (a 4-bit code
    times an 11-bit significand plus an 11-bit significand), so one numpy cast to
    binary32 gives the correctly rounded value."""
    codes, sb = W.random_packed_table(3000, d, seed=d)
    got = oracle.dequantize_rows(codes, sb, d)
    S = sb[:, 0].view(np.float16).astype(np.float64)[:, None]
    B = sb[:, 1].view(np.float16).astype(np.float64)[:, None]
    want = (_unpack(codes, d) * S + B).astype(np.float32)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def _tables(T, n, d, seed):
    return [W.random_packed_table(n + 7 * t, d, seed=seed + t) for t in range(T)]


def test_bag_small_case_exact_rational():
    """Tiny case against the exact rational sum of the dequantized rows, rounded
    once (ties to even): the binary64 sum of <= 9 binary32 terms is exact here."""
    d, T, B = 5, 2, 6
    tabs = _tables(T, 11, d, 3)
    r = np.random.default_rng(0)
    lens = r.integers(0, 10, T * B)
    off = np.zeros(T * B + 1, np.int32)
    off[1:] = np.cumsum(lens)
    idx = np.concatenate([r.integers(0, tabs[g // B][0].shape[0], lens[g]) for g in range(T * B)]).astype(np.int32)
    out, mag, skipped = oracle.embbag(tabs, d, idx, off, B, with_abs_sum=True)
    assert skipped == 0
    deq = [oracle.dequantize_rows(c, s, d) for c, s in tabs]
    for g in range(T * B):
        t, b = divmod(g, B)
        ids = idx[off[g]:off[g + 1]]
        for k in range(d):
            exact = sum((F(deq[t][i, k]) for i in ids), Fraction(0))
            assert out[b, t * d + k] == round_to_f32(exact)
            assert mag[b, t * d + k] == float(sum((abs(F(deq[t][i, k])) for i in ids), Fraction(0)))


def test_bag_pooling_one_is_the_dequantized_row_and_empty_is_zero():
    d, T, B = 64, 3, 50
    tabs = _tables(T, 1000, d, 5)
    r = np.random.default_rng(1)
    lens = r.integers(0, 2, T * B)              # bags of 0 or 1 ids
    off = np.zeros(T * B + 1, np.int32)
    off[1:] = np.cumsum(lens)
    idx = r.integers(0, 1000, int(off[-1])).astype(np.int32)
    out, _, _ = oracle.embbag(tabs, d, idx, off, B)
    deq = [oracle.dequantize_rows(c, s, d) for c, s in tabs]
    for g in range(T * B):
        t, b = divmod(g, B)
        o = out[b, t * d:(t + 1) * d]
        if lens[g] == 0:
            assert np.all(o.view(np.uint32) == 0)  # +0
        else:
            assert np.array_equal(o.view(np.uint32), deq[t][idx[off[g]]].view(np.uint32))


def test_bag_permutation_within_bag():
    """Reordering the ids of a bag changes the binary64 sum's binary32 rounding by
    at most one ulp."""
    d, B = 32, 40
    tabs = _tables(1, 500, d, 9)
    r = np.random.default_rng(2)
    lens = r.integers(20, 81, B)
    off = np.zeros(B + 1, np.int32)
    off[1:] = np.cumsum(lens)
    idx = r.integers(0, 500, int(off[-1])).astype(np.int32)
    idx2 = idx.copy()
    for b in range(B):
        idx2[off[b]:off[b + 1]] = r.permutation(idx[off[b]:off[b + 1]])
    o1, _, _ = oracle.embbag(tabs, d, idx, off, B)
    o2, _, _ = oracle.embbag(tabs, d, idx2, off, B)
    diff = np.abs(o1.view(np.int32).astype(np.int64) - o2.view(np.int32).astype(np.int64))
    assert diff.max() <= 1


def test_bag_skips_bad_ids_and_decreasing_offsets():
    d, B = 16, 4
    tabs = _tables(1, 10, d, 11)
    idx = np.array([0, 10, -1, 3, 5], np.int32)
    off = np.array([0, 2, 4, 3, 5], np.int32)   # bag 2 has decreasing offsets
    out, _, skipped = oracle.embbag(tabs, d, idx, off, B)
    deq = oracle.dequantize_rows(*tabs[0], d)
    assert skipped == 3
    assert np.array_equal(out[0], deq[0])
    assert np.array_equal(out[1], deq[3])
    assert np.all(out[2] == 0)
    assert np.array_equal(out[3], (deq[3].astype(np.float64) + deq[5]).astype(np.float32))


def test_byte_ratio_golden():
    """13.28% of the binary32 size at d=128 with FP16 scale and bias
    ("Post-Training 4-bit Quantization on Embedding Tables", section 主要发现 /
    main findings, bullet 4); fixture tests/golden/byte_ratio.txt."""
    path = os.path.join(os.path.dirname(__file__), "golden", "byte_ratio.txt")
    vals = dict(l.split("=") for l in open(path) if "=" in l and not l.startswith("#"))
    d = int(vals["d"])
    wl = W.workload("tiny")
    x = np.repeat(W.table_rows(wl, 0, 0, 64), d // 16, axis=1)
    codes, sb, _, _ = oracle.quantize_rows(x)
    ratio = (codes.nbytes + sb.nbytes) / x.nbytes
    assert ratio == Fraction(int(vals["packed_bytes_per_row"]), 4 * d) == Fraction(68, 512)
    assert round(100 * ratio, 2) == float(vals["percent"])

"""Pins the oracle's bag backward + SGD step + re-quantization of touched rows.

Reading (the DQRM repository page trains INT4 embedding tables with quantization-
aware training on binary32 masters; the pages fix no arithmetic for the step):
entries (key = row_base[t] + id, position p) sorted by (key, p); a row's gradient is
the plain binary64 sum of its entries' output-gradient rows, from +0, one addition
after the other in that list order, rounded once to binary32 (G); the master
becomes fma(-lr, G, w); every touched row is quantized again.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests.exact import F, round_to_f32


def _tables(T, n, d, seed, cld=None):
    r = np.random.default_rng(seed)
    cld = cld or (d + 1) // 2
    W = [r.standard_normal((n, d)).astype(np.float32) for _ in range(T)]
    C = [np.zeros((n, cld), np.uint8) for _ in range(T)]
    S = [np.zeros((n, 2), np.uint16) for _ in range(T)]
    return W, C, S


def _quantize_into(W, C, S):
    for t in range(len(W)):
        c, sb, _, _ = oracle.quantize_rows(W[t])
        C[t][:, :c.shape[1]] = c
        S[t][:] = sb


def _bags(T, B, n, lo, hi, seed):
    r = np.random.default_rng(seed)
    lens = r.integers(lo, hi + 1, T * B)
    off = np.zeros(T * B + 1, np.int64)
    off[1:] = np.cumsum(lens)
    idx = np.concatenate([r.integers(0, n, lens[g]) for g in range(T * B)] + [np.zeros(0, np.int64)])
    return idx.astype(np.int32), off.astype(np.int32)


def _dyadic_grad(B, cols, seed):
    # k * 2^-40 with |k| < 2^44: every binary64 sum of a few hundred of them is exact,
    # so no summation order can matter and G is the exact sum rounded once.
    r = np.random.default_rng(seed)
    k = r.integers(-(1 << 20), 1 << 20, (B, cols)).astype(np.float64)
    e = r.integers(-40, -16, (B, cols)).astype(np.float64)
    return (k * np.exp2(e)).astype(np.float32)


@pytest.mark.parametrize("lr", [0.03125, float(np.float32(1 / 3)), 1.7])
def test_sgd_is_exact_gradient_then_one_fma(lr):
    T, B, n, d = 3, 40, 9, 6
    W, C, S = _tables(T, n, d, 0)
    _quantize_into(W, C, S)
    W0 = [w.copy() for w in W]
    C0 = [c.copy() for c in C]
    S0 = [s.copy() for s in S]
    idx, off = _bags(T, B, n, 0, 5, 1)
    g = _dyadic_grad(B, T * d, 2)
    assert oracle.embbag_bwd_sgd(W, C, S, d, idx, off, B, g, lr) == 0
    lrF = F(np.float32(lr))
    for t in range(T):
        G = [[Fraction(0)] * d for _ in range(n)]
        touched = set()
        for b in range(B):
            gg = t * B + b
            for p in range(off[gg], off[gg + 1]):
                i = int(idx[p])
                touched.add(i)
                for k in range(d):
                    G[i][k] += F(g[b, t * d + k])
        for i in range(n):
            if i not in touched:
                assert np.array_equal(W[t][i], W0[t][i]) and np.array_equal(C[t][i], C0[t][i])
                assert np.array_equal(S[t][i], S0[t][i])
                continue
            for k in range(d):
                Gk = F(round_to_f32(G[i][k]))
                want = round_to_f32(F(W0[t][i, k]) - lrF * Gk)
                assert W[t][i, k] == want, (t, i, k)
        # e: touched rows carry the quantizer's codes of their new masters
        rows = sorted(touched)
        c, sb, _, _ = oracle.quantize_rows(np.ascontiguousarray(W[t][rows]))
        assert np.array_equal(C[t][rows], c) and np.array_equal(S[t][rows], sb)


def _one_row_case(prefix, row_grads):
    """One table, one-hot bags: `prefix` bags of row 0 come first, then one bag of row 1
    per value in row_grads (its output gradient, d = 1). W = 0 and lr = 1, so row 1's
    new master is -G."""
    n_b = prefix + len(row_grads)
    idx = np.array([0] * prefix + [1] * len(row_grads), np.int32)
    off = np.arange(n_b + 1, dtype=np.int32)
    g = np.zeros((n_b, 1), np.float32)
    g[prefix:, 0] = np.asarray(row_grads, np.float64).astype(np.float32)
    W = [np.zeros((2, 1), np.float32)]
    C = [np.zeros((2, 1), np.uint8)]
    S = [np.zeros((2, 2), np.uint16)]
    assert oracle.embbag_bwd_sgd(W, C, S, 1, idx, off, n_b, g, 1.0) == 0
    return W[0][1, 0]


TINY = 2.0 ** -54  # a quarter of the binary64 ulp of 1


@pytest.mark.parametrize("prefix", [0, 1, 32, 63])
@pytest.mark.parametrize("tiny_at", [(2, 3, 4), (64, 65, 66), (30, 31, 32, 33)])
def test_gradient_is_a_binary64_sum_not_the_exact_one(prefix, tiny_at):
    # 1 then 2^-24 (the binary32 midpoint above 1, exact in binary64), then zeros and a
    # few 2^-54 later on. One addition at a time in binary64, each 2^-54 falls below half
    # an ulp of the running sum and is lost, wherever it sits in the list: G = 1 + 2^-24,
    # a binary32 tie, rounds to even, G = 1. The exact sum lies above the midpoint and
    # would round to 1 + 2^-23.
    grads = [0.0] * 70
    grads[0], grads[1] = 1.0, 2.0 ** -24
    for e in tiny_at:
        grads[e] = TINY
    exact = Fraction(1) + Fraction(1, 2 ** 24) + len(tiny_at) * F(np.float64(TINY))
    assert round_to_f32(exact) == 1 + 2.0 ** -23
    assert _one_row_case(prefix, grads) == -1.0


def test_gradient_is_summed_in_list_order():
    # The same values, the 2^-54 first: 3 * 2^-54 is exact, 1 + 3 * 2^-54 rounds up to
    # 1 + 2^-52 in binary64, adding 2^-24 is exact, and the binary32 rounding now goes
    # up: G = 1 + 2^-23. Only the order of the entries in the list differs from the
    # case above (a binary32 running sum would give 1 both ways).
    assert _one_row_case(5, [TINY, TINY, TINY, 1.0, 2.0 ** -24]) == -(1 + 2.0 ** -23)
    assert _one_row_case(5, [1.0, 2.0 ** -24, TINY, TINY, TINY]) == -1.0
    # cancellation: 1 + 2^-60 loses the 2^-60 in binary64; after -1 it is 0
    assert _one_row_case(0, [1.0, 2.0 ** -60, -1.0]) == 0.0
    assert _one_row_case(0, [1.0, -1.0, 2.0 ** -60]) == -(2.0 ** -60)


def test_invalid_ids_skip_duplicates_count_twice_and_tables_are_separate():
    d = 2
    W = [np.zeros((3, d), np.float32), np.zeros((3, d), np.float32)]
    C = [np.zeros((3, 1), np.uint8) for _ in range(2)]
    S = [np.zeros((3, 2), np.uint16) for _ in range(2)]
    # table 0: bag0 = [1, 1, 7], bag1 = [-1]; table 1: bag0 = [1], bag1 = [2, 1]
    idx = np.array([1, 1, 7, -1, 1, 2, 1], np.int32)
    off = np.array([0, 3, 4, 5, 7], np.int32)
    g = np.array([[1, 2, 10, 20], [3, 4, 30, 40]], np.float32)
    assert oracle.embbag_bwd_sgd(W, C, S, d, idx, off, 2, g, 0.5) == 2
    assert W[0].tolist() == [[0, 0], [-1, -2], [0, 0]]
    assert W[1].tolist() == [[0, 0], [-20, -30], [-15, -20]]
    # touched rows only are quantized again
    for t, rows in ((0, [1]), (1, [1, 2])):
        c, sb, _, _ = oracle.quantize_rows(np.ascontiguousarray(W[t][rows]))
        assert np.array_equal(C[t][rows], c) and np.array_equal(S[t][rows], sb)
    assert not C[0][[0, 2]].any() and not S[0][[0, 2]].any() and not S[1][0].any()


@pytest.mark.parametrize("bad", ["decreasing", "first", "last"])
def test_bad_offsets_change_nothing(bad):
    d, B = 3, 4
    W, C, S = _tables(1, 5, d, 3)
    _quantize_into(W, C, S)
    before = [W[0].copy(), C[0].copy(), S[0].copy()]
    idx = np.array([0, 1, 2, 3, 4, 0], np.int32)
    off = np.array([0, 2, 3, 5, 6], np.int32)
    if bad == "decreasing":
        off[2] = 1
    elif bad == "first":
        off[0] = 1
    else:
        off[-1] = 5
    g = np.ones((B, d), np.float32)
    assert oracle.embbag_bwd_sgd(W, C, S, d, idx, off, B, g, 0.1) == oracle.BAD_OFFSETS
    assert all(np.array_equal(a, b) for a, b in zip([W[0], C[0], S[0]], before))


def test_min_max_mode_requantizes_with_min_max():
    d = 8
    W, C, S = _tables(1, 6, d, 4)
    idx = np.array([2, 5], np.int32)
    off = np.array([0, 1, 2], np.int32)
    g = np.random.default_rng(5).standard_normal((2, d)).astype(np.float32)
    oracle.embbag_bwd_sgd(W, C, S, d, idx, off, 2, g, 0.25, mode=oracle.MINMAX)
    c, sb, _, _ = oracle.quantize_rows(np.ascontiguousarray(W[0][[2, 5]]), mode=oracle.MINMAX)
    assert np.array_equal(C[0][[2, 5]], c) and np.array_equal(S[0][[2, 5]], sb)
    assert not C[0][[0, 1, 3, 4]].any()


def test_sample_updates_exactly_the_sampled_rows():
    # a sample restricts steps c-e to its rows; each sampled row gets what the full
    # call gives it
    T, B, n, d = 2, 60, 40, 4
    W, C, S = _tables(T, n, d, 21)
    idx, off = _bags(T, B, n, 1, 9, 22)
    g = np.random.default_rng(23).standard_normal((B, T * d)).astype(np.float32)
    full = ([w.copy() for w in W], [c.copy() for c in C], [s.copy() for s in S])
    oracle.embbag_bwd_sgd(*full, d, idx, off, B, g, 0.1)
    part = ([w.copy() for w in W], [c.copy() for c in C], [s.copy() for s in S])
    keys = np.array([0, 7, n + 3, n + 39], np.uint32)  # rows 0, 7 of table 0; 3, 39 of table 1
    oracle.embbag_bwd_sgd(*part, d, idx, off, B, g, 0.1, sample_keys=keys)
    picked = {(0, 0), (0, 7), (1, 3), (1, 39)}
    for t in range(T):
        for r in range(n):
            src = full if (t, r) in picked else (W, C, S)
            for k in range(3):
                assert np.array_equal(part[k][t][r], src[k][t][r]), (t, r, k)

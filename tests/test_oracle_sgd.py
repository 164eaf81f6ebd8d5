"""Pins the oracle's bag backward + SGD step + re-quantization of touched rows.

Reading (the DQRM repository page trains INT4 embedding tables with quantization-
aware training on binary32 masters; the pages fix no arithmetic for the step):
entries (key = row_base[t] + id, position p) sorted by (key, p); a row's gradient is
summed in binary64 inside windows of 64 consecutive entries of that sorted list,
then across windows, and rounded once to binary32 (G); the master becomes
fma(-lr, G, w); every touched row is quantized again.
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
    # so the window order cannot matter and G is the exact sum rounded once.
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


def _window_case(prefix, tiny_at):
    """One table, one-hot bags; `prefix` bags of row 0 come first, then 67 bags of row 1
    whose gradients are 1, 2^-24, zeros, and 2^-54 at the entries listed in tiny_at
    (entry numbers counted within row 1's run)."""
    n_b = prefix + 67
    idx = np.array([0] * prefix + [1] * 67, np.int32)
    off = np.arange(n_b + 1, dtype=np.int32)
    g = np.zeros((n_b, 1), np.float32)
    g[prefix + 0, 0] = 1.0
    g[prefix + 1, 0] = 2.0 ** -24
    for e in tiny_at:
        g[prefix + e, 0] = 2.0 ** -54
    W = [np.zeros((2, 1), np.float32)]
    C = [np.zeros((2, 1), np.uint8)]
    S = [np.zeros((2, 2), np.uint16)]
    assert oracle.embbag_bwd_sgd(W, C, S, 1, idx, off, n_b, g, 1.0) == 0
    return W[0][1, 0]


def test_window_split_changes_the_rounding():
    # Entries 64..66 of row 1 (sorted positions 64..66) fall in the second window, whose
    # part 3 * 2^-54 lifts 1 + 2^-24 above the binary32 midpoint: G = 1 + 2^-23.
    assert _window_case(0, [64, 65, 66]) == -(1 + 2.0 ** -23)
    # Inside one window the sum is sequential: each 2^-54 is a quarter of an ulp and is
    # lost, G = 1 + 2^-24 rounds to even, G = 1.
    assert _window_case(0, [2, 3, 4]) == -1.0


def test_windows_are_aligned_on_the_whole_sorted_list():
    # 32 entries of row 0 come first: row 1's entries 32..34 sit at sorted positions
    # 64..66, the second window, so they are summed apart from the 1 and the 2^-24.
    assert _window_case(32, [32, 33, 34]) == -(1 + 2.0 ** -23)
    # (Windows cut at the row's own first entry would put entries 32..34 with the 1.)
    # Entries 29..31 sit at positions 61..63, in the first window with the 1: G = 1.
    assert _window_case(32, [29, 30, 31]) == -1.0


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
    # call gives it (the windows still count every entry)
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

"""Pins the oracle's row-wise greedy INT4 quantizer to exact arithmetic,
brute force and closed forms.

Method: "Post-Training 4-bit Quantization on Embedding Tables" (Guan et al.,
2019), review page, section 提出的方法 (proposed method): row-wise uniform 4-bit
quantization whose clipping thresholds come from a greedy search toward a local
minimum of the squared error (bullet 1), FP16 scale and bias (bullet 2).
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from int4_row_wise_b200 import workloads as W
from tests.exact import (F, exact_codes, exact_loss, loss_error_bound, round_half_even,
                         round_to_f32)

f32 = np.float32


def _rows(d, n, seed, kind="normal"):
    r = np.random.default_rng(seed)
    if kind == "normal":
        return r.standard_normal((n, d)).astype(np.float32)
    if kind == "t3":
        return (r.standard_t(3, (n, d)) * r.lognormal(0, 1, (n, 1))).astype(np.float32)
    if kind == "offset":
        # rows far from zero relative to their range: the binary16 bias error is
        # a sizeable fraction of the scale
        return (r.uniform(-200, 200, (n, 1)) + r.standard_normal((n, d)) * 0.5).astype(np.float32)
    raise ValueError(kind)


def _s(lo, hi):
    # s = fl(fl(hi - lo) / 15): the definition's own binary32 steps, in numpy
    return f32(f32(f32(hi) - f32(lo)) / f32(15))


@pytest.mark.parametrize("d", [2, 3, 5, 8, 16, 33, 64])
def test_loss_matches_exact_arithmetic(d):
    """L(lo, hi) equals the exact sum of squared reconstruction errors within the
    rounding bound of the binary32 pipeline; a dropped term, a wrong sign or an
    off-by-one code would exceed it by orders of magnitude."""
    rng = np.random.default_rng(100 + d)
    xs = _rows(d, 40, d, "t3")
    checked = 0
    for x in xs:
        xmin, xmax = float(x.min()), float(x.max())
        a, b = sorted(rng.uniform(0, 0.45, 2))
        lo = f32(xmin + a * (xmax - xmin))
        hi = f32(xmax - b * (xmax - xmin))
        s = _s(lo, hi)
        qs, gaps = exact_codes(x, lo, s)
        if min(gaps) < 1e-4:
            continue  # a near-tie: the binary32 quotient may round the other way
        lex, errs = exact_loss(x, lo, s, qs)
        got = oracle.row_loss(x, lo, hi)
        bound = loss_error_bound(x, lo, s, qs, errs, d)
        assert abs(F(got) - lex) <= Fraction(bound), (d, float(got), float(lex), bound)
        checked += 1
    assert checked >= 25


def _pairwise_rounded(c):
    if len(c) == 1:
        return c[0]
    h = len(c) // 2
    return round_to_f32(F(_pairwise_rounded(c[:h])) + F(_pairwise_rounded(c[h:])))


@pytest.mark.parametrize("d", [3, 16, 64])
def test_loss_rounding_sequence_bit_exact(d):
    """The oracle's compiled binary32 arithmetic performs exactly the rounding
    sequence of its definition (one rounding for the fused reconstruction, none
    contracted elsewhere), evaluated here in exact rationals with explicit
    round-to-nearest-even after each operation."""
    rng = np.random.default_rng(200 + d)
    for x in _rows(d, 20, 60 + d, "t3"):
        xmin, xmax = float(x.min()), float(x.max())
        lo = f32(xmin + 0.1 * rng.random() * (xmax - xmin))
        hi = f32(xmax - 0.1 * rng.random() * (xmax - xmin))
        s = round_to_f32(F(round_to_f32(F(hi) - F(lo))) / 15)
        c = []
        for xk in x:
            y = F(round_to_f32(F(xk) - F(lo))) / F(s)
            q = min(max(round_half_even(F(round_to_f32(y))), 0), 15)
            xh = round_to_f32(q * F(s) + F(lo))
            e = round_to_f32(F(xk) - F(xh))
            c.append(round_to_f32(F(e) * F(e)))
        p = 1
        while p < d:
            p *= 2
        c += [f32(0)] * (p - d)
        assert oracle.row_loss(x, lo, hi) == _pairwise_rounded(c)


def test_loss_degenerate_clip_is_distance_to_lo():
    # s == 0: every element reconstructs to lo
    x = np.array([0.5, -1.0, 2.0, 0.25], np.float32)
    lex = sum((F(v) - F(0.5)) ** 2 for v in x)
    got = oracle.row_loss(x, 0.5, 0.5)
    assert abs(F(got) - lex) <= Fraction(1e-6) * lex


def _grid_of(x):
    xmin, xmax = x.min(), x.max()
    step = f32(f32(xmax - xmin) / f32(200))
    return xmin, xmax, step


@pytest.mark.parametrize("d", [2, 4, 6, 16])
def test_trace_grid_points_and_walk(d):
    """Every evaluated (lo, hi) is the grid point xmin + i*step / xmax - j*step
    rounded once; the walk starts at (0, 0), makes exactly 168 moves of one step
    each, and the two candidates of a move are (i+1, j) and (i, j+1)."""
    for x in _rows(d, 12, 7 + d):
        xmin, xmax, step = _grid_of(x)
        tr = oracle.greedy_trace(x)
        assert tr["lo"][0] == xmin and tr["hi"][0] == xmax
        i = j = 0
        for m in range(oracle.MOVES):
            lo_l, hi_l = tr["lo"][2 * m + 1], tr["hi"][2 * m + 1]
            lo_r, hi_r = tr["lo"][2 * m + 2], tr["hi"][2 * m + 2]
            assert lo_l == round_to_f32(F(xmin) + (i + 1) * F(step))
            assert hi_l == round_to_f32(F(xmax) - j * F(step))
            assert lo_r == round_to_f32(F(xmin) + i * F(step))
            assert hi_r == round_to_f32(F(xmax) - (j + 1) * F(step))
            ni, nj = int(tr["i"][m]), int(tr["j"][m])
            assert (ni, nj) in ((i + 1, j), (i, j + 1))
            i, j = ni, nj
        assert i + j == 168


@pytest.mark.parametrize("d", [2, 3, 4, 5, 6, 16])
def test_moves_follow_exact_losses(d):
    """Each move goes to the candidate with the lower loss, computed exactly
    (moves whose two losses are closer than the rounding bound are skipped), and
    the reported best is the first minimum over the visited points."""
    decided = 0
    for x in _rows(d, 10, 50 + d, "t3"):
        tr = oracle.greedy_trace(x)
        visited = [(0, 0, tr["loss"][0])]
        for m in range(oracle.MOVES):
            cand = []
            for e in (2 * m + 1, 2 * m + 2):
                lo, hi = tr["lo"][e], tr["hi"][e]
                s = _s(lo, hi)
                qs, gaps = exact_codes(x, lo, s)
                lex, errs = exact_loss(x, lo, s, qs)
                cand.append((lex, loss_error_bound(x, lo, s, qs, errs, d), min(gaps)))
            (ll, bl, gl), (lr, br, gr) = cand
            moved_right = int(tr["j"][m]) > (int(tr["j"][m - 1]) if m else 0)
            if min(gl, gr) > 1e-4 and abs(ll - lr) > Fraction(bl + br):
                assert moved_right == (lr < ll), (d, m)
                decided += 1
            e = 2 * m + 2 if moved_right else 2 * m + 1
            visited.append((int(tr["i"][m]), int(tr["j"][m]), tr["loss"][e]))
        losses = [v[2] for v in visited]
        k = int(np.argmin(losses))  # first occurrence of the minimum
        assert tr["best"] == (visited[k][0], visited[k][1])
        assert tr["lbest"] == losses[k] <= tr["loss"][0]
    assert decided > 300


@pytest.mark.parametrize("d", [2, 3, 4, 5, 6])
def test_brute_force_grid(d):
    """Over the whole grid {i + j <= 168}, no point the greedy walk visited is
    below the grid minimum, and the reported loss is L(i*, j*) recomputed."""
    for x in _rows(d, 3, 300 + d, "t3"):
        xmin, xmax, step = _grid_of(x)
        c, sb, loss, ij = oracle.quantize_rows(x[None, :])
        i_s, j_s = int(ij[0, 0]), int(ij[0, 1])
        lo = round_to_f32(F(xmin) + i_s * F(step))
        hi = round_to_f32(F(xmax) - j_s * F(step))
        assert oracle.row_loss(x, lo, hi) == loss[0]
        grid_min = min(
            oracle.row_loss(x, round_to_f32(F(xmin) + i * F(step)), round_to_f32(F(xmax) - j * F(step)))
            for i in range(169) for j in range(169 - i))
        assert grid_min <= loss[0]


def test_constant_rows_walk_left_and_keep_first_best():
    """A constant row has loss 0 everywhere: every move is a tie (taken to the
    left) and the first-seen best (0, 0) is kept."""
    x = np.full(5, 0.375, np.float32)
    tr = oracle.greedy_trace(x)
    assert np.all(tr["loss"] == 0)
    assert np.array_equal(tr["i"], np.arange(1, 169)) and np.all(tr["j"] == 0)
    assert tr["best"] == (0, 0)


@pytest.mark.parametrize("c", [0.0, 1.0, -1.0, -2.5, 0.125, 1024.0, 0.1, 3.14159, -1e-3, 7e-6])
def test_constant_rows_dequantize_to_fp16_of_the_constant(c):
    x = np.full((1, 16), c, np.float32)
    codes, sb, loss, ij = oracle.quantize_rows(x)
    assert sb[0, 0] == 0 and np.all(codes == 0) and loss[0] == 0 and tuple(ij[0]) == (0, 0)
    back = oracle.dequantize_rows(codes, sb, 16)
    want = np.float32(np.float16(np.float32(c)))
    assert np.all(back.view(np.uint32) == np.full(16, want, np.float32).view(np.uint32))
    if float(np.float16(c)) == c:
        assert np.all(back == np.float32(c))  # fp16-representable constants come back exactly


@pytest.mark.parametrize("d,c,b", [(16, 2.0 ** -3, 0.0), (2, 2.0 ** -5, 0.0), (7, 1.0, -4.0),
                                   (32, 2.0 ** -4, 1.0), (64, 2.0 ** -8, -0.5)])
def test_rows_on_an_exact_16_level_grid(d, c, b):
    """x_k = b + c*q_k with q covering 0 and 15 and every operation exact: the
    min/max quantizer is already lossless, so greedy keeps (0, 0), returns loss 0,
    scale c, bias b and the codes q (packed low nibble first)."""
    r = np.random.default_rng(d)
    q = r.integers(0, 16, d)
    q[0], q[-1] = 0, 15
    x = (b + c * q).astype(np.float32)
    codes, sb, loss, ij = oracle.quantize_rows(x[None, :])
    assert loss[0] == 0 and tuple(ij[0]) == (0, 0)
    assert sb[0, 0] == np.float16(c).view(np.uint16) and sb[0, 1] == np.float16(b).view(np.uint16)
    qq = np.zeros(2 * ((d + 1) // 2), np.int64)
    qq[:d] = q
    assert np.array_equal(codes[0], (qq[0::2] | (qq[1::2] << 4)).astype(np.uint8))


def test_pack_layout_golden():
    # fixture: tests/golden/pack_layout.txt (codes 0..15 and the expected bytes)
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "pack_layout.txt")
    rows = [l.split("|") for l in open(path) if l.strip() and not l.startswith("#")]
    for qtxt, btxt in rows:
        q = np.array([int(v) for v in qtxt.split()])
        want = bytes.fromhex(btxt.strip())
        x = (q * 0.25).astype(np.float32)  # exact 16-level grid with scale 1/4, bias 0
        codes, sb, loss, ij = oracle.quantize_rows(x[None, :])
        assert codes[0].tobytes() == want


@pytest.mark.parametrize("kind", ["t3", "offset"])
def test_codes_and_params_against_exact_rounding(kind):
    """scale16/bias16 are the binary16 roundings (numpy) of the binary32 s and lo*,
    s is within half an ulp of the exact (hi* - lo*)/15, and each code is the
    exact nearest integer of (x - B)/S clamped to [0, 15] (near-ties skipped)."""
    for x in _rows(16, 200, 9, kind):
        codes, sb, loss, ij = oracle.quantize_rows(x[None, :])
        xmin, xmax, step = _grid_of(x)
        lo = round_to_f32(F(xmin) + int(ij[0, 0]) * F(step))
        hi = round_to_f32(F(xmax) - int(ij[0, 1]) * F(step))
        w = round_to_f32(F(hi) - F(lo))
        s = round_to_f32(F(w) / 15)
        assert sb[0, 0] == np.float16(s).view(np.uint16)
        assert sb[0, 1] == np.float16(lo).view(np.uint16)
        S = F(np.float16(s)) if sb[0, 0] else None
        B = F(np.float16(lo))
        q = np.concatenate([codes[0] & 15, codes[0] >> 4])[np.argsort(np.r_[0:16:2, 1:16:2])]
        for k in range(16):
            y = (F(round_to_f32(F(x[k]) - B)) / S)
            if abs(float(y - math.floor(y)) - 0.5) < 1e-5:
                continue
            assert q[k] == min(max(round_half_even(y), 0), 15)


@pytest.mark.parametrize("name", ["tiny", "kaggle", "terabyte", "production", "sweep-16", "sweep-256"])
def test_greedy_not_worse_than_minmax(name):
    """Greedy loss <= plain min/max loss on every sampled row; min/max mode
    reports (0, 0) and L(xmin, xmax)."""
    wl = W.workload(name)
    t = int(np.argmax(wl.rows))
    n = min(wl.rows[t], 400 if wl.d <= 64 else 60)
    x = W.table_rows(wl, t, 0, n)
    _, _, lg, _ = oracle.quantize_rows(x)
    _, _, lm, ijm = oracle.quantize_rows(x, mode=oracle.MINMAX)
    assert np.all(lg <= lm)
    assert np.all(ijm == 0)
    for r in range(0, n, max(n // 8, 1)):
        assert lm[r] == oracle.row_loss(x[r], x[r].min(), x[r].max())

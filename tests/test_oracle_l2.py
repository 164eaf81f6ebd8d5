"""Pins the oracle's normalized l2 error, sqrt(sum (x - xhat)^2) / sqrt(sum x^2) per
row ("Post-Training 4-bit Quantization on Embedding Tables", section 提出的方法 /
proposed method, bullet 5: quantization error measured as normalized l2 loss; the
pages do not define it further)."""
import math
from fractions import Fraction

import numpy as np

import oracle
from int4_row_wise_b200 import workloads as W
from tests.exact import F


def _exact_err(x, xh):
    se = sum((F(a) - F(b)) ** 2 for a, b in zip(x, xh))
    sx = sum(F(a) ** 2 for a in x)
    return math.sqrt(se / sx) if sx else (0.0 if se == 0 else math.inf)


def test_exact_grid_rows_have_zero_error():
    q = np.arange(16)
    x = np.stack([(0.25 * q).astype(np.float32), (-3.0 + 0.0625 * q[::-1]).astype(np.float32)])
    codes, sb, _, _ = oracle.quantize_rows(x)
    err, tot = oracle.row_l2_error(x, codes, sb)
    assert np.all(err == 0) and tot == 0


def test_constant_rows_error_is_the_fp16_rounding():
    for c in (0.1, 3.14159, -7e-3, 1024.0, 65504.0):
        x = np.full((1, 8), c, np.float32)
        codes, sb, _, _ = oracle.quantize_rows(x)
        err, _ = oracle.row_l2_error(x, codes, sb)
        h = np.float32(np.float16(np.float32(c)))
        want = abs(F(np.float32(c)) - F(h)) / abs(F(np.float32(c)))
        assert abs(err[0] - float(want)) <= 1e-15 * max(float(want), 1e-300)


def test_perturbed_reconstructions_against_exact_rationals():
    r = np.random.default_rng(5)
    d = 24
    codes, sb = W.random_packed_table(200, d, seed=3)
    xh = oracle.dequantize_rows(codes, sb, d)
    x = (xh + r.standard_normal(xh.shape).astype(np.float32) * np.float32(1e-3)).astype(np.float32)
    err, tot = oracle.row_l2_error(x, codes, sb)
    for i in range(0, 200, 7):
        assert abs(err[i] - _exact_err(x[i], xh[i])) <= 1e-13 * err[i]
    assert abs(tot - sum(_exact_err(x[i], xh[i]) for i in range(200))) <= 1e-12 * tot


def test_zero_rows():
    x = np.zeros((2, 4), np.float32)
    codes = np.array([[0, 0], [0x10, 0]], np.uint8)
    sb = np.array([[0, 0], [np.float16(1.0).view(np.uint16), 0]], np.uint16)
    err, _ = oracle.row_l2_error(x, codes, sb)
    assert err[0] == 0 and err[1] == math.inf

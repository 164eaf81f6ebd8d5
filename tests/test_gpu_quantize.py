"""GPU parity of dq_quantize_rows_int4 against the oracle, element by element:
codes, FP16 scale/bias, chosen grid indices and loss bit-identical on every row.

Method: "Post-Training 4-bit Quantization on Embedding Tables", section
提出的方法 (proposed method), bullets 1-2."""
import numpy as np
import pytest

import int4_row_wise_b200 as dq
import oracle
from int4_row_wise_b200 import workloads as W
from tests.gpu_util import assert_quant_parity, gpu_quantize

pytestmark = pytest.mark.gpu


def _rows(n, d, seed, kind):
    r = np.random.default_rng(seed)
    if kind == "normal":
        return r.standard_normal((n, d)).astype(np.float32)
    if kind == "t3":
        return (r.standard_t(3, (n, d)) * r.lognormal(0, 1, (n, 1))).astype(np.float32)
    if kind == "offset":
        return (r.uniform(-200, 200, (n, 1)) + r.standard_normal((n, d)) * 0.5).astype(np.float32)
    if kind == "tiny":
        return (r.uniform(-1, 1, (n, d)) * 3e-4).astype(np.float32)  # subnormal fp16 scales
    raise ValueError(kind)


def test_tiny_workload_every_row(cuda_device):
    wl = W.workload("tiny")
    x = W.table_rows(wl, 0)
    for mode in (dq.DQ_MODE_GREEDY, dq.DQ_MODE_MINMAX):
        assert_quant_parity(x, mode)


@pytest.mark.parametrize("d", [1, 2, 3, 4, 5, 7, 8, 9, 13, 16, 17, 24, 31, 32, 33, 48, 64, 65, 100,
                               128, 129, 200, 256, 300, 512, 777, 1024])
def test_every_width(cuda_device, d):
    # ragged row counts (not a multiple of the rows a block holds)
    n = max(7, min(1500, 60000 // d)) + 3
    x = _rows(n, d, d, "t3" if d % 2 else "normal")
    assert_quant_parity(x)


@pytest.mark.parametrize("kind", ["t3", "offset", "tiny", "normal"])
@pytest.mark.parametrize("d", [16, 64, 128, 256])
def test_value_shapes(cuda_device, kind, d):
    x = _rows(max(200, 40000 // d), d, 7 * d + len(kind), kind)
    assert_quant_parity(x)
    assert_quant_parity(x, dq.DQ_MODE_MINMAX)


@pytest.mark.parametrize("d,x_ld,codes_ld,x_offset", [
    (16, 20, 8, 0), (16, 16, 9, 1), (64, 67, 40, 3), (128, 128, 64, 1), (32, 33, 17, 2), (5, 9, 4, 1),
])
def test_strides_and_alignment(cuda_device, d, x_ld, codes_ld, x_offset):
    x = _rows(333, d, 5 + d, "t3")
    g = gpu_quantize(x, x_ld=x_ld, codes_ld=codes_ld, x_offset=x_offset)
    o = oracle.quantize_rows(x)
    assert np.array_equal(g[0], o[0]) and np.array_equal(g[1], o[1]) and np.array_equal(g[3], o[3])
    assert np.array_equal(g[2].view(np.uint32), o[2].view(np.uint32))


@pytest.mark.parametrize("name", ["kaggle", "terabyte", "production", "sweep-16", "sweep-32",
                                  "sweep-64", "sweep-128", "sweep-256"])
def test_workload_samples(cuda_device, name):
    """Rows of each workload: the start of its largest and its smallest table (the
    Kaggle-shaped largest tables have subnormal binary16 scales)."""
    wl = W.workload(name)
    n = {16: 6000, 32: 4000, 64: 2000, 128: 1200, 256: 600}[wl.d]
    for t in {int(np.argmax(wl.rows)), int(np.argmin(wl.rows))}:
        x = W.table_rows(wl, t, 0, min(n, wl.rows[t]))
        assert_quant_parity(x)


def test_special_rows(cuda_device):
    d = 16
    rows = [np.full(d, c, np.float32) for c in (0.0, 1.0, -2.5, 0.1, 1024.0, 7e-6)]
    q = np.arange(16)
    rows.append((0.125 * q).astype(np.float32))                   # exact 16-level grid
    rows.append((3.0 + 0.0625 * q[::-1]).astype(np.float32))
    rows.append(np.where(q % 2, 1e-39, 2e-39).astype(np.float32))  # subnormal inputs, tiny range
    rows.append(np.linspace(-1e30, 1e30, d).astype(np.float32))    # huge but fp32-finite range
    r = np.random.default_rng(11)
    rows.append((1000.0 + 1e-3 * r.standard_normal(d)).astype(np.float32))  # offset >> range: IEEE walk
    rows.append((-3e4 + 0.05 * r.standard_normal(d)).astype(np.float32))
    x = np.stack(rows)
    g, o = assert_quant_parity(x)
    assert np.all(g[1][:6, 0] == 0) and np.all(g[0][:6] == 0)
    assert g[2][6] == 0 and tuple(g[3][6]) == (0, 0)


def test_flags(cuda_device):
    d = 16
    x = np.random.default_rng(0).standard_normal((40, d)).astype(np.float32)
    assert gpu_quantize(x, flags=True)[4] == 0
    x[3, 5] = np.nan
    x[7, 0] = np.inf
    x[9] = np.linspace(-1e6, 1e6, d)  # scale ~ 1.3e5 > 65504: binary16 overflow
    fl = gpu_quantize(x, flags=True)[4]
    assert fl & dq.DQ_FLAG_NONFINITE and fl & dq.DQ_FLAG_FP16_OVERFLOW
    assert not fl & (dq.DQ_FLAG_BAD_INDEX | dq.DQ_FLAG_BAD_OFFSETS)


def test_zero_rows_and_repeat_calls(cuda_device):
    x = _rows(100, 16, 1, "t3")
    a = gpu_quantize(x)
    b = gpu_quantize(x)
    for u, v in zip(a[:4], b[:4]):
        assert np.array_equal(u, v)
    import torch
    dq.dq_quantize_rows_int4(None, 0, 16, 16, None, 8, None)
    torch.cuda.synchronize()


def _tie_rows(n, d, seed):
    """Rows whose elements sit at (or within an ulp of) half-integer quotients for
    both candidates of the first greedy move, so the division-free codes have to
    defer to IEEE division on most elements."""
    r = np.random.default_rng(seed)
    rows = []
    for _ in range(n):
        R = np.float32(r.uniform(0.5, 4.0))
        off = np.float32(r.uniform(-2, 2))
        step = np.float32(R / np.float32(200))
        lo1 = np.float32(off + step)             # left candidate: (xmin + step, xmax)
        hi1 = np.float32(off + R - step)         # right candidate: (xmin, xmax - step)
        s_l = np.float32(np.float32((off + R) - lo1) / np.float32(15))
        s_r = np.float32(np.float32(hi1 - off) / np.float32(15))
        k = r.integers(0, 15, d - 2)
        half = np.where(r.random(d - 2) < 0.5, lo1 + (k + 0.5) * s_l, off + (k + 0.5) * s_r).astype(np.float32)
        # each tie value itself or its neighbour one ulp up or down
        direction = np.where(r.random(d - 2) < 0.5, np.inf, -np.inf).astype(np.float32)
        half = np.where(r.random(d - 2) < 0.5, half, np.nextafter(half, direction))
        rows.append(np.concatenate([[off, off + R], half]).astype(np.float32))
    return np.stack(rows)


@pytest.mark.parametrize("d", [16, 64])
def test_rows_built_on_rounding_ties(cuda_device, d):
    x = _tie_rows(800 if d == 16 else 200, d, d)
    assert_quant_parity(x)


@pytest.mark.parametrize("d", [32, 64, 128, 256])
@pytest.mark.parametrize("mode", [dq.DQ_MODE_GREEDY, dq.DQ_MODE_MINMAX])
def test_rows_of_one_warp_on_different_paths(cuda_device, d, mode):
    # rows that share a warp (d >= 32) but need different walks: normal rows next to
    # constant rows (no walk), rows outside the fast path's range (IEEE walk: huge range,
    # offset far above the range, subnormal values), in every group of consecutive rows
    r = np.random.default_rng(d)
    specials = [
        lambda: np.full(d, 2.5, np.float32),
        lambda: np.linspace(-1e30, 1e30, d).astype(np.float32),
        lambda: (1000.0 + 1e-3 * r.standard_normal(d)).astype(np.float32),
        lambda: np.where(np.arange(d) % 2, 1e-39, 3e-39).astype(np.float32),
        lambda: np.zeros(d, np.float32),
    ]
    rows = []
    for i in range(600):
        rows.append(specials[(i // 3) % len(specials)]() if i % 3 == 1 else r.standard_normal(d).astype(np.float32))
    assert_quant_parity(np.stack(rows), mode=mode)

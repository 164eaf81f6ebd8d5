"""Helpers for the GPU parity tests: run the CUDA path through the binding and
compare with the oracle on the same inputs."""
import math

import numpy as np
import torch

import int4_row_wise_b200 as dq
import oracle


def to_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def gpu_quantize(x: np.ndarray, mode=dq.DQ_MODE_GREEDY, x_ld=None, codes_ld=None, x_offset=0,
                 flags=False):
    """Quantize host rows on the GPU through dq_quantize_rows_int4; returns numpy
    (codes [n, (d+1)//2], scale_bias uint16 [n, 2], loss [n], best_ij [n, 2], flags)."""
    n, d = x.shape
    ld = d if x_ld is None else x_ld
    buf = np.zeros((n * ld + x_offset + 4,), np.float32)
    view = buf[x_offset:x_offset + n * ld].reshape(n, ld)
    view[:, :d] = x
    xd = to_dev(buf)
    cld = (d + 1) // 2 if codes_ld is None else codes_ld
    codes = torch.full((max(n, 1), cld), 0xAB, dtype=torch.uint8, device="cuda")
    sb = torch.zeros((max(n, 1), 2), dtype=torch.int16, device="cuda")
    loss = torch.zeros(max(n, 1), dtype=torch.float32, device="cuda")
    ij = torch.zeros((max(n, 1), 2), dtype=torch.uint8, device="cuda")
    fl = torch.zeros(1, dtype=torch.int32, device="cuda") if flags else None
    dq.dq_quantize_rows_int4(xd.data_ptr() + 4 * x_offset, n, d, ld, codes, cld, sb, loss, ij, mode, fl)
    torch.cuda.synchronize()
    c = codes.cpu().numpy()
    # bytes past the row's (d+1)//2 must be untouched
    assert np.all(c[:n, (d + 1) // 2:] == 0xAB)
    return (c[:n, :(d + 1) // 2], sb.cpu().numpy().view(np.uint16)[:n], loss.cpu().numpy()[:n],
            ij.cpu().numpy()[:n], int(fl.item()) if flags else None)


def compare_quant(g, o, d):
    """Rows where (codes, scale_bias, best_ij, loss bits) all agree, and the max
    relative loss difference."""
    gc, gs, gl, gi = g[:4]
    oc, os_, ol, oi = o
    oc = oc[:, :(d + 1) // 2]
    same = (np.all(gc == oc, axis=1) & np.all(gs == os_, axis=1) & np.all(gi == oi, axis=1)
            & (gl.view(np.uint32) == ol.view(np.uint32)))
    with np.errstate(invalid="ignore"):  # inf - inf on rows whose loss overflows on both sides
        rel = np.abs(gl.astype(np.float64) - ol) / np.maximum(np.abs(ol.astype(np.float64)), 1e-300)
    rel[np.isnan(rel)] = 0
    rel[(gl == 0) & (ol == 0)] = 0
    return same, float(rel.max()) if rel.size else 0.0


def assert_quant_parity(x, mode=dq.DQ_MODE_GREEDY, **kw):
    g = gpu_quantize(x, mode, **kw)
    o = oracle.quantize_rows(x, mode=mode)
    same, rel = compare_quant(g, o, x.shape[1])
    bad = np.nonzero(~same)[0]
    assert bad.size == 0, (f"{bad.size}/{len(same)} rows differ; first {bad[:5]}; "
                           f"gpu ij {g[3][bad[:3]]} oracle ij {o[3][bad[:3]]} max rel loss {rel}")
    return g, o


def bag_tolerance_check(gpu_out, ref_out, abs_sum, rtol=1e-5):
    """|gpu - ref| <= rtol * sum_p |xhat| per element; returns the worst ratio."""
    err = np.abs(gpu_out.astype(np.float64) - ref_out.astype(np.float64))
    lim = rtol * abs_sum
    zero = abs_sum == 0
    assert np.all(gpu_out[zero] == 0)
    ratio = np.where(zero, 0.0, err / np.where(zero, 1.0, abs_sum))
    worst = float(ratio.max()) if ratio.size else 0.0
    assert np.all(err <= lim), f"bag error beyond {rtol} x sum|xhat|: worst ratio {worst}"
    return worst


def touched_masks(rows, batch, idx, off):
    """Per table, the rows that a bag backward over (idx, off) touches (valid ids only)."""
    masks = []
    for t, n in enumerate(rows):
        ids = idx[off[t * batch]:off[(t + 1) * batch]].astype(np.int64)
        m = np.zeros(n, bool)
        m[ids[(ids >= 0) & (ids < n)]] = True
        masks.append(m)
    return masks


def within_one_ulp(a, b):
    """Elementwise |a - b| <= one binary32 ulp of the larger magnitude."""
    big = np.maximum(np.abs(a), np.abs(b)).astype(np.float32)
    return np.abs(a.astype(np.float64) - b.astype(np.float64)) <= np.spacing(big).astype(np.float64)


def assert_bwd_parity(got, want, touched, d, mode=dq.DQ_MODE_GREEDY, n_touched=None):
    """The backward's parity criterion against the oracle (whose gradient is one plain
    binary64 sum per row in list order; the kernels sum the same binary64 values in
    64-entry pieces, which can move a binary32 rounding when a result lies within
    binary64 rounding error of a binary32 midpoint):
      - master rows bit-identical on at least 99.99 % of the touched rows (at most
        ceil(1e-4 * touched) rows differ), every element of the others within 1 ulp;
      - a row whose masters agree has the oracle's codes and scale/bias; a row whose
        masters differ has the oracle's quantization of the GPU's own master row;
      - untouched rows are never changed (the oracle leaves them as they were).
    got / want: per table (masters [n, ld], codes [n, cld], scale_bias uint16 [n, 2]).
    Returns (rows that differ, touched rows)."""
    cb = (d + 1) // 2
    differ = 0
    for t, ((gm, gc, gs), (om, oc, os_), tm) in enumerate(zip(got, want, touched)):
        same = np.all(gm.view(np.uint32) == om.view(np.uint32), axis=1)
        bad = np.nonzero(~same)[0]
        assert tm[bad].all(), f"table {t}: untouched rows changed: {bad[~tm[bad]][:5]}"
        assert np.array_equal(gm[bad, d:].view(np.uint32), om[bad, d:].view(np.uint32)), "padding changed"
        close = within_one_ulp(gm[bad, :d], om[bad, :d])
        assert close.all(), f"table {t}: master rows beyond 1 ulp: {bad[~np.all(close, axis=1)][:5]}"
        packed_same = np.all(gc == oc, axis=1) & np.all(gs == os_, axis=1)
        assert packed_same[same].all(), \
            f"table {t}: packed rows differ where masters agree: {np.nonzero(same & ~packed_same)[0][:5]}"
        if bad.size:
            c, sb, _, _ = oracle.quantize_rows(np.ascontiguousarray(gm[bad, :d]), mode=mode)
            assert np.array_equal(gc[bad, :cb], c[:, :cb]) and np.array_equal(gs[bad], sb), \
                f"table {t}: re-quantized rows are not the oracle's quantization of the GPU masters"
            assert np.array_equal(gc[bad, cb:], oc[bad, cb:]), "bytes past a code row changed"
        differ += bad.size
    if n_touched is None:
        n_touched = sum(int(m.sum()) for m in touched)
    assert differ <= math.ceil(1e-4 * n_touched), f"{differ} of {n_touched} touched rows differ"
    return differ, n_touched

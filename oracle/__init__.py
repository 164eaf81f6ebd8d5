"""CPU oracle for row-wise INT4 quantization and the INT4 embedding bag.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the bench's CPU
baseline are its only users. It is plain C (dq_oracle.c) behind ctypes and
shares nothing with the CUDA path; see dq_oracle.c for the definition it
implements and the reading taken of each step.

Parity of every function here is pinned by the `-m "not gpu"` tests against
closed forms, exact rational arithmetic, brute force on tiny rows and numpy's
binary16 conversion.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-pthread"]

GREEDY, MINMAX = 0, 1
MOVES = 168
N_EVALS = 1 + 2 * MOVES

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile dq_oracle.c into liboracle.so next to it (gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Table(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scale_bias", ctypes.c_void_p),
                ("n_rows", ctypes.c_int64), ("codes_ld", ctypes.c_int64), ("codebook", ctypes.c_void_p)]


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
            L.oracle_f32_to_f16.argtypes, L.oracle_f32_to_f16.restype = [f32], ctypes.c_uint16
            L.oracle_f16_to_f32.argtypes, L.oracle_f16_to_f32.restype = [ctypes.c_uint16], f32
            L.oracle_f32_to_f16_array.argtypes = [vp, vp, i64]
            L.oracle_f16_to_f32_array.argtypes = [vp, vp, i64]
            L.oracle_row_loss.argtypes, L.oracle_row_loss.restype = [vp, i32, f32, f32], f32
            L.oracle_greedy_trace.argtypes = [vp, i32, vp, vp, vp, vp, vp, vp]
            L.oracle_greedy_trace.restype = f32
            L.oracle_quantize_rows.argtypes = [vp, i64, i32, i64, vp, i64, vp, vp, vp, i32, i32]
            L.oracle_quantize_rows.restype = i32
            L.oracle_dequantize_rows.argtypes = [vp, i64, vp, i64, i32, vp, i64]
            L.oracle_dequantize_rows.restype = i32
            L.oracle_row_l2_error.argtypes = [vp, i64, i32, i64, vp, i64, vp, vp]
            L.oracle_row_l2_error.restype = ctypes.c_double
            L.oracle_embbag_bwd_sgd.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, vp, vp, i32, i64, vp,
                                                ctypes.c_float, i32, vp, i64]
            L.oracle_embbag_bwd_sgd.restype = i64
            L.oracle_embbag.argtypes = [vp, i32, i32, vp, vp, i32, vp, vp, i32]
            L.oracle_quantize_rows_kmeans.argtypes = [vp, i64, i32, i64, vp, i64, vp, vp, i32, i32]
            L.oracle_quantize_rows_kmeans.restype = i32
            L.oracle_dequantize_rows_kmeans.argtypes = [vp, i64, vp, i64, i32, vp, i64]
            L.oracle_dequantize_rows_kmeans.restype = i32
            L.oracle_kmeans_means.argtypes = [vp, vp, i32, vp]
            L.oracle_kmeans_means.restype = i32
            L.oracle_embbag.restype = i64
            _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def f32_to_f16_bits(v: float) -> int:
    return int(lib().oracle_f32_to_f16(float(v)))


def f16_bits_to_f32(h: int) -> float:
    return float(lib().oracle_f16_to_f32(int(h)))


def f32_to_f16_array(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint16)
    lib().oracle_f32_to_f16_array(_p(v), _p(out), v.size)
    return out


def f16_to_f32_array(h: np.ndarray) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, np.float32)
    lib().oracle_f16_to_f32_array(_p(h), _p(out), h.size)
    return out


def row_loss(x: np.ndarray, lo: float, hi: float) -> np.float32:
    x = np.ascontiguousarray(x, dtype=np.float32)
    return np.float32(lib().oracle_row_loss(_p(x), x.size, np.float32(lo), np.float32(hi)))


def greedy_trace(x: np.ndarray):
    """Every evaluation of one row's search: dict of lo, hi, loss [337], i, j [168], best, lbest."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    lo = np.zeros(N_EVALS, np.float32)
    hi = np.zeros(N_EVALS, np.float32)
    loss = np.zeros(N_EVALS, np.float32)
    ti = np.zeros(MOVES, np.int32)
    tj = np.zeros(MOVES, np.int32)
    best = np.zeros(2, np.int32)
    lb = lib().oracle_greedy_trace(_p(x), x.size, _p(lo), _p(hi), _p(loss), _p(ti), _p(tj), _p(best))
    return dict(lo=lo, hi=hi, loss=loss, i=ti, j=tj, best=(int(best[0]), int(best[1])),
                lbest=np.float32(lb))


def quantize_rows(x: np.ndarray, mode: int = GREEDY, nthreads: int = 0, codes_ld: int | None = None):
    """(codes uint8 [n, codes_ld], scale_bias uint16 [n, 2], loss float32 [n], best_ij uint8 [n, 2])."""
    x = np.asarray(x, dtype=np.float32)
    if x.ndim != 2 or x.strides[1] != 4:
        x = np.ascontiguousarray(x)
    n, d = x.shape
    ld = x.strides[0] // 4 if n > 1 else d
    cld = (d + 1) // 2 if codes_ld is None else codes_ld
    codes = np.zeros((n, cld), np.uint8)
    sb = np.zeros((n, 2), np.uint16)
    loss = np.zeros(n, np.float32)
    ij = np.zeros((n, 2), np.uint8)
    rc = lib().oracle_quantize_rows(_p(x), n, d, ld, _p(codes), cld, _p(sb), _p(loss), _p(ij),
                                    int(mode), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_quantize_rows: bad arguments")
    return codes, sb, loss, ij


def dequantize_rows(codes: np.ndarray, scale_bias: np.ndarray, d: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    sb = np.ascontiguousarray(scale_bias, dtype=np.uint16)
    n = codes.shape[0]
    out = np.zeros((n, d), np.float32)
    rc = lib().oracle_dequantize_rows(_p(codes), codes.shape[1], _p(sb), n, d, _p(out), d)
    if rc != 0:
        raise ValueError("oracle_dequantize_rows: bad arguments")
    return out


def row_l2_error(x: np.ndarray, codes: np.ndarray, scale_bias: np.ndarray):
    """(per-row normalized l2 error float64 [n], their sum float64)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    sb = np.ascontiguousarray(scale_bias, dtype=np.uint16)
    n, d = x.shape
    err = np.zeros(n, np.float64)
    tot = lib().oracle_row_l2_error(_p(x), n, d, d, _p(codes), codes.shape[1], _p(sb), _p(err))
    if np.isnan(tot):
        raise ValueError("oracle_row_l2_error: bad arguments")
    return err, float(tot)


def embbag(tables, d: int, indices: np.ndarray, offsets: np.ndarray, batch: int,
           with_abs_sum: bool = False, nthreads: int = 0, codebook: bool = False):
    """tables: list of (codes uint8 [n, ld], scale_bias uint16 [n, 2]), or with codebook=True
    list of (codes uint8 [n, ld], codebook uint16 [n, 16]).

    Returns (out float32 [batch, T*d], abs_sum float64 or None, skipped count)."""
    keep = []
    arr = (_Table * len(tables))()
    for t, (codes, sb) in enumerate(tables):
        codes = np.ascontiguousarray(codes, dtype=np.uint8)
        sb = np.ascontiguousarray(sb, dtype=np.uint16)
        keep += [codes, sb]
        if codebook:
            arr[t] = _Table(codes.ctypes.data, None, codes.shape[0], codes.shape[1], sb.ctypes.data)
        else:
            arr[t] = _Table(codes.ctypes.data, sb.ctypes.data, codes.shape[0], codes.shape[1], None)
    idx = np.ascontiguousarray(indices, dtype=np.int32)
    off = np.ascontiguousarray(offsets, dtype=np.int32)
    T = len(tables)
    out = np.zeros((batch, T * d), np.float32)
    mag = np.zeros((batch, T * d), np.float64) if with_abs_sum else None
    skipped = lib().oracle_embbag(ctypes.cast(arr, ctypes.c_void_p), T, d, _p(idx), _p(off), batch,
                                  _p(out), _p(mag) if mag is not None else None, int(nthreads))
    if skipped < 0:
        raise ValueError("oracle_embbag: bad arguments")
    return out, mag, int(skipped)


KMEANS_ITERS = 10


def quantize_rows_kmeans(x: np.ndarray, iters: int = KMEANS_ITERS, nthreads: int = 0, codes_ld: int | None = None):
    """Codebook (per-row k-means) quantization: (codes uint8 [n, codes_ld], codebook
    uint16 [n, 16] binary16 patterns, loss float32 [n])."""
    x = np.asarray(x, dtype=np.float32)
    if x.ndim != 2 or x.strides[1] != 4:
        x = np.ascontiguousarray(x)
    n, d = x.shape
    ld = x.strides[0] // 4 if n > 1 else d
    cld = (d + 1) // 2 if codes_ld is None else codes_ld
    codes = np.zeros((n, cld), np.uint8)
    cb = np.zeros((n, 16), np.uint16)
    loss = np.zeros(n, np.float32)
    rc = lib().oracle_quantize_rows_kmeans(_p(x), n, d, ld, _p(codes), cld, _p(cb), _p(loss), iters, nthreads)
    if rc != 0:
        raise ValueError("oracle_quantize_rows_kmeans: bad arguments")
    return codes, cb, loss


def kmeans_means(x: np.ndarray, a: np.ndarray, c: np.ndarray) -> np.ndarray:
    """One centroid update of the codebook quantizer: the new c[16] from the row x and
    its assignment a (clusters without members keep their c)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    a = np.ascontiguousarray(a, dtype=np.int32)
    out = np.array(c, dtype=np.float32, copy=True)
    if x.ndim != 1 or a.shape != x.shape or out.shape != (16,):
        raise ValueError("kmeans_means: x and a of one row, c of 16")
    if lib().oracle_kmeans_means(_p(x), _p(a), x.size, _p(out)) != 0:
        raise ValueError("oracle_kmeans_means: bad arguments")
    return out


def dequantize_rows_kmeans(codes: np.ndarray, codebook: np.ndarray, d: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    cb = np.ascontiguousarray(codebook, dtype=np.uint16)
    n = codes.shape[0]
    out = np.zeros((n, d), np.float32)
    if lib().oracle_dequantize_rows_kmeans(_p(codes), codes.shape[1], _p(cb), n, d, _p(out), d) != 0:
        raise ValueError("oracle_dequantize_rows_kmeans: bad arguments")
    return out


BAD_OFFSETS = -2


def embbag_bwd_sgd(masters, codes, scale_bias, d: int, indices: np.ndarray, offsets: np.ndarray,
                   batch: int, grad: np.ndarray, lr: float, mode: int = GREEDY, sample_keys=None) -> int:
    """Bag backward, SGD step on the binary32 masters and re-quantization of the touched
    rows, all in place. masters: list of float32 [n, ld]; codes: list of uint8 [n, cld];
    scale_bias: list of uint16 [n, 2]; grad: float32 [batch, T*d]. sample_keys (global
    keys = rows of the tables before t + id): update only those rows. Returns the number
    of invalid ids, or BAD_OFFSETS when the offsets are not a CSR array (nothing changed)."""
    T = len(masters)
    for w, c, sb in zip(masters, codes, scale_bias):
        assert w.dtype == np.float32 and w.flags["C_CONTIGUOUS"]
        assert c.dtype == np.uint8 and c.flags["C_CONTIGUOUS"] and c.shape[0] == w.shape[0]
        assert sb.dtype == np.uint16 and sb.flags["C_CONTIGUOUS"] and sb.shape == (w.shape[0], 2)

    def ptrs(arrs):
        return ctypes.cast((ctypes.c_void_p * T)(*[a.ctypes.data for a in arrs]), ctypes.c_void_p)

    wld = np.array([w.shape[1] for w in masters], np.int64)
    cld = np.array([c.shape[1] for c in codes], np.int64)
    nrows = np.array([w.shape[0] for w in masters], np.int64)
    idx = np.ascontiguousarray(indices, dtype=np.int32)
    off = np.ascontiguousarray(offsets, dtype=np.int32)
    g = np.ascontiguousarray(grad, dtype=np.float32)
    sk = None if sample_keys is None else np.ascontiguousarray(np.unique(sample_keys), dtype=np.uint32)
    r = lib().oracle_embbag_bwd_sgd(ptrs(masters), _p(wld), ptrs(codes), _p(cld), ptrs(scale_bias), _p(nrows),
                                    T, d, _p(idx), _p(off), batch, int(idx.size), _p(g), np.float32(lr), mode,
                                    None if sk is None else _p(sk), 0 if sk is None else int(sk.size))
    if r == -1:
        raise ValueError("oracle_embbag_bwd_sgd: bad arguments")
    return int(r)

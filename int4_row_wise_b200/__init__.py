"""int4_row_wise_b200 -- row-wise INT4 quantization of embedding tables and the
sum-pooled INT4 embedding bag, as CUDA kernels for B200 (sm_100a).

This module is a thin binding over libdq.so's C ABI (include/dq.h): it marshals
arguments (torch CUDA tensors -> device pointers, the current torch stream) and
turns status codes into exceptions. Every step of the computation runs in
libdq's kernels; there is no CPU path. If libdq.so is missing, the first call
raises DqError (build it with `python -m int4_row_wise_b200.build`).

Low-level calls with the C names:
    dq_quantize_rows_int4, dq_dequantize_rows, dq_embbag_int4_fwd, dq_row_l2_error,
    dq_embbag_int4_bwd_workspace_bytes, dq_embbag_int4_bwd_sgd, dq_embbag_int4_bwd_sgd_noalloc,
    dq_quantize_rows_kmeans4, dq_dequantize_rows_kmeans4, dq_embbag_kmeans4_fwd,
    dq_status_string, dq_last_error, dq_version
Convenience wrappers that allocate their outputs with torch:
    quantize_rows, dequantize_rows, embbag, row_l2_error, embbag_bwd_sgd,
    quantize_rows_kmeans, dequantize_rows_kmeans, embbag_kmeans
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import NamedTuple, Optional, Sequence

__all__ = [
    "DQ_OK", "DQ_ERR_INVALID_ARG", "DQ_ERR_UNSUPPORTED", "DQ_ERR_CUDA",
    "DQ_MODE_GREEDY", "DQ_MODE_MINMAX",
    "DQ_FLAG_BAD_INDEX", "DQ_FLAG_BAD_OFFSETS", "DQ_FLAG_NONFINITE", "DQ_FLAG_FP16_OVERFLOW",
    "DQ_MAX_D", "DQ_MAX_TABLES", "DqError", "PackedTable", "lib_path", "load",
    "dq_quantize_rows_int4", "dq_dequantize_rows", "dq_embbag_int4_fwd", "dq_embbag_int4_fwd_to_owners",
    "dq_row_l2_error",
    "dq_embbag_int4_bwd_workspace_bytes", "dq_embbag_int4_bwd_sgd", "MasterTable",
    "dq_embbag_int4_bwd_sgd_noalloc", "DQ_BWD_STATIC_SCRATCH_BYTES",
    "dq_quantize_rows_kmeans4", "dq_dequantize_rows_kmeans4", "dq_embbag_kmeans4_fwd", "KmeansTable",
    "DQ_KMEANS_MAX_ITERS", "KMEANS_ITERS", "quantize_rows_kmeans", "dequantize_rows_kmeans", "embbag_kmeans",
    "dq_status_string", "dq_last_error", "dq_version",
    "quantize_rows", "dequantize_rows", "embbag", "row_l2_error", "embbag_bwd_sgd",
]

DQ_OK, DQ_ERR_INVALID_ARG, DQ_ERR_UNSUPPORTED, DQ_ERR_CUDA = 0, 1, 2, 3
DQ_MODE_GREEDY, DQ_MODE_MINMAX = 0, 1
DQ_FLAG_BAD_INDEX, DQ_FLAG_BAD_OFFSETS, DQ_FLAG_NONFINITE, DQ_FLAG_FP16_OVERFLOW = 1, 2, 4, 8
DQ_MAX_D, DQ_MAX_TABLES = 1024, 64
DQ_BWD_STATIC_SCRATCH_BYTES = 32 << 20
DQ_KMEANS_MAX_ITERS = 64
KMEANS_ITERS = 10  # Lloyd iterations of the convenience wrapper

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libdq.so")
_lock = threading.Lock()
_lib = None


class DqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


class _Table(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scale_bias", ctypes.c_void_p),
                ("n_rows", ctypes.c_int64), ("codes_ld", ctypes.c_int64)]


class _MasterTable(ctypes.Structure):
    _fields_ = [("master", ctypes.c_void_p), ("master_ld", ctypes.c_int64), ("codes", ctypes.c_void_p),
                ("codes_ld", ctypes.c_int64), ("scale_bias", ctypes.c_void_p), ("n_rows", ctypes.c_int64)]


def lib_path() -> str:
    return _LIB_PATH


def load():
    """The loaded libdq (ctypes.CDLL); raises DqError if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise DqError(DQ_ERR_UNSUPPORTED,
                              f"libdq.so not found at {_LIB_PATH}; build it with "
                              "`python -m int4_row_wise_b200.build`")
            L = ctypes.CDLL(_LIB_PATH)
            vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
            L.dq_quantize_rows_int4.argtypes = [vp, i64, i32, i64, vp, i64, vp, vp, vp, i32, vp, vp]
            L.dq_quantize_rows_int4.restype = ctypes.c_int
            L.dq_dequantize_rows.argtypes = [vp, i64, vp, i64, i32, vp, i64, vp]
            L.dq_dequantize_rows.restype = ctypes.c_int
            L.dq_embbag_int4_fwd.argtypes = [vp, i32, i32, vp, vp, i32, vp, vp, vp]
            L.dq_embbag_int4_fwd.restype = ctypes.c_int
            L.dq_embbag_int4_fwd_to_owners.argtypes = [vp, i32, i32, vp, vp, i32, vp, i32, vp, i32, vp, vp]
            L.dq_embbag_int4_fwd_to_owners.restype = ctypes.c_int
            L.dq_row_l2_error.argtypes = [vp, i64, i32, i64, vp, i64, vp, vp, vp, vp]
            L.dq_row_l2_error.restype = ctypes.c_int
            L.dq_embbag_int4_bwd_workspace_bytes.argtypes = [i32, i64]
            L.dq_embbag_int4_bwd_workspace_bytes.restype = ctypes.c_size_t
            L.dq_embbag_int4_bwd_sgd.argtypes = [vp, i32, i32, vp, vp, i32, i64, vp, ctypes.c_float, i32, vp,
                                                 ctypes.c_size_t, vp, vp]
            L.dq_embbag_int4_bwd_sgd.restype = ctypes.c_int
            L.dq_embbag_int4_bwd_sgd_noalloc.argtypes = [vp, i32, i32, vp, vp, i32, i64, vp, ctypes.c_float, i32,
                                                         vp, vp]
            L.dq_embbag_int4_bwd_sgd_noalloc.restype = ctypes.c_int
            L.dq_quantize_rows_kmeans4.argtypes = [vp, i64, i32, i64, vp, i64, vp, vp, vp, i32, vp, vp]
            L.dq_quantize_rows_kmeans4.restype = ctypes.c_int
            L.dq_dequantize_rows_kmeans4.argtypes = [vp, i64, vp, i64, i32, vp, i64, vp]
            L.dq_dequantize_rows_kmeans4.restype = ctypes.c_int
            L.dq_embbag_kmeans4_fwd.argtypes = [vp, i32, i32, vp, vp, i32, vp, vp, vp]
            L.dq_embbag_kmeans4_fwd.restype = ctypes.c_int
            L.dq_status_string.argtypes, L.dq_status_string.restype = [ctypes.c_int], ctypes.c_char_p
            L.dq_last_error.argtypes, L.dq_last_error.restype = [], ctypes.c_char_p
            L.dq_version.argtypes, L.dq_version.restype = [], i32
            _lib = L
    return _lib


def _ptr(a) -> Optional[int]:
    """Device address of a CUDA tensor; ints pass through; None stays NULL."""
    if a is None:
        return None
    if isinstance(a, int):
        return a
    if not a.is_cuda:
        raise DqError(DQ_ERR_INVALID_ARG, "libdq takes CUDA tensors (device pointers)")
    return a.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, what: str) -> None:
    if status != DQ_OK:
        L = load()
        raise DqError(status, f"{what}: {L.dq_status_string(status).decode()}: {L.dq_last_error().decode()}")


def dq_status_string(status: int) -> str:
    return load().dq_status_string(status).decode()


def dq_last_error() -> str:
    return load().dq_last_error().decode()


def dq_version() -> int:
    return int(load().dq_version())


def dq_quantize_rows_int4(x, n_rows: int, d: int, x_ld: int, codes, codes_ld: int, scale_bias,
                          row_loss=None, best_ij=None, mode: int = DQ_MODE_GREEDY, d_flags=None,
                          stream=None) -> None:
    """C: dq_quantize_rows_int4. Tensors (or raw device addresses) for every buffer."""
    st = load().dq_quantize_rows_int4(_ptr(x), n_rows, d, x_ld, _ptr(codes), codes_ld, _ptr(scale_bias),
                                      _ptr(row_loss), _ptr(best_ij), mode, _ptr(d_flags), _stream(stream))
    _check(st, "dq_quantize_rows_int4")


def dq_dequantize_rows(codes, codes_ld: int, scale_bias, n_rows: int, d: int, out, out_ld: int,
                       stream=None) -> None:
    """C: dq_dequantize_rows."""
    st = load().dq_dequantize_rows(_ptr(codes), codes_ld, _ptr(scale_bias), n_rows, d, _ptr(out), out_ld,
                                   _stream(stream))
    _check(st, "dq_dequantize_rows")


def dq_row_l2_error(x, n_rows: int, d: int, x_ld: int, codes, codes_ld: int, scale_bias, row_err=None,
                    err_sum=None, stream=None) -> None:
    """C: dq_row_l2_error (err_sum is accumulated into)."""
    st = load().dq_row_l2_error(_ptr(x), n_rows, d, x_ld, _ptr(codes), codes_ld, _ptr(scale_bias),
                                _ptr(row_err), _ptr(err_sum), _stream(stream))
    _check(st, "dq_row_l2_error")


class PackedTable(NamedTuple):
    """A packed INT4 table on the device: codes uint8 [n, codes_ld], scale_bias int16 [n, 2]
    (binary16 bit patterns)."""
    codes: object
    scale_bias: object

    @property
    def n_rows(self) -> int:
        return int(self.codes.shape[0])


def _table_array(tables: Sequence):
    """The dq_table array of PackedTable (or (codes, scale_bias)) entries."""
    arr = (_Table * max(len(tables), 1))()
    for t, tab in enumerate(tables):
        codes, sb = tab[0], tab[1]
        if codes.dim() != 2:
            raise DqError(DQ_ERR_INVALID_ARG, "table codes must be a [n_rows, codes_ld] tensor")
        # a table of 0 or 1 rows has no meaningful row stride: its row width is the stride
        ld = int(codes.stride(0)) if codes.shape[0] > 1 else int(codes.shape[1])
        arr[t] = _Table(_ptr(codes), _ptr(sb), int(codes.shape[0]), ld)
    return arr


def dq_embbag_int4_fwd(tables: Sequence, d: int, indices, offsets, batch: int, out, d_flags=None,
                       stream=None) -> None:
    """C: dq_embbag_int4_fwd. tables: PackedTable (or (codes, scale_bias)) per table."""
    arr = _table_array(tables)
    st = load().dq_embbag_int4_fwd(ctypes.cast(arr, ctypes.c_void_p), len(tables), d, _ptr(indices),
                                   _ptr(offsets), batch, _ptr(out), _ptr(d_flags), _stream(stream))
    _check(st, "dq_embbag_int4_fwd")


def dq_embbag_int4_fwd_to_owners(tables: Sequence, d: int, indices, offsets, batch: int, table_slot: Sequence[int],
                                 t_out: int, dest: Sequence, d_flags=None, stream=None) -> None:
    """C: dq_embbag_int4_fwd_to_owners. dest: one device buffer (tensor or address) per
    rank, [batch // len(dest), t_out * d] binary32; table_slot: the column block of each
    local table."""
    arr = _table_array(tables)
    slots = (ctypes.c_int32 * max(len(tables), 1))(*[int(v) for v in table_slot])
    ptrs = (ctypes.c_void_p * max(len(dest), 1))(*[_ptr(x) for x in dest])
    st = load().dq_embbag_int4_fwd_to_owners(ctypes.cast(arr, ctypes.c_void_p), len(tables), d, _ptr(indices),
                                             _ptr(offsets), batch, ctypes.cast(slots, ctypes.c_void_p), t_out,
                                             ctypes.cast(ptrs, ctypes.c_void_p), len(dest), _ptr(d_flags),
                                             _stream(stream))
    _check(st, "dq_embbag_int4_fwd_to_owners")


class MasterTable(NamedTuple):
    """A trained table on the device: binary32 masters [n, master_ld] and their packed
    form (codes uint8 [n, codes_ld], scale_bias int16 [n, 2])."""
    master: object
    codes: object
    scale_bias: object


def dq_embbag_int4_bwd_workspace_bytes(d: int, n_indices: int) -> int:
    """C: dq_embbag_int4_bwd_workspace_bytes."""
    return int(load().dq_embbag_int4_bwd_workspace_bytes(d, n_indices))


def _row_stride(t) -> int:
    return int(t.stride(0)) if t.shape[0] > 1 else int(t.shape[1])


def dq_embbag_int4_bwd_sgd(tables: Sequence, d: int, indices, offsets, batch: int, n_indices: int, grad_out,
                           lr: float, mode: int, workspace, workspace_bytes: int, d_flags=None,
                           stream=None) -> None:
    """C: dq_embbag_int4_bwd_sgd. tables: MasterTable (or (master, codes, scale_bias)) per table."""
    arr = (_MasterTable * max(len(tables), 1))()
    for t, tab in enumerate(tables):
        master, codes, sb = tab[0], tab[1], tab[2]
        if master.dim() != 2 or codes.dim() != 2:
            raise DqError(DQ_ERR_INVALID_ARG, "master and codes must be 2-d tensors")
        arr[t] = _MasterTable(_ptr(master), _row_stride(master), _ptr(codes), _row_stride(codes), _ptr(sb),
                              int(master.shape[0]))
    st = load().dq_embbag_int4_bwd_sgd(ctypes.cast(arr, ctypes.c_void_p), len(tables), d, _ptr(indices),
                                       _ptr(offsets), batch, n_indices, _ptr(grad_out), float(lr), mode,
                                       _ptr(workspace), workspace_bytes, _ptr(d_flags), _stream(stream))
    _check(st, "dq_embbag_int4_bwd_sgd")


class _KmeansTable(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("codebook", ctypes.c_void_p),
                ("n_rows", ctypes.c_int64), ("codes_ld", ctypes.c_int64)]


class KmeansTable(NamedTuple):
    """A codebook-quantized table on the device: codes uint8 [n, codes_ld], codebook int16
    [n, 16] (binary16 bit patterns)."""
    codes: object
    codebook: object


def dq_quantize_rows_kmeans4(x, n_rows: int, d: int, x_ld: int, codes, codes_ld: int, codebook, row_loss=None,
                             iters: int = KMEANS_ITERS, d_flags=None, stream=None, row_iters=None) -> None:
    """C: dq_quantize_rows_kmeans4 (row_iters: optional int32 [n_rows] device tensor)."""
    st = load().dq_quantize_rows_kmeans4(_ptr(x), n_rows, d, x_ld, _ptr(codes), codes_ld, _ptr(codebook),
                                         _ptr(row_loss), _ptr(row_iters), iters, _ptr(d_flags), _stream(stream))
    _check(st, "dq_quantize_rows_kmeans4")


def dq_dequantize_rows_kmeans4(codes, codes_ld: int, codebook, n_rows: int, d: int, out, out_ld: int,
                               stream=None) -> None:
    """C: dq_dequantize_rows_kmeans4."""
    st = load().dq_dequantize_rows_kmeans4(_ptr(codes), codes_ld, _ptr(codebook), n_rows, d, _ptr(out), out_ld,
                                           _stream(stream))
    _check(st, "dq_dequantize_rows_kmeans4")


def dq_embbag_kmeans4_fwd(tables: Sequence, d: int, indices, offsets, batch: int, out, d_flags=None,
                          stream=None) -> None:
    """C: dq_embbag_kmeans4_fwd. tables: KmeansTable (or (codes, codebook)) per table."""
    arr = (_KmeansTable * max(len(tables), 1))()
    for t, tab in enumerate(tables):
        codes, cb = tab[0], tab[1]
        if codes.dim() != 2:
            raise DqError(DQ_ERR_INVALID_ARG, "table codes must be a [n_rows, codes_ld] tensor")
        arr[t] = _KmeansTable(_ptr(codes), _ptr(cb), int(codes.shape[0]), _row_stride(codes))
    st = load().dq_embbag_kmeans4_fwd(ctypes.cast(arr, ctypes.c_void_p), len(tables), d, _ptr(indices),
                                      _ptr(offsets), batch, _ptr(out), _ptr(d_flags), _stream(stream))
    _check(st, "dq_embbag_kmeans4_fwd")


def _master_array(tables):
    arr = (_MasterTable * max(len(tables), 1))()
    for t, tab in enumerate(tables):
        master, codes, sb = tab[0], tab[1], tab[2]
        if master.dim() != 2 or codes.dim() != 2:
            raise DqError(DQ_ERR_INVALID_ARG, "master and codes must be 2-d tensors")
        arr[t] = _MasterTable(_ptr(master), _row_stride(master), _ptr(codes), _row_stride(codes), _ptr(sb),
                              int(master.shape[0]))
    return arr


def dq_embbag_int4_bwd_sgd_noalloc(tables: Sequence, d: int, indices, offsets, batch: int, n_indices: int,
                                   grad_out, lr: float, mode: int, d_flags=None, stream=None) -> None:
    """C: dq_embbag_int4_bwd_sgd_noalloc -- the backward on the library's static device
    scratch (DQ_BWD_STATIC_SCRATCH_BYTES), for callers that cannot allocate device
    memory. Calls that overlap on the GPU race on that scratch."""
    arr = _master_array(tables)
    st = load().dq_embbag_int4_bwd_sgd_noalloc(ctypes.cast(arr, ctypes.c_void_p), len(tables), d, _ptr(indices),
                                               _ptr(offsets), batch, n_indices, _ptr(grad_out), float(lr), mode,
                                               _ptr(d_flags), _stream(stream))
    _check(st, "dq_embbag_int4_bwd_sgd_noalloc")


# -------------------------------------------------------------------------
# convenience wrappers (torch allocates the outputs on the input's device)
# -------------------------------------------------------------------------

def _codes_ld(d: int) -> int:
    cb = (d + 1) // 2
    return cb if cb < 16 else (cb + 15) // 16 * 16


def quantize_rows(x, mode: int = DQ_MODE_GREEDY, with_loss: bool = True, d_flags=None, stream=None):
    """x: CUDA float32 [n, d] (unit stride along d). Returns (codes uint8 [n, codes_ld],
    scale_bias int16 [n, 2], row_loss float32 [n] or None, best_ij uint8 [n, 2] or None)."""
    import torch
    if x.dim() != 2 or x.dtype != torch.float32 or (x.shape[0] > 1 and x.stride(1) != 1):
        raise DqError(DQ_ERR_INVALID_ARG, "x must be a float32 [n, d] tensor with unit stride along d")
    n, d = x.shape
    cld = _codes_ld(d)
    codes = torch.empty((n, cld), dtype=torch.uint8, device=x.device)
    sb = torch.empty((n, 2), dtype=torch.int16, device=x.device)
    loss = torch.empty(n, dtype=torch.float32, device=x.device) if with_loss else None
    ij = torch.empty((n, 2), dtype=torch.uint8, device=x.device) if with_loss else None
    ld = x.stride(0) if n > 1 else d
    dq_quantize_rows_int4(x, n, d, ld, codes, cld, sb, loss, ij, mode, d_flags, stream)
    return codes, sb, loss, ij


def dequantize_rows(codes, scale_bias, d: int, stream=None):
    import torch
    n = codes.shape[0]
    out = torch.empty((n, d), dtype=torch.float32, device=codes.device)
    dq_dequantize_rows(codes, codes.stride(0) if n > 1 else codes.shape[1], scale_bias, n, d, out, d, stream)
    return out


def embbag(tables: Sequence, d: int, indices, offsets, batch: int, d_flags=None, stream=None):
    """Sum-pooled lookup; returns float32 [batch, len(tables) * d]."""
    import torch
    out = torch.empty((batch, len(tables) * d), dtype=torch.float32, device=indices.device)
    dq_embbag_int4_fwd(tables, d, indices, offsets, batch, out, d_flags, stream)
    return out


def row_l2_error(x, codes, scale_bias, stream=None):
    """Normalized l2 error of each row of x against its packed form: (float64 [n], mean)."""
    import torch
    n, d = x.shape
    err = torch.empty(n, dtype=torch.float64, device=x.device)
    tot = torch.zeros(1, dtype=torch.float64, device=x.device)
    dq_row_l2_error(x, n, d, x.stride(0) if n > 1 else d, codes, codes.stride(0) if n > 1 else codes.shape[1],
                    scale_bias, err, tot, stream)
    return err, tot / max(n, 1)


def embbag_bwd_sgd(tables: Sequence, d: int, indices, offsets, batch: int, grad_out, lr: float,
                   mode: int = DQ_MODE_GREEDY, workspace=None, d_flags=None, stream=None):
    """Backward of the lookup + SGD step on the masters + re-quantization of the touched
    rows, in place. Allocates the workspace with torch unless one (uint8 CUDA tensor,
    256-byte aligned) is given; returns it for reuse."""
    import torch
    n = int(indices.numel())
    need = dq_embbag_int4_bwd_workspace_bytes(d, n)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=indices.device)
    dq_embbag_int4_bwd_sgd(tables, d, indices, offsets, batch, n, grad_out, lr, mode, workspace,
                           int(workspace.numel()), d_flags, stream)
    return workspace


def quantize_rows_kmeans(x, iters: int = KMEANS_ITERS, with_loss: bool = True, d_flags=None, stream=None):
    """Codebook quantization of x (CUDA float32 [n, d], unit stride along d). Returns
    (codes uint8 [n, codes_ld], codebook int16 [n, 16], row_loss float32 [n] or None)."""
    import torch
    if x.dim() != 2 or x.dtype != torch.float32 or (x.shape[0] > 1 and x.stride(1) != 1):
        raise DqError(DQ_ERR_INVALID_ARG, "x must be a float32 [n, d] tensor with unit stride along d")
    n, d = x.shape
    cld = _codes_ld(d)
    codes = torch.empty((n, cld), dtype=torch.uint8, device=x.device)
    cb = torch.empty((n, 16), dtype=torch.int16, device=x.device)
    loss = torch.empty(n, dtype=torch.float32, device=x.device) if with_loss else None
    dq_quantize_rows_kmeans4(x, n, d, x.stride(0) if n > 1 else d, codes, cld, cb, loss, iters, d_flags, stream)
    return codes, cb, loss


def dequantize_rows_kmeans(codes, codebook, d: int, stream=None):
    import torch
    n = codes.shape[0]
    out = torch.empty((n, d), dtype=torch.float32, device=codes.device)
    dq_dequantize_rows_kmeans4(codes, _row_stride(codes) if n else codes.shape[1], codebook, n, d, out, d, stream)
    return out


def embbag_kmeans(tables: Sequence, d: int, indices, offsets, batch: int, d_flags=None, stream=None):
    """Sum-pooled lookup over codebook tables; returns float32 [batch, len(tables) * d]."""
    import torch
    out = torch.empty((batch, len(tables) * d), dtype=torch.float32, device=indices.device)
    dq_embbag_kmeans4_fwd(tables, d, indices, offsets, batch, out, d_flags, stream)
    return out

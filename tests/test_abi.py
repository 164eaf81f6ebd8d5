"""The C-ABI boundary without a GPU: libdq.so loads, exports every function
include/dq.h declares, and rejects bad arguments on the host before touching
the device (no compute call is made here)."""
import ctypes
import os
import re

import pytest

import int4_row_wise_b200 as dq
from int4_row_wise_b200 import build as dqbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    dqbuild.build()
    return dq.load()


def _declared():
    src = open(os.path.join(ROOT, "include", "dq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dq_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = _declared()
    assert {"dq_quantize_rows_int4", "dq_dequantize_rows", "dq_embbag_int4_fwd",
            "dq_status_string"} <= set(names)
    for n in names:
        assert hasattr(L, n), n
    out = os.popen(f"nm -D --defined-only {dq.lib_path()}").read()
    exported = set(re.findall(r"\bT (dq_[a-z0-9_]+)$", out, flags=re.M))
    assert set(names) <= exported


def test_status_strings_and_version(L):
    assert dq.dq_status_string(dq.DQ_OK) == "DQ_OK"
    assert "INVALID" in dq.dq_status_string(dq.DQ_ERR_INVALID_ARG)
    assert "CUDA" in dq.dq_status_string(dq.DQ_ERR_CUDA)
    assert dq.dq_version() == 10000


NULL = None


@pytest.mark.parametrize("args,msg", [
    ((NULL, -1, 16, 16, NULL, 8, NULL, NULL, NULL, 0, NULL, NULL), "n_rows"),
    ((NULL, 4, 0, 16, NULL, 8, NULL, NULL, NULL, 0, NULL, NULL), "d = 0"),
    ((NULL, 4, 1025, 1025, NULL, 513, NULL, NULL, NULL, 0, NULL, NULL), "d = 1025"),
    ((NULL, 4, 16, 15, NULL, 8, NULL, NULL, NULL, 0, NULL, NULL), "x_ld"),
    ((NULL, 4, 16, 16, NULL, 7, NULL, NULL, NULL, 0, NULL, NULL), "codes_ld"),
    ((NULL, 4, 16, 16, NULL, 8, NULL, NULL, NULL, 2, NULL, NULL), "mode"),
    ((NULL, 4, 16, 16, NULL, 8, NULL, NULL, NULL, 0, NULL, NULL), "non-NULL"),
])
def test_quantize_rejects(L, args, msg):
    assert L.dq_quantize_rows_int4(*args) == dq.DQ_ERR_INVALID_ARG
    assert msg in L.dq_last_error().decode()


def test_zero_rows_is_a_noop(L):
    assert L.dq_quantize_rows_int4(NULL, 0, 16, 16, NULL, 8, NULL, NULL, NULL, 0, NULL, NULL) == dq.DQ_OK
    assert L.dq_dequantize_rows(NULL, 8, NULL, 0, 16, NULL, 16, NULL) == dq.DQ_OK
    t = (dq._Table * 1)(dq._Table(None, None, 0, 8))
    assert L.dq_embbag_int4_fwd(ctypes.cast(t, ctypes.c_void_p), 1, 16, NULL, NULL, 0, NULL, NULL, NULL) == dq.DQ_OK


@pytest.mark.parametrize("args,msg", [
    ((NULL, 8, NULL, -1, 16, NULL, 16, NULL), "n_rows"),
    ((NULL, 7, NULL, 3, 16, NULL, 16, NULL), "codes_ld"),
    ((NULL, 8, NULL, 3, 16, NULL, 15, NULL), "out_ld"),
    ((NULL, 8, NULL, 3, 2000, NULL, 2000, NULL), "d = 2000"),
    ((NULL, 8, NULL, 3, 16, NULL, 16, NULL), "non-NULL"),
])
def test_dequantize_rejects(L, args, msg):
    assert L.dq_dequantize_rows(*args) == dq.DQ_ERR_INVALID_ARG
    assert msg in L.dq_last_error().decode()


def _tables(*specs):
    arr = (dq._Table * max(len(specs), 1))(*[dq._Table(*s) for s in specs])
    return ctypes.cast(arr, ctypes.c_void_p), arr


@pytest.mark.parametrize("tabspec,T,d,batch,msg", [
    ([(None, None, 10, 8)], 0, 16, 4, "n_tables = 0"),
    ([(None, None, 10, 8)], 65, 16, 4, "n_tables = 65"),
    ([(None, None, 10, 8)], 1, 16, -1, "batch"),
    ([(None, None, -1, 8)], 1, 16, 4, "n_rows"),
    ([(None, None, 10, 7)], 1, 16, 4, "codes_ld"),
    ([(None, None, 10, 8)], 1, 16, 4, "non-NULL"),
    ([(1 << 20, 1 << 21, 10, 8)], 1, 16, 4, "indices"),
    ([(1 << 20, 1 << 21, 10, 8)], 1, 0, 4, "d = 0"),
])
def test_embbag_rejects(L, tabspec, T, d, batch, msg):
    p, keep = _tables(*tabspec)
    assert L.dq_embbag_int4_fwd(p, T, d, None, None, batch, None, None, None) == dq.DQ_ERR_INVALID_ARG
    assert msg in L.dq_last_error().decode()


@pytest.mark.parametrize("batch,slots,t_out,n_dest,msg", [
    (6, [0], 1, 4, "not a multiple"),
    (4, [0], 1, 0, "n_dest = 0"),
    (4, [0], 1, 65, "n_dest = 65"),
    (4, [1], 1, 2, "table_slot[0] = 1"),
    (4, [-1], 3, 2, "table_slot[0] = -1"),
    (4, [0, 0], 3, 2, "both 0"),
    (4, [0, 1], 1, 2, "t_out = 1"),
])
def test_embbag_to_owners_rejects(L, batch, slots, t_out, n_dest, msg):
    """The placement checks come before anything touches a GPU."""
    T = len(slots)
    p, keep = _tables(*[(1 << 20, 1 << 21, 10, 8)] * T)
    sl = (ctypes.c_int32 * T)(*slots)
    dest = (ctypes.c_void_p * max(n_dest, 1))(*([1 << 24] * max(n_dest, 1)))
    st = L.dq_embbag_int4_fwd_to_owners(p, T, 16, 1 << 22, 1 << 23, batch, ctypes.cast(sl, ctypes.c_void_p), t_out,
                                        ctypes.cast(dest, ctypes.c_void_p), n_dest, None, None)
    assert st == dq.DQ_ERR_INVALID_ARG
    assert msg in L.dq_last_error().decode()


def test_binding_raises_with_status(L):
    with pytest.raises(dq.DqError) as ei:
        dq.dq_quantize_rows_int4(None, 4, 0, 16, None, 8, None, stream=0)
    assert ei.value.status == dq.DQ_ERR_INVALID_ARG and "d = 0" in str(ei.value)


def test_library_sources_allocate_nothing():
    # the library allocates no device or host memory of its own
    import glob
    for path in glob.glob(os.path.join(ROOT, "int4_row_wise_b200", "csrc", "*")):
        src = open(path).read()
        for call in ("cudaMalloc", "cudaFree", "cudaHostAlloc", "cudaMallocHost", "malloc(", "new "):
            assert call not in src, (path, call)


def _masters(*specs):
    arr = (dq._MasterTable * max(len(specs), 1))(*[dq._MasterTable(*s) for s in specs])
    return ctypes.cast(arr, ctypes.c_void_p), arr


_M, _C, _S = 1 << 20, 1 << 22, 1 << 24  # placeholder device addresses (never dereferenced)


@pytest.mark.parametrize("tabspec,T,d,batch,n,lr,mode,ws,wsb,msg", [
    ([(_M, 16, _C, 8, _S, 10)], 0, 16, 4, 8, 0.1, 0, 1 << 26, 1 << 30, "n_tables = 0"),
    ([(_M, 16, _C, 8, _S, 10)], 1, 0, 4, 8, 0.1, 0, 1 << 26, 1 << 30, "d = 0"),
    ([(_M, 16, _C, 8, _S, 10)], 1, 16, -1, 8, 0.1, 0, 1 << 26, 1 << 30, "batch"),
    ([(_M, 16, _C, 8, _S, 10)], 1, 16, 4, -1, 0.1, 0, 1 << 26, 1 << 30, "n_indices"),
    ([(_M, 16, _C, 8, _S, 10)], 1, 16, 0, 3, 0.1, 0, 1 << 26, 1 << 30, "batch = 0"),
    ([(_M, 16, _C, 8, _S, 10)], 1, 16, 4, 8, 0.1, 5, 1 << 26, 1 << 30, "mode"),
    ([(_M, 16, _C, 8, _S, 10)], 1, 16, 4, 8, float("inf"), 0, 1 << 26, 1 << 30, "lr"),
    ([(_M, 15, _C, 8, _S, 10)], 1, 16, 4, 8, 0.1, 0, 1 << 26, 1 << 30, "master_ld"),
    ([(_M, 16, _C, 7, _S, 10)], 1, 16, 4, 8, 0.1, 0, 1 << 26, 1 << 30, "codes_ld"),
    ([(_M, 16, _C, 8, _S, -2)], 1, 16, 4, 8, 0.1, 0, 1 << 26, 1 << 30, "n_rows"),
    ([(None, 16, _C, 8, _S, 10)], 1, 16, 4, 8, 0.1, 0, 1 << 26, 1 << 30, "non-NULL"),
    ([(_M + 2, 16, _C, 8, _S, 10)], 1, 16, 4, 8, 0.1, 0, 1 << 26, 1 << 30, "aligned"),
    ([(_M, 16, _C, 8, _S, 1 << 31), (_M, 16, _C, 8, _S, 1 << 31)], 2, 16, 4, 8, 0.1, 0, 1 << 26, 1 << 30,
     "2^32 - 2"),
    ([(_M, 16, _C, 8, _S, 10)], 1, 16, 4, 8, 0.1, 0, (1 << 26) + 16, 1 << 30, "256-byte"),
    ([(_M, 16, _C, 8, _S, 10)], 1, 16, 4, 8, 0.1, 0, 1 << 26, 100, "workspace_bytes"),
])
def test_embbag_bwd_rejects(L, tabspec, T, d, batch, n, lr, mode, ws, wsb, msg):
    p, keep = _masters(*tabspec)
    idx, off, g = 1 << 27, 1 << 28, 1 << 29
    st = L.dq_embbag_int4_bwd_sgd(p, T, d, idx, off, batch, n, g, lr, mode, ws, wsb, None, None)
    assert st == dq.DQ_ERR_INVALID_ARG
    assert msg in L.dq_last_error().decode()


def test_embbag_bwd_no_entries_is_a_noop_and_workspace_size(L):
    p, keep = _masters((_M, 16, _C, 8, _S, 10))
    assert L.dq_embbag_int4_bwd_sgd(p, 1, 16, None, None, 4, 0, None, 0.1, 0, None, 0, None, None) == dq.DQ_OK
    assert dq.dq_embbag_int4_bwd_workspace_bytes(16, -1) == 0
    assert dq.dq_embbag_int4_bwd_workspace_bytes(0, 10) == 0
    small, big = dq.dq_embbag_int4_bwd_workspace_bytes(64, 1000), dq.dq_embbag_int4_bwd_workspace_bytes(64, 10 ** 6)
    assert small % 256 == 0 and big % 256 == 0
    # keys, bags (twice each), list: 20 B; G rows: 4 d B; window parts: d / 4 B per entry
    assert 10 ** 6 * (20 + 4 * 64 + 64 // 4) <= big <= 10 ** 6 * (20 + 4 * 64 + 64 // 4) + 10 ** 6


@pytest.mark.parametrize("args,msg", [
    ((NULL, -1, 16, 16, NULL, 8, NULL, NULL, NULL, 10, NULL, NULL), "n_rows"),
    ((NULL, 4, 0, 16, NULL, 8, NULL, NULL, NULL, 10, NULL, NULL), "d = 0"),
    ((NULL, 4, 16, 15, NULL, 8, NULL, NULL, NULL, 10, NULL, NULL), "x_ld"),
    ((NULL, 4, 16, 16, NULL, 7, NULL, NULL, NULL, 10, NULL, NULL), "codes_ld"),
    ((NULL, 4, 16, 16, NULL, 8, NULL, NULL, NULL, 65, NULL, NULL), "iters"),
    ((NULL, 4, 16, 16, NULL, 8, NULL, NULL, NULL, -1, NULL, NULL), "iters"),
    ((NULL, 4, 16, 16, NULL, 8, NULL, NULL, NULL, 10, NULL, NULL), "non-NULL"),
])
def test_kmeans_quantize_rejects(L, args, msg):
    assert L.dq_quantize_rows_kmeans4(*args) == dq.DQ_ERR_INVALID_ARG
    assert msg in L.dq_last_error().decode()


def test_kmeans_dequantize_and_bag_reject(L):
    assert L.dq_dequantize_rows_kmeans4(None, 8, None, 3, 16, None, 15, None) == dq.DQ_ERR_INVALID_ARG
    assert "out_ld" in L.dq_last_error().decode()
    arr = (dq._KmeansTable * 1)(dq._KmeansTable(None, None, 10, 8))
    p = ctypes.cast(arr, ctypes.c_void_p)
    assert L.dq_embbag_kmeans4_fwd(p, 1, 16, None, None, 4, None, None, None) == dq.DQ_ERR_INVALID_ARG
    assert "codebook" in L.dq_last_error().decode()
    assert L.dq_embbag_kmeans4_fwd(p, 1, 16, None, None, 0, None, None, None) == dq.DQ_ERR_INVALID_ARG
    arr0 = (dq._KmeansTable * 1)(dq._KmeansTable(None, None, 0, 8))
    assert L.dq_embbag_kmeans4_fwd(ctypes.cast(arr0, ctypes.c_void_p), 1, 16, None, None, 0, None, None,
                                   None) == dq.DQ_OK


def test_misaligned_arrays_are_rejected_before_any_launch(L):
    """Typed arrays the kernels read element-wise must be aligned to their element size."""
    A = 1 << 24   # stand-in device addresses: only compared and checked, never touched
    # dequantize: binary16 scale/bias, binary32 output
    assert L.dq_dequantize_rows(A, 8, A + 1, 3, 16, A, 16, None) == dq.DQ_ERR_INVALID_ARG
    assert "2-byte" in L.dq_last_error().decode()
    assert L.dq_dequantize_rows(A, 8, A, 3, 16, A + 2, 16, None) == dq.DQ_ERR_INVALID_ARG
    assert "4-byte" in L.dq_last_error().decode()
    assert L.dq_dequantize_rows_kmeans4(A, 8, A + 1, 3, 16, A, 16, None) == dq.DQ_ERR_INVALID_ARG
    assert "2-byte" in L.dq_last_error().decode()
    # lookup: a table's scale/bias, the ids, offsets and output
    p, keep = _tables((A, A + 1, 10, 8))
    assert L.dq_embbag_int4_fwd(p, 1, 16, A, A, 4, A, None, None) == dq.DQ_ERR_INVALID_ARG
    assert "scale_bias must be 2-byte" in L.dq_last_error().decode()
    p, keep = _tables((A, A, 10, 8))
    for idx, off, out in ((A + 2, A, A), (A, A + 1, A), (A, A, A + 2)):
        assert L.dq_embbag_int4_fwd(p, 1, 16, idx, off, 4, out, None, None) == dq.DQ_ERR_INVALID_ARG
        assert "4-byte aligned" in L.dq_last_error().decode()
    # the owners' buffers
    sl = (ctypes.c_int32 * 1)(0)
    dest = (ctypes.c_void_p * 2)(A, A + 2)
    assert L.dq_embbag_int4_fwd_to_owners(p, 1, 16, A, A, 4, ctypes.cast(sl, ctypes.c_void_p), 1,
                                          ctypes.cast(dest, ctypes.c_void_p), 2, None, None) == dq.DQ_ERR_INVALID_ARG
    assert "dest[1] must be 4-byte" in L.dq_last_error().decode()
    # codebook tables
    arr = (dq._KmeansTable * 1)(dq._KmeansTable(A, A + 1, 10, 8))
    assert L.dq_embbag_kmeans4_fwd(ctypes.cast(arr, ctypes.c_void_p), 1, 16, A, A, 4, A, None,
                                   None) == dq.DQ_ERR_INVALID_ARG
    assert "codebook must be 2-byte" in L.dq_last_error().decode()
    arr = (dq._KmeansTable * 1)(dq._KmeansTable(A, A, 10, 8))
    assert L.dq_embbag_kmeans4_fwd(ctypes.cast(arr, ctypes.c_void_p), 1, 16, A + 2, A, 4, A, None,
                                   None) == dq.DQ_ERR_INVALID_ARG
    assert "4-byte aligned" in L.dq_last_error().decode()


def test_quantizer_outputs_must_be_aligned(L):
    A = 1 << 24
    assert L.dq_quantize_rows_int4(A + 2, 4, 16, 16, A, 8, A, None, None, 0, None, None) == dq.DQ_ERR_INVALID_ARG
    assert "4-byte" in L.dq_last_error().decode()
    assert L.dq_quantize_rows_int4(A, 4, 16, 16, A, 8, A + 1, None, None, 0, None, None) == dq.DQ_ERR_INVALID_ARG
    assert "scale_bias 2-byte" in L.dq_last_error().decode()
    assert L.dq_quantize_rows_int4(A, 4, 16, 16, A, 8, A, A + 2, None, 0, None, None) == dq.DQ_ERR_INVALID_ARG
    assert L.dq_quantize_rows_kmeans4(A, 4, 16, 16, A, 8, A, None, A + 1, 10, None, None) == dq.DQ_ERR_INVALID_ARG
    assert "row_iters" in L.dq_last_error().decode()

"""dq_embbag_int4_bwd_sgd_noalloc: the bag backward for callers that cannot allocate
device memory (a plugin inside a host program that owns the allocator, a process
under a fixed memory budget). It runs on the library's static device scratch and
must give exactly what dq_embbag_int4_bwd_sgd gives with a caller workspace, call
after call, although the scratch keeps the previous call's contents.

This file is collected last on purpose: if it fails, a run that stops at the first
failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import int4_row_wise_b200 as dq


def _batch(rows, d, B, seed):
    r = np.random.default_rng(seed)
    T = len(rows)
    lens = r.integers(0, 12, T * B)
    off = np.zeros(T * B + 1, np.int64)
    off[1:] = np.cumsum(lens)
    ids = []
    for g in range(T * B):
        n = rows[g // B]
        x = r.integers(0, n, lens[g])
        x = np.where(r.random(lens[g]) < 0.3, 2, x)       # a hot row spanning many windows
        x = np.where(r.random(lens[g]) < 0.02, n + 5, x)  # a few invalid ids
        ids.append(x)
    idx = np.concatenate(ids).astype(np.int32)
    grad = r.standard_normal((B, T * d)).astype(np.float32)
    return (torch.from_numpy(idx).cuda(), torch.from_numpy(off.astype(np.int32)).cuda(),
            torch.from_numpy(grad).cuda(), B, int(idx.size))


@pytest.mark.gpu
def test_noalloc_matches_the_workspace_entry_point_on_two_calls(cuda_device):
    rows, d = [4000, 700, 1500], 32
    r = np.random.default_rng(0)
    init = [(r.standard_normal((n, d)).astype(np.float32), r.integers(0, 256, (n, 16), dtype=np.uint8),
             r.integers(0, 1 << 16, (n, 2), dtype=np.uint16).view(np.int16)) for n in rows]

    def tables():
        return [dq.MasterTable(*(torch.from_numpy(a.copy()).cuda() for a in t)) for t in init]

    with_ws, no_ws = tables(), tables()
    fl_ws = torch.zeros(1, dtype=torch.int32, device="cuda")
    fl_na = torch.zeros(1, dtype=torch.int32, device="cuda")
    # the second call is smaller, so stale scratch from the first would show
    for seed, B, lr in ((1, 400, 0.05), (2, 150, 0.2)):
        idx, off, grad, B, n = _batch(rows, d, B, seed)
        ws = torch.empty(dq.dq_embbag_int4_bwd_workspace_bytes(d, n), dtype=torch.uint8, device="cuda")
        assert ws.numel() <= dq.DQ_BWD_STATIC_SCRATCH_BYTES
        dq.dq_embbag_int4_bwd_sgd(with_ws, d, idx, off, B, n, grad, lr, dq.DQ_MODE_GREEDY, ws, ws.numel(), fl_ws)
        dq.dq_embbag_int4_bwd_sgd_noalloc(no_ws, d, idx, off, B, n, grad, lr, dq.DQ_MODE_GREEDY, fl_na)
        torch.cuda.synchronize()
        for a, b in zip(with_ws, no_ws):
            assert torch.equal(a.master.view(torch.int32), b.master.view(torch.int32))
            assert torch.equal(a.codes, b.codes) and torch.equal(a.scale_bias, b.scale_bias)
        assert int(fl_ws.item()) == int(fl_na.item()) == dq.DQ_FLAG_BAD_INDEX
    # the masters did move
    assert not np.array_equal(with_ws[0].master.cpu().numpy(), init[0][0])


def test_noalloc_rejects_calls_beyond_its_static_scratch():
    L = dq.load()
    arr = (dq._MasterTable * 1)(dq._MasterTable(1 << 20, 64, 1 << 22, 32, 1 << 24, 1000))
    n = 10 ** 6  # needs about 290 MB at d = 64
    assert dq.dq_embbag_int4_bwd_workspace_bytes(64, n) > dq.DQ_BWD_STATIC_SCRATCH_BYTES
    st = L.dq_embbag_int4_bwd_sgd_noalloc(ctypes.cast(arr, ctypes.c_void_p), 1, 64, 1 << 26, 1 << 27, 1000, n,
                                          1 << 28, 0.1, 0, None, None)
    assert st == dq.DQ_ERR_INVALID_ARG
    msg = L.dq_last_error().decode()
    assert "static" in msg and "dq_embbag_int4_bwd_sgd" in msg

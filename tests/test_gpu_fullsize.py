"""Parity at the workloads' full sizes, in the launch configuration bench.py
times: each workload's largest table quantized in one launch and each
workload's full lookup call. The oracle checks sampled rows and bags one by
one; properties that hold at any size are checked on every row.

Method: "Post-Training 4-bit Quantization on Embedding Tables", section
提出的方法 (proposed method); lookup: "Deep Learning Recommendation Model for
Personalization and Recommendation Systems", section 提出的方法."""
import numpy as np
import pytest
import torch

import int4_row_wise_b200 as dq
import oracle
from int4_row_wise_b200 import workloads as W
from tests.gpu_util import bag_tolerance_check, to_dev

pytestmark = pytest.mark.gpu

QUANT_CASES = ["kaggle", "terabyte", "production", "sweep-256"]


def _largest_table(name):
    wl = W.workload(name)
    t = int(np.argmax(wl.rows))
    if wl.rows[t] * wl.d * 4 > (1 << 30):
        st = W.SharedTable(wl, t)
        x = torch.from_numpy(st.array).cuda()
        st.close()
    else:
        x = torch.from_numpy(W.table_rows(wl, t)).cuda()
    return wl, t, x


@pytest.mark.parametrize("name", QUANT_CASES)
def test_quantize_full_table(cuda_device, name):
    wl, t, x = _largest_table(name)
    n, d = x.shape
    codes, sb, loss, ij = dq.quantize_rows(x)                 # greedy, one launch, bench's layout
    mcodes, msb, mloss, mij = dq.quantize_rows(x, mode=dq.DQ_MODE_MINMAX)
    deq = dq.dequantize_rows(codes, sb, d)
    torch.cuda.synchronize()
    del x
    loss_h, mloss_h = loss.cpu().numpy(), mloss.cpu().numpy()
    ij_h = ij.cpu().numpy().astype(np.int64)
    # properties on every row
    assert np.all(loss_h <= mloss_h), "greedy loss above the min/max loss"
    assert np.all(ij_h.sum(axis=1) <= 168)
    assert torch.all(mij == 0)
    sbh = sb.cpu().numpy().view(np.uint16)
    assert np.all((sbh & 0x7c00) != 0x7c00), "non-finite binary16 scale or bias"
    # sampled rows against the oracle, bit for bit
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([[0, n - 1], rng.choice(n, 3000 if d <= 64 else 1200, replace=False)]))
    xs = W.sample_rows(wl, t, rows)
    oc, osb, ol, oij = oracle.quantize_rows(xs)
    cb = (d + 1) // 2
    rows_t = torch.from_numpy(rows).cuda()
    assert np.array_equal(codes[rows_t].cpu().numpy()[:, :cb], oc)
    assert np.array_equal(sbh[rows], osb)
    assert np.array_equal(ij_h[rows].astype(np.uint8), oij)
    assert np.array_equal(loss_h[rows].view(np.uint32), ol.view(np.uint32))
    assert np.array_equal(deq[rows_t].cpu().numpy().view(np.uint32),
                          oracle.dequantize_rows(oc, osb, d).view(np.uint32))


def _subset(idx, off, bags):
    """indices/offsets of the listed bags only (same ids, same order)."""
    lens = off[bags + 1] - off[bags]
    o = np.zeros(bags.size + 1, np.int64)
    o[1:] = np.cumsum(lens)
    ids = np.concatenate([idx[off[g]:off[g + 1]] for g in bags]) if o[-1] else np.zeros(0, np.int32)
    return ids.astype(np.int32), o.astype(np.int32)


@pytest.mark.parametrize("name", ["kaggle", "terabyte", "production", "sweep-128"])
def test_lookup_full_call(cuda_device, name):
    wl = W.workload(name)
    d, B, T = wl.d, wl.batch, wl.n_tables
    cld = dq._codes_ld(d)
    host = [W.random_packed_table(n, d, 900 + t, cld) for t, n in enumerate(wl.rows)]
    tabs = [dq.PackedTable(to_dev(c), to_dev(s.view(np.int16))) for c, s in host]
    idx, off = W.lookup_batch(wl)
    out = dq.embbag(tabs, d, to_dev(idx), to_dev(off), B)
    torch.cuda.synchronize()
    out_h = out.cpu().numpy()
    rng = np.random.default_rng(3)
    bags = np.sort(rng.choice(T * B, min(T * B, 4000), replace=False))
    # the oracle on the sampled bags of each table
    for t in range(T):
        bt = bags[(bags >= t * B) & (bags < (t + 1) * B)]
        if bt.size == 0:
            continue
        sidx, soff = _subset(idx, off, bt)
        ref, mag, skipped = oracle.embbag([host[t]], d, sidx, soff, bt.size, with_abs_sum=True)
        assert skipped == 0
        got = out_h[bt - t * B, t * d:(t + 1) * d]
        bag_tolerance_check(got, ref, mag)
        if wl.pooling == (1, 1):
            assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))

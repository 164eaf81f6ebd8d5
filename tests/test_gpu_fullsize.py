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
from tests.gpu_util import assert_bwd_parity, bag_tolerance_check, to_dev

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


def test_bwd_full_kaggle_call(cuda_device):
    """The bag backward + SGD + re-quantization on the Kaggle-shaped workload's own
    tables (all 26, 12.1M rows) and its full lookup batch, as bench.py --bwd launches
    it. Sampled rows (the hottest ones, with hundreds of entries each, and random
    touched ones) against the oracle by the backward's criterion (masters bit-identical
    on at least 99.99 % of the sampled rows, within 1 ulp on the rest; packed rows the
    oracle's quantization of the GPU's masters); sampled untouched rows unchanged.
    (Training step of "Deep Quantized Recommendation Model (DQRM)", repository page.)"""
    wl = W.workload("kaggle")
    d, B, T = wl.d, wl.batch, wl.n_tables
    cld = dq._codes_ld(d)
    rng = np.random.default_rng(31)
    masters = [np.ascontiguousarray(W.table_rows(wl, t)) for t in range(T)]
    codes = [rng.integers(0, 256, (n, cld), dtype=np.uint8) for n in wl.rows]
    sbs = [rng.integers(0, 1 << 16, (n, 2), dtype=np.uint16) for n in wl.rows]
    idx, off = W.lookup_batch(wl, 0)
    grad = rng.standard_normal((B, T * d)).astype(np.float32)
    lr = 0.05
    tabs = [dq.MasterTable(to_dev(m), to_dev(c), to_dev(s.view(np.int16))) for m, c, s in zip(masters, codes, sbs)]
    dq.embbag_bwd_sgd(tabs, d, to_dev(idx), to_dev(off), B, to_dev(grad), lr)
    torch.cuda.synchronize()
    # rows touched, with their entry counts
    base = np.concatenate([[0], np.cumsum(wl.rows)]).astype(np.int64)
    t_of = np.repeat(np.arange(T), [off[(t + 1) * B] - off[t * B] for t in range(T)])
    keys, counts = np.unique(base[t_of] + idx.astype(np.int64), return_counts=True)
    hot = keys[np.argsort(-counts)[:20]]
    sample = np.unique(np.concatenate([hot, rng.choice(keys, 2000, replace=False)]))
    assert counts.max() > 64  # some rows have more entries than one 64-entry piece of the kernels
    oracle.embbag_bwd_sgd(masters, codes, sbs, d, idx, off, B, grad, lr, sample_keys=sample)
    got, want, touched = [], [], []
    for key in sample:
        t = int(np.searchsorted(base, key, side="right") - 1)
        r = int(key - base[t])
        got.append((tabs[t].master[r:r + 1].cpu().numpy(), tabs[t].codes[r:r + 1].cpu().numpy(),
                    tabs[t].scale_bias[r:r + 1].cpu().numpy().view(np.uint16)))
        want.append((masters[t][r:r + 1], codes[t][r:r + 1], sbs[t][r:r + 1]))
        touched.append(np.ones(1, bool))
    assert_bwd_parity(got, want, touched, d)
    # untouched rows keep their values (the host arrays still hold the inputs there)
    for t in range(0, T, 5):
        n = wl.rows[t]
        rows = rng.choice(n, min(n, 500), replace=False)
        mine = keys[(keys >= base[t]) & (keys < base[t + 1])] - base[t]
        rows = np.setdiff1d(rows, mine)
        rt = torch.from_numpy(rows).cuda()
        assert np.array_equal(tabs[t].master[rt].cpu().numpy(), masters[t][rows])
        assert np.array_equal(tabs[t].codes[rt].cpu().numpy(), codes[t][rows])

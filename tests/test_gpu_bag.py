"""GPU parity of dq_dequantize_rows (bit-exact) and dq_embbag_int4_fwd (within
1e-5 of the summed magnitudes, bit-exact for bags of one id) against the oracle.

Lookup: "Deep Learning Recommendation Model for Personalization and
Recommendation Systems", section 提出的方法 (proposed method), bullet 1."""
import numpy as np
import pytest
import torch

import int4_row_wise_b200 as dq
import oracle
from int4_row_wise_b200 import workloads as W
from tests.gpu_util import bag_tolerance_check, gpu_quantize, to_dev

pytestmark = pytest.mark.gpu


def _packed(n, d, seed, codes_ld=None):
    return W.random_packed_table(n, d, seed, codes_ld)


@pytest.mark.parametrize("d,codes_ld,out_ld", [(16, 8, 16), (128, 64, 128), (256, 128, 256), (32, 16, 32),
                                               (7, 4, 7), (16, 9, 16), (64, 32, 65), (1, 1, 1), (48, 24, 48),
                                               (100, 50, 100), (12, 6, 12), (20, 10, 24)])
def test_dequantize_bit_exact(cuda_device, d, codes_ld, out_ld):
    n = 5003
    codes, sb = _packed(n, d, d, codes_ld)
    want = oracle.dequantize_rows(codes, sb, d)
    out = torch.full((n, out_ld), -7.0, dtype=torch.float32, device="cuda")
    dq.dq_dequantize_rows(to_dev(codes), codes_ld, to_dev(sb.view(np.int16)), n, d, out, out_ld)
    got = out.cpu().numpy()
    assert np.array_equal(got[:, :d].view(np.uint32), want.view(np.uint32))
    assert np.all(got[:, d:] == -7.0)


def _bags(T, B, rows, lo, hi, seed, bad=False):
    r = np.random.default_rng(seed)
    lens = r.integers(lo, hi + 1, T * B)
    off = np.zeros(T * B + 1, np.int64)
    off[1:] = np.cumsum(lens)
    idx = np.concatenate([r.integers(0, rows[g // B], lens[g]) for g in range(T * B)]) if off[-1] else np.zeros(0)
    idx = idx.astype(np.int32)
    if bad and idx.size > 10:
        idx[3] = -1
        idx[7] = rows[0] + 5
    return idx, off.astype(np.int32)


def _gpu_bag(tabs, d, idx, off, B, flags=False):
    dev_tabs = [dq.PackedTable(to_dev(c), to_dev(s.view(np.int16))) for c, s in tabs]
    fl = torch.zeros(1, dtype=torch.int32, device="cuda") if flags else None
    out = torch.full((B, len(tabs) * d), 123.0, dtype=torch.float32, device="cuda")
    dq.dq_embbag_int4_fwd(dev_tabs, d, to_dev(idx if idx.size else np.zeros(1, np.int32)), to_dev(off), B,
                          out, fl)
    torch.cuda.synchronize()
    return out.cpu().numpy(), (int(fl.item()) if flags else None)


@pytest.mark.parametrize("d", [16, 32, 64, 128, 256, 512, 1024, 7, 48, 100])
@pytest.mark.parametrize("pool", [(1, 1), (0, 3), (0, 10), (20, 80)])
def test_bag_matches_oracle(cuda_device, d, pool):
    T, B = 3, 97
    rows = [500, 1000, 37]
    tabs = [_packed(n, d, 10 * d + t, ((d + 1) // 2 + 15) // 16 * 16) for t, n in enumerate(rows)]
    idx, off = _bags(T, B, rows, pool[0], pool[1], d)
    got, _ = _gpu_bag(tabs, d, idx, off, B)
    ref, mag, skipped = oracle.embbag(tabs, d, idx, off, B, with_abs_sum=True)
    assert skipped == 0
    bag_tolerance_check(got, ref, mag)
    if pool == (1, 1):
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def _scaled_table(n, d, seed, scales):
    """A random packed table whose rows cycle through the given binary16 scales."""
    codes, sb = _packed(n, d, seed, ((d + 1) // 2 + 15) // 16 * 16)
    s = np.asarray(scales, np.float16)[np.arange(n) % len(scales)]
    sb[:, 0] = s.view(np.uint16)
    return codes, sb


@pytest.mark.parametrize("d", [16, 48, 128])
def test_dequantize_rows_of_every_scale(cuda_device, d):
    """Rows whose binary16 scales run from zero and subnormals through 1/2 to 60000, both
    signs: rows with |scale| < 1/2 take the scaled-subnormal decode, the others the
    exponent-byte decode; both must give fma(q, scale, bias) bit for bit."""
    scales = [0.0, -0.0, 6e-8, 1e-4, 0.01, 0.4998, 0.5, 0.5005, 1.0, 3.0, 250.0, 60000.0, -0.3, -0.7, -2.0]
    n = 3001
    codes, sb = _scaled_table(n, d, 77, scales)
    want = oracle.dequantize_rows(codes, sb, d)
    out = torch.empty((n, d), dtype=torch.float32, device="cuda")
    dq.dq_dequantize_rows(to_dev(codes), codes.shape[1], to_dev(sb.view(np.int16)), n, d, out, d)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("d", [16, 64, 128, 256])
def test_bag_rows_of_every_scale(cuda_device, d):
    """Bags averaging 6 ids (the long-bag layout), some of one id, over rows whose
    binary16 scales run from zero and subnormals through 1/2 to 60000, both signs: a
    group of rows takes the scaled-subnormal decode only while every |scale| < 1/2, the
    exponent-byte decode otherwise, and both must sum fma(q, scale, bias)."""
    scales = [0.0, -0.0, 6e-8, 1e-4, 0.01, 0.4998, 0.5, 0.5005, 1.0, 3.0, 250.0, 60000.0, -0.3, -0.7, -2.0]
    T, B = 2, 64
    rows = [300, 77]
    tabs = [_scaled_table(n, d, 40 + t, scales) for t, n in enumerate(rows)]
    for seed, (lo, hi) in ((d, (0, 12)), (d + 1, (4, 8))):
        idx, off = _bags(T, B, rows, lo, hi, seed)
        got, _ = _gpu_bag(tabs, d, idx, off, B)
        ref, mag, skipped = oracle.embbag(tabs, d, idx, off, B, with_abs_sum=True)
        assert skipped == 0
        bag_tolerance_check(got, ref, mag)
        lens = np.diff(off.astype(np.int64)).reshape(T, B).T          # [B, T]
        one = np.repeat(lens == 1, d, axis=1)
        assert np.array_equal(got[one].view(np.uint32), ref[one].view(np.uint32))


@pytest.mark.parametrize("n_dest", [1, 2, 3, 4])
@pytest.mark.parametrize("d,pool", [(16, (1, 1)), (64, (4, 12)), (128, (0, 3)), (100, (1, 6))])
def test_bag_to_owners_matches_oracle(cuda_device, n_dest, d, pool):
    """dq_embbag_int4_fwd_to_owners over n_dest buffers on one GPU: bag (t, b) lands in
    buffer b // bl, row b % bl, column block slot[t] of t_out, with the lookup's values;
    the other column blocks are left as they were."""
    T, B, t_out = 3, 96, 5
    slots = [4, 0, 2]
    rows = [500, 1000, 37]
    cld = ((d + 1) // 2 + 15) // 16 * 16
    tabs = [_packed(n, d, 30 * d + t, cld) for t, n in enumerate(rows)]
    idx, off = _bags(T, B, rows, pool[0], pool[1], d + n_dest)
    ref, mag, _ = oracle.embbag(tabs, d, idx, off, B, with_abs_sum=True)
    bl = B // n_dest
    dest = [torch.full((bl, t_out * d), 7.0, dtype=torch.float32, device="cuda") for _ in range(n_dest)]
    dev_tabs = [dq.PackedTable(to_dev(c), to_dev(s.view(np.int16))) for c, s in tabs]
    dq.dq_embbag_int4_fwd_to_owners(dev_tabs, d, to_dev(idx if idx.size else np.zeros(1, np.int32)), to_dev(off), B,
                                    slots, t_out, dest)
    torch.cuda.synchronize()
    got = np.empty((B, T * d), np.float32)
    for r in range(n_dest):
        o = dest[r].cpu().numpy()
        for t, sl in enumerate(slots):
            got[r * bl:(r + 1) * bl, t * d:(t + 1) * d] = o[:, sl * d:(sl + 1) * d]
        for sl in set(range(t_out)) - set(slots):
            assert np.all(o[:, sl * d:(sl + 1) * d] == 7.0)
    bag_tolerance_check(got, ref, mag)
    lens = np.diff(off.astype(np.int64)).reshape(T, B).T
    one = np.repeat(lens == 1, d, axis=1)
    assert np.array_equal(got[one].view(np.uint32), ref[one].view(np.uint32))


@pytest.mark.parametrize("d", [16, 64, 100])
def test_bag_to_owners_flags_bad_ids(cuda_device, d):
    """Invalid ids are skipped and flagged in the owner-store form as in the plain lookup."""
    T, B = 2, 64
    rows = [300, 40]
    cld = ((d + 1) // 2 + 15) // 16 * 16
    tabs = [_packed(n, d, 70 + t, cld) for t, n in enumerate(rows)]
    idx, off = _bags(T, B, rows, 1, 6, d, bad=True)
    ref, mag, skipped = oracle.embbag(tabs, d, idx, off, B, with_abs_sum=True)
    assert skipped > 0
    dest = [torch.zeros((B // 2, T * d), dtype=torch.float32, device="cuda") for _ in range(2)]
    fl = torch.zeros(1, dtype=torch.int32, device="cuda")
    dev_tabs = [dq.PackedTable(to_dev(c), to_dev(s.view(np.int16))) for c, s in tabs]
    dq.dq_embbag_int4_fwd_to_owners(dev_tabs, d, to_dev(idx), to_dev(off), B, [0, 1], T, dest, d_flags=fl)
    torch.cuda.synchronize()
    got = np.concatenate([x.cpu().numpy() for x in dest])
    bag_tolerance_check(got, ref, mag)
    assert fl.item() & dq.DQ_FLAG_BAD_INDEX


def test_bag_bad_ids_and_offsets(cuda_device):
    d, T, B = 64, 2, 50
    rows = [100, 100]
    tabs = [_packed(n, d, 5 + t) for t, n in enumerate(rows)]
    idx, off = _bags(T, B, rows, 1, 6, 3, bad=True)
    off2 = off.copy()
    off2[20] = off2[21] + 2   # bag 19 gets decreasing offsets... and bag 20 a longer span
    got, fl = _gpu_bag(tabs, d, idx, off2, B, flags=True)
    ref, mag, skipped = oracle.embbag(tabs, d, idx, off2, B, with_abs_sum=True)
    assert skipped > 0
    assert fl & dq.DQ_FLAG_BAD_INDEX and fl & dq.DQ_FLAG_BAD_OFFSETS
    bag_tolerance_check(got, ref, mag)
    got, fl = _gpu_bag(tabs, d, *_bags(T, B, rows, 1, 6, 4), B, flags=True)
    assert fl == 0


def test_tiny_workload_end_to_end(cuda_device):
    """Quantize the tiny table on the GPU, then look it up on the GPU; the oracle
    sums the same packed table."""
    wl = W.workload("tiny")
    x = W.table_rows(wl, 0)
    codes, sb, _, _, _ = gpu_quantize(x)
    idx, off = W.lookup_batch(wl)
    got, _ = _gpu_bag([(codes, sb)], wl.d, idx, off, wl.batch)
    ref, mag, _ = oracle.embbag([(codes, sb)], wl.d, idx, off, wl.batch, with_abs_sum=True)
    bag_tolerance_check(got, ref, mag)
    deq = torch.empty((x.shape[0], wl.d), dtype=torch.float32, device="cuda")
    dq.dq_dequantize_rows(to_dev(codes), codes.shape[1], to_dev(sb.view(np.int16)), x.shape[0], wl.d, deq, wl.d)
    assert np.array_equal(deq.cpu().numpy().view(np.uint32), oracle.dequantize_rows(codes, sb, wl.d).view(np.uint32))


@pytest.mark.parametrize("name", ["kaggle", "sweep-64"])
def test_workload_batches_on_random_tables(cuda_device, name):
    """A full lookup call of the workload (its ids, offsets and batch), over random
    packed tables of its table sizes."""
    wl = W.workload(name)
    tabs = [_packed(n, wl.d, 1000 + t, ((wl.d + 1) // 2 + 15) // 16 * 16) for t, n in enumerate(wl.rows)]
    idx, off = W.lookup_batch(wl)
    got, _ = _gpu_bag(tabs, wl.d, idx, off, wl.batch)
    ref, mag, _ = oracle.embbag(tabs, wl.d, idx, off, wl.batch, with_abs_sum=True)
    bag_tolerance_check(got, ref, mag)
    if wl.pooling == (1, 1):
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_bag_into_empty_table_skips_every_id(cuda_device):
    d, B = 64, 8
    full = _packed(50, d, 1)
    empty = (np.zeros((0, 32), np.uint8), np.zeros((0, 2), np.uint16))
    idx = np.array([0, 1, 2, 3, 4, 5, 6, 7, 0, 1, 2, 3, 4, 5, 6, 7], np.int32)
    off = np.arange(0, 17, 1, dtype=np.int32)  # 2 tables x 8 one-id bags
    got, fl = _gpu_bag([full, empty], d, idx, off, B, flags=True)
    ref, mag, skipped = oracle.embbag([full, empty], d, idx, off, B, with_abs_sum=True)
    assert skipped == 8 and fl & dq.DQ_FLAG_BAD_INDEX
    assert np.all(got[:, d:] == 0)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_injected_launch_failure_raises(cuda_device, monkeypatch):
    x = torch.zeros((10, 16), dtype=torch.float32, device="cuda")
    codes = torch.full((10, 8), 7, dtype=torch.uint8, device="cuda")
    sb = torch.zeros((10, 2), dtype=torch.int16, device="cuda")
    monkeypatch.setenv("DQ_FAULT_INJECT", "launch")
    with pytest.raises(dq.DqError) as ei:
        dq.dq_quantize_rows_int4(x, 10, 16, 16, codes, 8, sb)
    assert ei.value.status == dq.DQ_ERR_CUDA and "injected" in str(ei.value)
    torch.cuda.synchronize()
    assert torch.all(codes == 7)  # nothing was launched
    monkeypatch.delenv("DQ_FAULT_INJECT")
    dq.dq_quantize_rows_int4(x, 10, 16, 16, codes, 8, sb)
    torch.cuda.synchronize()
    assert torch.all(codes == 0)

"""GPU parity of dq_embbag_int4_bwd_sgd (bag backward, SGD step on binary32 masters,
re-quantization of the touched rows) against the oracle, by the criterion of
tests.gpu_util.assert_bwd_parity: masters bit-identical on at least 99.99 % of the
touched rows and within 1 ulp on the rest, packed rows equal to the oracle's
quantization of the GPU's masters, untouched rows unchanged.

The training step of "Deep Quantized Recommendation Model (DQRM)", repository page
(INT4 quantization-aware training of the embedding tables)."""
import numpy as np
import pytest
import torch

import int4_row_wise_b200 as dq
import oracle
from tests.gpu_util import assert_bwd_parity, to_dev, touched_masks

pytestmark = pytest.mark.gpu


def _case(rows, d, B, pool, seed, hot=0.0, bad_ids=0.0, ld_pad=0, cld=None, scale=1.0):
    """Masters, packed tables (random bytes: only touched rows may change), bags and the
    output gradient for len(rows) tables of width d."""
    r = np.random.default_rng(seed)
    T = len(rows)
    cld = cld or dq._codes_ld(d)
    masters = [(r.standard_normal((n, d + ld_pad)) * scale).astype(np.float32) for n in rows]
    codes = [r.integers(0, 256, (n, cld), dtype=np.uint8) for n in rows]
    sbs = [r.integers(0, 1 << 16, (n, 2), dtype=np.uint16) for n in rows]
    lens = r.integers(pool[0], pool[1] + 1, T * B)
    off = np.zeros(T * B + 1, np.int64)
    off[1:] = np.cumsum(lens)
    parts = []
    for g in range(T * B):
        n = rows[g // B]
        ids = r.integers(0, max(n, 1), lens[g])
        if hot:
            ids = np.where(r.random(lens[g]) < hot, min(3, max(n - 1, 0)), ids)
        if bad_ids:
            ids = np.where(r.random(lens[g]) < bad_ids, r.choice([-1, n, n + 7, -(1 << 30)], lens[g]), ids)
        if n == 0:
            ids = np.full(lens[g], -1)
        parts.append(ids)
    idx = np.concatenate(parts + [np.zeros(0, np.int64)]).astype(np.int32)
    grad = r.standard_normal((B, T * d)).astype(np.float32)
    return masters, codes, sbs, idx, off.astype(np.int32), grad


def _run_gpu(masters, codes, sbs, d, idx, off, B, grad, lr, mode, repeat=1):
    tabs = [dq.MasterTable(to_dev(m), to_dev(c), to_dev(s.view(np.int16))) for m, c, s in zip(masters, codes, sbs)]
    fl = torch.zeros(1, dtype=torch.int32, device="cuda")
    gi, go, gg = to_dev(idx), to_dev(off), to_dev(grad)
    ws = None
    for _ in range(repeat):
        ws = dq.embbag_bwd_sgd(tabs, d, gi, go, B, gg, lr, mode, workspace=ws, d_flags=fl)
    torch.cuda.synchronize()
    out = [(t.master.cpu().numpy(), t.codes.cpu().numpy(), t.scale_bias.cpu().numpy().view(np.uint16)) for t in tabs]
    return out, int(fl.item())


def _run_oracle(masters, codes, sbs, d, idx, off, B, grad, lr, mode):
    M = [m.copy() for m in masters]
    C = [c.copy() for c in codes]
    S = [s.copy() for s in sbs]
    # the oracle takes d-wide rows at stride ld: pass the padded arrays, it reads d of each
    rc = oracle.embbag_bwd_sgd(M, C, S, d, idx, off, B, grad, lr, mode)
    return list(zip(M, C, S)), rc


def _assert_same(got, want, masters, d, idx, off, B, mode=dq.DQ_MODE_GREEDY):
    assert_bwd_parity(got, want, touched_masks([m.shape[0] for m in masters], B, idx, off), d, mode)


def _check(rows, d, B, pool, seed, lr=0.05, mode=dq.DQ_MODE_GREEDY, expect_flags=0, **kw):
    masters, codes, sbs, idx, off, grad = _case(rows, d, B, pool, seed, **kw)
    got, flags = _run_gpu(masters, codes, sbs, d, idx, off, B, grad, lr, mode)
    want, rc = _run_oracle(masters, codes, sbs, d, idx, off, B, grad, lr, mode)
    _assert_same(got, want, masters, d, idx, off, B, mode)
    assert flags & (dq.DQ_FLAG_BAD_INDEX | dq.DQ_FLAG_BAD_OFFSETS) == expect_flags
    return rc, flags


@pytest.mark.parametrize("d", [1, 2, 5, 16, 17, 32, 48, 64, 100, 128, 256, 512, 1024])
def test_bwd_widths(cuda_device, d):
    B = 96 if d <= 256 else 24
    _check([700, 35, 1200], d, B, (0, 9), seed=d, hot=0.3)


@pytest.mark.parametrize("pool,hot", [((1, 1), 0.0), ((1, 1), 0.9), ((20, 80), 0.2), ((0, 3), 0.5),
                                      ((30, 30), 0.99)])
def test_bwd_pools_and_hot_rows(cuda_device, pool, hot):
    # hot rows repeat hundreds of times: their entries span many windows of 64
    _check([5000, 300], 64, 512, pool, seed=11, hot=hot)


def test_bwd_min_max_mode(cuda_device):
    _check([900, 900], 32, 128, (1, 6), seed=3, mode=dq.DQ_MODE_MINMAX, hot=0.2)


@pytest.mark.parametrize("lr", [0.0, 1e-3, float(np.float32(1 / 3)), 17.0, -0.5])
def test_bwd_learning_rates(cuda_device, lr):
    _check([400], 16, 200, (1, 4), seed=5, lr=lr, hot=0.3)


def test_bwd_invalid_ids_and_empty_table(cuda_device):
    rc, flags = _check([300, 0, 200], 16, 64, (0, 8), seed=6, bad_ids=0.2, hot=0.1,
                       expect_flags=dq.DQ_FLAG_BAD_INDEX)
    assert rc > 0


def test_bwd_strided_masters_and_codes(cuda_device):
    _check([600, 250], 64, 80, (1, 5), seed=7, ld_pad=3, cld=40, hot=0.4)
    _check([600], 16, 80, (1, 5), seed=8, ld_pad=1, cld=9, hot=0.4)


@pytest.mark.parametrize("count", [1, 63, 64, 65, 127, 128, 129, 64 * 9 + 5])
def test_bwd_one_row_at_window_edges(cuda_device, count):
    # one-hot bags on one row, preceded by `lead` entries of a lower row, so the
    # hot row's entries start at different positions relative to the windows
    d = 32
    for lead in (0, 1, 63, 64):
        r = np.random.default_rng(count * 100 + lead)
        n_b = lead + count
        idx = np.array([0] * lead + [5] * count, np.int32)
        off = np.arange(n_b + 1, dtype=np.int32)
        grad = r.standard_normal((n_b, d)).astype(np.float32)
        masters = [r.standard_normal((8, d)).astype(np.float32)]
        codes = [np.zeros((8, dq._codes_ld(d)), np.uint8)]
        sbs = [np.zeros((8, 2), np.uint16)]
        got, flags = _run_gpu(masters, codes, sbs, d, idx, off, n_b, grad, 0.1, dq.DQ_MODE_GREEDY)
        want, _ = _run_oracle(masters, codes, sbs, d, idx, off, n_b, grad, 0.1, dq.DQ_MODE_GREEDY)
        _assert_same(got, want, masters, d, idx, off, n_b)


@pytest.mark.parametrize("bad", ["decreasing", "first", "last"])
def test_bwd_bad_offsets_change_nothing(cuda_device, bad):
    masters, codes, sbs, idx, off, grad = _case([500, 400], 16, 50, (1, 4), seed=9)
    off = off.copy()
    if bad == "decreasing":
        off[10] = off[11] + 1
    elif bad == "first":
        off[0] = 1
    else:
        off[-1] -= 1
    got, flags = _run_gpu(masters, codes, sbs, 16, idx, off, 50, grad, 0.1, dq.DQ_MODE_GREEDY)
    assert flags & dq.DQ_FLAG_BAD_OFFSETS
    for (gm, gc, gs), m, c, s in zip(got, masters, codes, sbs):
        assert np.array_equal(gm, m) and np.array_equal(gc, c) and np.array_equal(gs, s)


def test_bwd_repeated_steps_match_the_oracle(cuda_device):
    # three steps on the same batch: each starts from the previous step's masters
    masters, codes, sbs, idx, off, grad = _case([3000, 800], 64, 256, (1, 30), seed=12, hot=0.3)
    got, _ = _run_gpu(masters, codes, sbs, 64, idx, off, 256, grad, 0.01, dq.DQ_MODE_GREEDY, repeat=3)
    state = (masters, codes, sbs)
    for _ in range(3):
        want, _ = _run_oracle(*state, 64, idx, off, 256, grad, 0.01, dq.DQ_MODE_GREEDY)
        state = tuple(list(x) for x in zip(*want))
    _assert_same(got, want, masters, 64, idx, off, 256)


def test_bwd_touched_rows_only(cuda_device):
    masters, codes, sbs, idx, off, grad = _case([2000], 16, 100, (1, 3), seed=13)
    got, _ = _run_gpu(masters, codes, sbs, 16, idx, off, 100, grad, 0.1, dq.DQ_MODE_GREEDY)
    touched = np.zeros(2000, bool)
    touched[idx] = True
    gm, gc, gs = got[0]
    assert np.array_equal(gm[~touched], masters[0][~touched])
    assert np.array_equal(gc[~touched], codes[0][~touched]) and np.array_equal(gs[~touched], sbs[0][~touched])
    assert not np.any(np.all(gm[touched] == masters[0][touched], axis=1))

"""CPU checks of the backward's parity criterion (tests.gpu_util.assert_bwd_parity):
it must accept the oracle's own result and a rare 1-ulp row that carries the oracle's
quantization of its master, and reject everything else."""
import numpy as np
import pytest

import oracle
from tests.gpu_util import assert_bwd_parity, touched_masks


def _state(seed=0, n=3000, d=8, B=2000):
    r = np.random.default_rng(seed)
    W = [r.standard_normal((n, d)).astype(np.float32)]
    C = [np.zeros((n, (d + 1) // 2), np.uint8)]
    S = [np.zeros((n, 2), np.uint16)]
    idx = r.integers(0, n, B).astype(np.int32)
    off = np.arange(B + 1, dtype=np.int32)
    g = r.standard_normal((B, d)).astype(np.float32)
    oracle.embbag_bwd_sgd(W, C, S, d, idx, off, B, g, 0.1)
    return W, C, S, touched_masks([n], B, idx, off), d


def _copy(W, C, S):
    return [(W[0].copy(), C[0].copy(), S[0].copy())]


def _bump(got, row, d, ulps=1):
    m, c, s = got[0]
    m[row, 0] = np.nextafter(m[row, 0], np.float32(np.inf)) if ulps == 1 else m[row, 0] * np.float32(1.001)
    cc, ss, _, _ = oracle.quantize_rows(np.ascontiguousarray(m[row:row + 1, :d]))
    c[row] = cc[0]
    s[row] = ss[0]


def test_accepts_the_oracle_itself():
    W, C, S, tm, d = _state()
    assert assert_bwd_parity(_copy(W, C, S), _copy(W, C, S), tm, d)[0] == 0


def test_accepts_one_row_one_ulp_off_with_its_own_quantization():
    W, C, S, tm, d = _state()
    got = _copy(W, C, S)
    row = int(np.nonzero(tm[0])[0][0])
    _bump(got, row, d)
    assert assert_bwd_parity(got, _copy(W, C, S), tm, d)[0] == 1


@pytest.mark.parametrize("mistake", ["two_rows", "beyond_ulp", "untouched", "stale_codes"])
def test_rejects(mistake):
    W, C, S, tm, d = _state()
    got = _copy(W, C, S)
    rows = np.nonzero(tm[0])[0]
    if mistake == "two_rows":        # 2 of ~1500 touched rows: above 99.99 %
        _bump(got, int(rows[0]), d)
        _bump(got, int(rows[1]), d)
    elif mistake == "beyond_ulp":
        _bump(got, int(rows[0]), d, ulps=1000)
    elif mistake == "untouched":
        r = int(np.nonzero(~tm[0])[0][0])
        got[0][0][r, 0] = np.nextafter(got[0][0][r, 0], np.float32(np.inf))
    else:                            # masters agree, codes do not
        got[0][1][int(rows[0]), 0] ^= 1
    with pytest.raises(AssertionError):
        assert_bwd_parity(got, _copy(W, C, S), tm, d)

"""GPU parity of dq_row_l2_error, the normalized l2 error of packed rows, against
the oracle (binary64 on both sides, summation orders differ: rtol 1e-12).

"Post-Training 4-bit Quantization on Embedding Tables", section 提出的方法 (proposed
method), bullet 5; section 主要发现 (main findings), bullet 2."""
import numpy as np
import pytest
import torch

import int4_row_wise_b200 as dq
import oracle
from int4_row_wise_b200 import workloads as W
from tests.gpu_util import gpu_quantize, to_dev

pytestmark = pytest.mark.gpu


def _gpu_l2(x, codes, sb, x_ld=None):
    n, d = x.shape
    ld = d if x_ld is None else x_ld
    buf = np.zeros((n, ld), np.float32)
    buf[:, :d] = x
    err = torch.full((n,), -1.0, dtype=torch.float64, device="cuda")
    tot = torch.zeros(1, dtype=torch.float64, device="cuda")
    dq.dq_row_l2_error(to_dev(buf), n, d, ld, to_dev(codes), codes.shape[1], to_dev(sb.view(np.int16)), err, tot)
    torch.cuda.synchronize()
    return err.cpu().numpy(), float(tot.item())


@pytest.mark.parametrize("d,x_ld", [(1, 1), (3, 3), (7, 9), (16, 16), (16, 20), (33, 33), (64, 64), (128, 128),
                                    (256, 256), (1000, 1000), (1024, 1024)])
def test_row_l2_matches_oracle(cuda_device, d, x_ld):
    r = np.random.default_rng(d)
    n = max(50, 20000 // d) + 3
    x = (r.standard_t(3, (n, d)) * r.lognormal(0, 1, (n, 1))).astype(np.float32)
    codes, sb, _, _, _ = gpu_quantize(x)
    got, tot = _gpu_l2(x, codes, sb, x_ld)
    want, wtot = oracle.row_l2_error(x, codes, sb)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=0)
    assert abs(tot - wtot) <= 1e-12 * wtot


def test_row_l2_special_rows(cuda_device):
    q = np.arange(16)
    x = np.stack([(0.25 * q).astype(np.float32), np.zeros(16, np.float32), np.full(16, 0.1, np.float32)])
    codes, sb, _, _, _ = gpu_quantize(x)
    got, _ = _gpu_l2(x, codes, sb)
    want, _ = oracle.row_l2_error(x, codes, sb)
    assert got[0] == 0 and got[1] == 0
    np.testing.assert_allclose(got, want, rtol=1e-12)


@pytest.mark.parametrize("name", ["tiny", "kaggle", "terabyte", "sweep-256"])
def test_quality_on_workloads(cuda_device, name):
    """Greedy lowers the normalized l2 error against plain min/max on every
    workload (the pages' finding, on synthetic tables); the mean over the largest
    table matches the oracle's."""
    wl = W.workload(name)
    t = int(np.argmax(wl.rows))
    x = W.table_rows(wl, t, 0, min(wl.rows[t], 400_000))
    xd = to_dev(x)
    means = {}
    for mode in (dq.DQ_MODE_GREEDY, dq.DQ_MODE_MINMAX):
        codes, sb, _, _ = dq.quantize_rows(xd, mode=mode)
        err, mean = dq.row_l2_error(xd, codes, sb)
        torch.cuda.synchronize()
        cb = (wl.d + 1) // 2
        want, wtot = oracle.row_l2_error(x, codes.cpu().numpy()[:, :cb], sb.cpu().numpy().view(np.uint16))
        np.testing.assert_allclose(err.cpu().numpy(), want, rtol=1e-12)
        assert abs(float(mean.item()) - wtot / x.shape[0]) <= 1e-12 * wtot / x.shape[0]
        means[mode] = float(mean.item())
    assert means[dq.DQ_MODE_GREEDY] < means[dq.DQ_MODE_MINMAX]

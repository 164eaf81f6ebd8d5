"""Pins the oracle's binary16 conversions against library routines.

The scale and bias of a row are stored as FP16 ("Post-Training 4-bit
Quantization on Embedding Tables", section 提出的方法 / proposed method,
bullet 2). The oracle converts with its own code; these tests compare it with
torch's and numpy's IEEE round-to-nearest-even casts.
"""
import numpy as np
import pytest
import torch

import oracle


def _ref_f16(f32: np.ndarray) -> np.ndarray:
    return torch.from_numpy(f32).to(torch.float16).view(torch.int16).numpy().view(np.uint16)


def test_torch_and_numpy_casts_agree():
    # the two library routines agree with each other on a spread of patterns
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 2 ** 32, 1 << 22, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    with np.errstate(over="ignore"):
        assert np.array_equal(_ref_f16(f), f.astype(np.float16).view(np.uint16))


def test_f32_to_f16_exhaustive_where_rounding_happens():
    # Every positive binary32 with exponent field 101..143 (2^-26 <= x < 2^17):
    # the whole range whose result is neither forced to 0 nor to infinity,
    # subnormal binary16 results and the overflow boundary included.
    man = np.arange(1 << 23, dtype=np.uint32)
    for ef in range(101, 144):
        f = (man | np.uint32(ef << 23)).view(np.float32)
        got = oracle.f32_to_f16_array(f)
        ref = _ref_f16(f)
        bad = np.nonzero(got != ref)[0]
        assert bad.size == 0, (ef, f[bad[:4]], got[bad[:4]], ref[bad[:4]])


def test_f32_to_f16_forced_ranges_and_sign():
    rng = np.random.default_rng(2)
    # below 2^-26: zero; at or above 2^17: infinity; both signs; a stride over all patterns
    bits = np.concatenate([
        np.arange(0, 2 ** 32, 4099, dtype=np.uint64).astype(np.uint32),
        rng.integers(0, 2 ** 32, 1 << 20, dtype=np.uint64).astype(np.uint32),
        np.array([0x80000000, 0x7f800000, 0xff800000, 0x477fefff, 0x477ff000, 0x33000000,
                  0x33000001, 0xb3000001, 0x387fc000], dtype=np.uint32),
    ])
    f = bits.view(np.float32)
    got = oracle.f32_to_f16_array(f)
    fin = np.isfinite(f)
    assert np.array_equal(got[fin], _ref_f16(f[fin]))
    nan = np.isnan(f)
    assert np.all((got[nan] & 0x7c00) == 0x7c00) and np.all((got[nan] & 0x3ff) != 0)
    # 65520 is the midpoint between 65504 and 2^16: ties to even gives infinity
    assert oracle.f32_to_f16_bits(65520.0) == 0x7c00
    assert oracle.f32_to_f16_bits(65519.996) == 0x7bff
    # half of the smallest subnormal rounds to even (zero); just above it rounds up
    assert oracle.f32_to_f16_bits(2.0 ** -25) == 0
    assert oracle.f32_to_f16_bits(np.nextafter(np.float32(2.0 ** -25), np.float32(1))) == 1


def test_f16_to_f32_exhaustive():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = oracle.f16_to_f32_array(h)
    ref = h.view(np.float16).astype(np.float32)
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin].view(np.uint32), ref[fin].view(np.uint32))
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(np.isinf(got), np.isinf(ref))

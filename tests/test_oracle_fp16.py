"""Pins of the oracle's fp16 codec against numpy's IEEE binary16 conversions."""
import numpy as np

import oracle


def test_half_to_float_exhaustive():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = h.view(np.float16).astype(np.float32)
    got = oracle.half_to_float(h)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_float_to_half_against_numpy():
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 1 << 32, 2_000_000, dtype=np.uint64).astype(np.uint32)
    lo = np.float32(2.0 ** -27).view(np.uint32)
    hi = np.float32(66000.0).view(np.uint32)
    dense = np.arange(lo, hi, 1009, dtype=np.uint32)
    bits = np.concatenate([bits, dense, dense | np.uint32(0x80000000)])
    f = bits.view(np.float32)
    with np.errstate(over="ignore"):
        ref = f.astype(np.float16).view(np.uint16)
    got = oracle.float_to_half(f)
    nan = np.isnan(f)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.all((got[nan] & 0x7C00) == 0x7C00) and np.all((got[nan] & 0x3FF) != 0)


def test_float_to_half_special_cases():
    cases = {65504.0: 0x7BFF, 65519.99: 0x7BFF, 65520.0: 0x7C00, 2.0 ** -24: 0x0001,
             2.0 ** -25: 0x0000, 2.0 ** -25 * 1.0000001: 0x0001, 3 * 2.0 ** -25: 0x0002,
             2.0 ** -14: 0x0400, -0.0: 0x8000, float("inf"): 0x7C00, float("-inf"): 0xFC00,
             1.0 + 2.0 ** -11: 0x3C00, 1.0 + 3 * 2.0 ** -11: 0x3C02}
    for x, want in cases.items():
        assert int(oracle.float_to_half(np.array([x], dtype=np.float32))[0]) == want, x

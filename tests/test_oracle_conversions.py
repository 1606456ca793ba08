"""Pins for the oracle's IEEE conversions (fp32 -> fp16 / bf16 round-to-nearest-even,
fp16 / bf16 -> fp32).

The exported weights of the format are fp16 / bf16 roundings of a binary32
product, so these conversions decide bits.  The oracle writes them from the
IEEE 754 definitions; here they are checked against independent library
routines (numpy's float16 cast, torch's bfloat16 cast) over every binary32
input, plus hand-picked boundary cases.
"""
import os

import numpy as np
import pytest
import torch

import oracle

CHUNK = 1 << 26
EXHAUSTIVE = os.environ.get("SVQ_EXHAUSTIVE") == "1"


def _chunks():
    """Binary32 bit patterns to test.

    SVQ_EXHAUSTIVE=1: all 2^32 patterns (about ten minutes on 8 cores).
    Default: every sign and exponent combined with every pattern of the low 14
    mantissa bits (the bits that decide fp16 rounding of normal results, plus
    the even/odd bit) under four settings of the top 9 mantissa bits, then
    2^25 uniformly random patterns (about 40M inputs in all)."""
    if EXHAUSTIVE:
        for start in range(0, 1 << 32, CHUNK):
            yield np.arange(start, start + CHUNK, dtype=np.uint64).astype(np.uint32)
        return
    low = np.arange(1 << 14, dtype=np.uint32)
    r = np.random.Generator(np.random.PCG64(20261202))
    tops = np.array([0, 0x1FF, 0x100, 0x0FF], np.uint32)
    for se in range(512):                      # sign and 8-bit exponent
        hi = np.uint32(se) << np.uint32(23)
        t = np.concatenate([tops, r.integers(0, 512, 2, dtype=np.uint32)])
        yield (hi | (t[:, None] << np.uint32(14)) | low[None, :]).reshape(-1).astype(np.uint32)
    yield r.integers(0, 1 << 32, 1 << 25, dtype=np.uint64).astype(np.uint32)


def test_f16_to_f32_all_65536():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = oracle.h2f(bits)
    ref = bits.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_bf16_to_f32_all_65536():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    got = np.array([oracle.bf2f_scalar(int(b)) for b in bits], np.float32)
    r = ref
    nan = np.isnan(r)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), r[~nan].view(np.uint32))


def test_f32_to_f16_rne_exhaustive():
    """Binary32 patterns (see _chunks): oracle RNE == numpy's float16 cast (NaN -> NaN)."""
    for u in _chunks():
        x = u.view(np.float32)
        got = oracle.f2h_rne(x)
        with np.errstate(over="ignore"):
            ref = x.astype(np.float16).view(np.uint16)
        nan = np.isnan(x)
        if nan.any():
            gn = got[nan]
            assert np.all(((gn & 0x7C00) == 0x7C00) & ((gn & 0x3FF) != 0))
        ok = ~nan
        bad = np.nonzero(got[ok] != ref[ok])[0]
        assert bad.size == 0, f"first mismatch at {hex(int(u[ok][bad[0]]))}"


def test_f32_to_bf16_rne_exhaustive():
    """Binary32 patterns (see _chunks): oracle RNE == torch's bfloat16 cast (NaN -> NaN)."""
    for u in _chunks():
        x = u.view(np.float32)
        got = oracle.f2bf_rne(x)
        ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        nan = np.isnan(x)
        if nan.any():
            gn = got[nan]
            assert np.all(((gn & 0x7F80) == 0x7F80) & ((gn & 0x7F) != 0))
        ok = ~nan
        bad = np.nonzero(got[ok] != ref[ok])[0]
        assert bad.size == 0, f"first mismatch at {hex(int(u[ok][bad[0]]))}"


@pytest.mark.parametrize("x,bits", [
    (0.0, 0x0000), (-0.0, 0x8000), (1.0, 0x3C00), (65504.0, 0x7BFF),
    (65519.99, 0x7BFF), (65520.0, 0x7C00),            # tie at the top rounds to even = inf
    (2.0 ** -24, 0x0001), (2.0 ** -25, 0x0000),        # tie to even (0) at the bottom
    (1.5 * 2.0 ** -25, 0x0001), (2.0 ** -14, 0x0400),
    (1.0 + 2.0 ** -11, 0x3C00), (1.0 + 3 * 2.0 ** -11, 0x3C02),   # ties to even
    (0.35355339059327373, 0x35A8),
])
def test_f16_boundaries(x, bits):
    assert int(oracle.f2h_rne(np.array([x], np.float32))[0]) == bits

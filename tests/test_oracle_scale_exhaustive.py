"""Exhaustive pins of the oracle's block-scale rule over every block maximum a
bf16 block can have (every positive finite bf16 value, 32,639 of them).

Method: "NVIDIA NeMo RL erreicht 48% ..." section "Der technische
Durchbruch" (E4M3 blocks) and "FP8 Trainingsinfrastructuur" section "Het
landschap van numerieke precisie" (E4M3 up to +-448; E5M2 up to 57344);
the scale readings are s = fp32(amax / Q) (FP32 mode) and the smallest
power of two with amax <= Q * 2^e, clamped to [-127, 127] (POW2 mode).

Each FP32-mode scale is checked two independent ways: against numpy's IEEE
binary32 division, and against the definition of correct rounding (the
returned float is at least as close to amax/Q as both of its neighbours,
with every product formed exactly in fp64).  A scale computed as
amax * (1/Q), or rounded in another direction, fails both.  POW2-mode scales
are checked against the minimality property with exact fp64 arithmetic."""
import math

import numpy as np
import pytest

POS_BF16 = np.arange(0x0001, 0x7F80, dtype=np.uint32)          # +subnormals .. max finite
AMAX = (POS_BF16 << 16).view(np.float32)                         # every positive finite bf16


def _scales(orc, mode, fmt):
    return np.array([orc.block_scale_fmt(float(a), mode, fmt) for a in AMAX], np.float32)


@pytest.mark.parametrize("fmt,Q", [(0, 448.0), (1, 57344.0)])
def test_fp32_scale_is_ieee_division_for_every_bf16_amax(orc, fmt, Q):
    s = _scales(orc, orc.MODE_FP32, fmt)
    want = AMAX / np.float32(Q)                                  # IEEE binary32 division
    assert np.array_equal(s.view(np.uint32), want.view(np.uint32))
    # and it is the float nearest to amax/Q: compare |s*Q - amax| (exact in
    # fp64: 24-bit s times Q = 7*2^6 or 7*2^13) with both neighbours
    up = np.nextafter(s, np.float32(np.inf))
    dn = np.nextafter(s, np.float32(0))
    a = AMAX.astype(np.float64)
    err = np.abs(s.astype(np.float64) * Q - a)
    assert np.all(err <= np.abs(up.astype(np.float64) * Q - a))
    assert np.all(err <= np.abs(dn.astype(np.float64) * Q - a))
    # a reciprocal-multiply implementation would differ somewhere
    recip = AMAX * (np.float32(1.0) / np.float32(Q))
    assert not np.array_equal(recip.view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("fmt,Q", [(0, 448.0), (1, 57344.0)])
def test_pow2_scale_is_minimal_power_for_every_bf16_amax(orc, fmt, Q):
    s = _scales(orc, orc.MODE_POW2, fmt).astype(np.float64)
    e = np.array([math.frexp(v)[1] - 1 for v in s])
    assert np.all(s == np.ldexp(1.0, e))                         # exact powers of two
    assert np.all((e >= -127) & (e <= 127))
    a = AMAX.astype(np.float64)
    assert np.all(a <= Q * s)                                    # nothing saturates
    # minimal: the next smaller power would saturate, unless clamped
    assert np.all((a > Q * s / 2) | (e == -127))
    # the clamp engages exactly where 448 * 2^-127 would still be too large
    assert np.all((e == -127) == (a <= Q * 2.0 ** -127))

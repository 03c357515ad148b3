"""Pins for the oracle's E4M3 codec and block-scale rule (CPU only).

What fixes them (page titles, sections):
  * "FP8 Trainingsinfrastructuur", "Het landschap van numerieke precisie":
    E4M3 has 4 exponent bits, 3 mantissa bits and a largest value of 448.
  * "NVIDIA NeMo RL erreicht 48% ...", "Der technische Durchbruch": the
    recipe's tensors are E4M3; "Warum dies für die KI-Ökonomie wichtig ist":
    optional power-of-2 scale factors.
The checks below are independent of the oracle's own code: an exhaustive
round trip over all 256 codes, a brute-force nearest-value search written
here, two library conversions (torch, ml_dtypes), hand-worked points
(tests/golden/e4m3_points.txt) and closed forms.
"""
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_points.txt")


def _table(orc):
    return np.array([orc.e4m3_decode(c) for c in range(256)], dtype=np.float64)


def test_code_table_shape(orc):
    t = _table(orc)
    nan = np.isnan(t)
    assert sorted(np.nonzero(nan)[0].tolist()) == [0x7F, 0xFF]
    finite = t[~nan]
    assert finite.size == 254
    assert finite.max() == 448.0 and finite.min() == -448.0
    pos = t[:0x7F]
    assert np.all(np.diff(pos) > 0), "positive codes must be strictly increasing"
    assert pos[1] == 2.0 ** -9          # smallest subnormal
    assert pos[8] == 2.0 ** -6          # smallest normal
    assert pos[7] == 7 * 2.0 ** -9      # largest subnormal
    assert math.copysign(1.0, t[0x80]) == -1.0 and t[0x80] == 0.0
    # sign symmetry
    for c in range(0x7F):
        assert t[c | 0x80] == -t[c]


def test_decode_matches_libraries(orc):
    t = _table(orc)
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    tt = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    both_nan = np.isnan(t) & np.isnan(tt)
    assert np.all(both_nan | (t == tt))
    ml = pytest.importorskip("ml_dtypes")
    mt = np.arange(256, dtype=np.uint8).view(ml.float8_e4m3fn).astype(np.float64)
    assert np.all((np.isnan(t) & np.isnan(mt)) | (t == mt))


def test_round_trip_all_codes(orc):
    for c in range(256):
        v = orc.e4m3_decode(c)
        if math.isnan(v):
            continue
        assert orc.e4m3_encode(v) == c, hex(c)


def _brute_nearest(v, table):
    """Nearest finite E4M3 code to v, ties to the even mantissa, saturating."""
    pos = table[:0x7F]
    a = abs(v)
    sign = 0x80 if math.copysign(1.0, v) < 0 else 0
    if a >= 448.0:
        return sign | 0x7E
    d = np.abs(pos - a)
    best = d.min()
    cands = np.nonzero(d == best)[0]
    if cands.size == 2:
        c = int(cands[0] if cands[0] % 2 == 0 else cands[1])
    else:
        c = int(cands[0])
    return sign | c


def test_encode_brute_force_midpoints(orc):
    t = _table(orc)
    pos = t[:0x7F]
    vals = []
    for i in range(pos.size - 1):
        lo, hi = pos[i], pos[i + 1]
        mid = (lo + hi) / 2
        vals += [lo, hi, mid, np.nextafter(np.float32(mid), np.float32(0)),
                 np.nextafter(np.float32(mid), np.float32(1e9))]
    vals = np.array(vals, dtype=np.float32)
    vals = np.concatenate([vals, -vals])
    got = orc.e4m3_encode_array(vals)
    want = np.array([_brute_nearest(float(v), t) for v in vals], np.uint8)
    np.testing.assert_array_equal(got, want)


def test_encode_brute_force_random(orc):
    t = _table(orc)
    rng = np.random.default_rng(1234)
    e = rng.uniform(-14, 9.5, 4000)
    v = (np.sign(rng.standard_normal(4000)) * 2.0 ** e).astype(np.float32)
    got = orc.e4m3_encode_array(v)
    want = np.array([_brute_nearest(float(x), t) for x in v], np.uint8)
    np.testing.assert_array_equal(got, want)


def test_encode_matches_torch_and_ml_dtypes_in_range(orc):
    # Inside the finite range both libraries round to nearest, ties to even.
    rng = np.random.default_rng(7)
    e = rng.uniform(-20, 8.7, 200000)
    v = (rng.choice([-1.0, 1.0], e.size) * 2.0 ** e).astype(np.float32)
    v = v[np.abs(v) < 448.0]
    got = orc.e4m3_encode_array(v)
    tv = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(got, tv)
    ml = pytest.importorskip("ml_dtypes")
    mv = v.astype(ml.float8_e4m3fn).view(np.uint8)
    np.testing.assert_array_equal(got, mv)


def test_saturation(orc):
    for v in [448.0, 448.5, 463.9, 464.0, 480.0, 1e6, 3.0e38]:
        assert orc.e4m3_encode(v) == 0x7E
        assert orc.e4m3_encode(-v) == 0xFE


def test_golden_points(orc):
    n = 0
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            val, code = line.split()[:2]
            assert orc.e4m3_encode(float(val)) == int(code, 16), line
            n += 1
    assert n >= 20


# ------------------------------------------------------------ block scale --
def test_scale_fp32_closed_forms(orc):
    assert orc.block_scale(448.0, 0) == 1.0
    assert orc.block_scale(224.0, 0) == 0.5
    assert orc.block_scale(7.0, 0) == 2.0 ** -6
    assert orc.block_scale(0.0, 0) == 1.0
    # amax / s lands within a few fp32 ulps of 448 for ordinary amax
    rng = np.random.default_rng(3)
    for a in rng.uniform(1e-3, 1e3, 2000).astype(np.float32):
        s = np.float32(orc.block_scale(float(a), 0))
        assert abs(float(np.float32(a) / s) - 448.0) <= 448.0 * 2 ** -22


def _pow2_closed_form(amax):
    # amax = m * 2^E with m in [1,2): smallest e with amax <= 1.75 * 2^(8+e)
    f, E2 = math.frexp(amax)
    m, E = 2 * f, E2 - 1
    e = E - 8 + (1 if m > 1.75 else 0)
    return 2.0 ** max(-127, min(127, e))


def test_scale_pow2_closed_form(orc):
    rng = np.random.default_rng(5)
    vals = list((2.0 ** rng.uniform(-130, 127, 5000)).astype(np.float32))
    vals += [448.0, 448.0 * 1.0000001, 224.0, 1.75, 1.7500001, 3.5, 1e-40, 1e-45, 3.0e38]
    for a in vals:
        a = float(np.float32(a))
        if a == 0.0:
            continue
        s = orc.block_scale(a, 1)
        assert s == _pow2_closed_form(a), a
        # exact power of two: zero mantissa bits
        bits = np.array([s], np.float32).view(np.uint32)[0]
        if s >= 2.0 ** -126:
            assert bits & 0x7FFFFF == 0
        if 2.0 ** -100 < a < 2.0 ** 100:
            r = a / s
            assert 224.0 < r <= 448.0, (a, s)
    assert orc.block_scale(0.0, 1) == 1.0
    assert orc.block_scale(1e-45, 1) == 2.0 ** -127   # clamped


def test_bf16_ulp(orc):
    assert orc.bf16_ulp(1.0) == 2.0 ** -7
    assert orc.bf16_ulp(1.99) == 2.0 ** -7
    assert orc.bf16_ulp(2.0) == 2.0 ** -6
    assert orc.bf16_ulp(-0.75) == 2.0 ** -8
    assert orc.bf16_ulp(0.0) == 2.0 ** -133
    # agrees with torch's bf16 spacing
    for v in [3.7, 1000.0, 1e-3, 123456.0]:
        b = torch.tensor([v], dtype=torch.bfloat16)
        nxt = torch.nextafter(b.float(), torch.tensor([1e30])).to(torch.bfloat16)
        # nextafter in fp32 then rounding lands on b; step bf16 directly instead
        u = b.view(torch.int16) + 1
        gap = u.view(torch.bfloat16).double() - b.double()
        assert orc.bf16_ulp(float(b.double())) == float(gap), v
        del nxt

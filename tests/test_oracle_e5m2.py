"""Pins of the oracle's E5M2 codec and of the E5M2 paths of its quantizer and
GEMM reference (CPU only).

E5M2 is the gradient format of the per-tensor recipe on "FP8
Trainingsinfrastructuur: Numerieke Precisie van de Volgende Generatie",
section "Het landschap van numerieke precisie" (5 exponent bits, 2 mantissa
bits).  With an exponent bias of 15 its largest finite value is
1.75 * 2^15 = 57344, exponent field 31 holds the infinities (mantissa 0) and
NaN, and subnormals are m * 2^-16."""
import numpy as np
import pytest
import torch

import oracle as orc


def table():
    return np.array([orc.e5m2_decode(c) for c in range(256)])


def test_code_table():
    t = table()
    assert np.isnan(t).sum() == 6                      # 0x7D-0x7F and 0xFD-0xFF
    assert np.isinf(t).sum() == 2 and t[0x7C] == np.inf and t[0xFC] == -np.inf
    assert t[0x7B] == 57344.0 and t[0xFB] == -57344.0
    assert t[0x04] == 2.0 ** -14 and t[0x01] == 2.0 ** -16 and t[0x03] == 3 * 2.0 ** -16
    assert t[0x3C] == 1.0 and t[0x42] == 3.0 and t[0x80] == 0.0 and np.signbit(t[0x80])
    fin = t[np.isfinite(t)]
    assert len(np.unique(fin)) == 247                  # 248 finite codes, +-0 equal


def test_decode_matches_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e5m2).double().numpy()
    t = table()
    same = (t == ref) | (np.isnan(t) & np.isnan(ref))
    assert same.all()


def test_round_trip_all_codes():
    t = table()
    for c in range(256):
        v = t[c]
        if np.isnan(v):
            assert orc.e5m2_encode(np.float32(v)) & 0x7F == 0x7F
        elif np.isinf(v):
            assert orc.e5m2_encode(np.float32(v)) == (c & 0x80) | 0x7B   # saturates
        else:
            assert orc.e5m2_encode(np.float32(v)) == c, hex(c)


def test_midpoints_tie_to_even():
    t = table()
    pos = sorted((t[c], c) for c in range(0x7C))       # finite non-negative codes
    for (a, ca), (b, cb) in zip(pos, pos[1:]):
        mid = np.float32((a + b) / 2)
        even = ca if ca % 2 == 0 else cb
        assert orc.e5m2_encode(mid) == even, (a, b)
        lo, hi = np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(1e9))
        assert orc.e5m2_encode(lo) == ca and orc.e5m2_encode(hi) == cb


def test_encode_matches_torch_in_range():
    rng = np.random.default_rng(7)
    v = (rng.standard_normal(200000) * 10.0 ** rng.uniform(-6, 4, 200000)).astype(np.float32)
    v = v[np.abs(v) <= 57344]
    ours = orc.e5m2_encode_array(v)
    ref = torch.from_numpy(v).to(torch.float8_e5m2).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_saturation():
    for v, c in [(57344.0, 0x7B), (61439.0, 0x7B), (1e30, 0x7B), (-1e30, 0xFB), (np.inf, 0x7B)]:
        assert orc.e5m2_encode(np.float32(v)) == c


def test_scale_closed_forms():
    assert orc.block_scale_fmt(57344.0, orc.MODE_FP32, orc.FMT_E5M2) == 1.0
    assert orc.block_scale_fmt(0.0, orc.MODE_FP32, orc.FMT_E5M2) == 1.0
    rng = np.random.default_rng(3)
    for a in (2.0 ** rng.uniform(-60, 60, 3000)).astype(np.float32):
        assert orc.block_scale_fmt(a, orc.MODE_FP32, orc.FMT_E5M2) == np.float32(a) / np.float32(57344.0)
        m, E = np.frexp(np.float64(a))                 # a = m 2^E, m in [0.5, 1)
        e = int(E - 1 - 15 + (2 * m > 1.75))
        e = max(-127, min(127, e))
        assert orc.block_scale_fmt(a, orc.MODE_POW2, orc.FMT_E5M2) == np.float32(2.0 ** e)
    # the E4M3 rule is unchanged by the format argument
    assert orc.block_scale_fmt(448.0, orc.MODE_FP32, orc.FMT_E4M3) == orc.block_scale(448.0, orc.MODE_FP32)


def bits(x):
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


def test_hand_worked_block():
    # one 1x128 block with amax 57344: s = 1 and each code is the plain encoding
    x = torch.zeros((128, 128), dtype=torch.bfloat16)
    x[0, 0], x[0, 1], x[0, 2], x[0, 3] = 57344.0, 3.0, -1.0, 2.0 ** -15
    q, s, qc, sc = orc.quant_act_1x128(bits(x), orc.MODE_FP32, fmt=orc.FMT_E5M2)
    assert s[0, 0] == 1.0
    assert list(q[0, :4]) == [0x7B, 0x42, 0xBC, 0x02]
    # POW2 with amax 3: the smallest e with 3 <= 57344 * 2^e is -14
    y = torch.zeros((128, 128), dtype=torch.bfloat16)
    y[5, 7] = 3.0
    q, s, _, _ = orc.quant_act_1x128(bits(y), orc.MODE_POW2, fmt=orc.FMT_E5M2)
    assert s[0, 5] == 2.0 ** -14 and orc.e5m2_decode(int(q[5, 7])) == 3.0 * 2 ** 14


def test_gemm_reference_with_e5m2_operand():
    rng = np.random.default_rng(11)
    M, N, K = 128, 256, 256
    t5, t4 = table(), np.array([orc.e4m3_decode(c) for c in range(256)])
    A = rng.integers(0, 0x7B, (M, K), dtype=np.uint8) | (rng.integers(0, 2, (M, K), dtype=np.uint8) << 7)
    B = rng.integers(0, 0x7E, (N, K), dtype=np.uint8)
    sA = (2.0 ** rng.uniform(-20, 0, (K // 128, M))).astype(np.float32)
    sB = (2.0 ** rng.uniform(-5, 0, (N // 128, K // 128))).astype(np.float32)
    y, ya = orc.gemm_ref_tile(0, A, sA, B, sB, 0, M, 0, N, fa=orc.FMT_E5M2, fb=orc.FMT_E4M3)
    a = t5[A] * np.repeat(sA.T.astype(np.float64), 128, axis=1)
    b = t4[B] * np.repeat(np.repeat(sB.astype(np.float64), 128, axis=0), 128, axis=1)
    yabs = np.abs(a) @ np.abs(b).T
    np.testing.assert_allclose(ya, yabs, rtol=1e-12, atol=0)
    assert np.all(np.abs(y - a @ b.T) <= 1e-12 * yabs)   # fp64 summation order only
    # the E4M3 reading of the same bytes differs: the format argument is used
    y4, _ = orc.gemm_ref_tile(0, A, sA, B, sB, 0, M, 0, N)
    assert not np.allclose(y4, y)

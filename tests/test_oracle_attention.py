"""Pins of the oracle's FP8 attention forward reference (CPU only).

Method: "NVIDIA NeMo RL erreicht 48% ..." section "Leistungsgewinne in der
Praxis": the recipe extends FP8 to the KV cache and the attention
operations.  The readings (1x128 blocks along each contraction, P's block
scale by the FP32 rule, softmax normalizer from the unquantized numerator)
are stated in oracle.cpp.  Each pin below holds by construction or by the
mathematics, independently of the oracle's code: closed forms, an
independent brute force built on torch's own E4M3 cast, and invariants."""
import math

import numpy as np
import pytest
import torch

D = 128


def quant_rows(x, orc, mode=0):
    """1x128 row blocks (per token and head) with the oracle's quantizer."""
    q, s, _, _ = orc.quant_act_1x128(x.view(torch.int16).numpy().view(np.uint16), mode, colwise=False)
    return q, s


def quant_v(x, orc, mode=0):
    """V's column-wise copy: codes [H*128, T], scales [T/128, H*128]."""
    _, _, qc, sc = orc.quant_act_1x128(x.view(torch.int16).numpy().view(np.uint16), mode)
    return qc, sc


def make_case(orc, T, Hq, Hkv, seed, qscale=1.0, mode=0):
    g = torch.Generator().manual_seed(seed)
    Q = (torch.randn((T, Hq * D), generator=g) * qscale).to(torch.bfloat16)
    K = torch.randn((T, Hkv * D), generator=g).to(torch.bfloat16)
    V = torch.randn((T, Hkv * D), generator=g).to(torch.bfloat16)
    q, sq = quant_rows(Q, orc, mode)
    k, sk = quant_rows(K, orc, mode)
    vT, sv = quant_v(V, orc, mode)
    return q, sq, k, sk, vT, sv


def e4m3_decode_torch(codes):
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def pow2_scale(amax):
    """Power-of-2 rule by frexp: amax / 448 = m 2^x with m in [0.5, 1); the
    smallest power of two at or above it is 2^(x-1) when m == 0.5, else 2^x."""
    m, x = math.frexp(amax / 448.0)
    return math.ldexp(1.0, x - 1 if m == 0.5 else x)


def brute_force(q, sq, k, sk, vT, sv, Hq, Hkv, off, ln, causal, t, h, mode=0):
    """Independent restatement: torch's E4M3 decode and cast, numpy softmax.
    mode 1: p against the integer power-of-two reference ceil(max z log2 e)
    and power-of-2 block scales."""
    T = q.shape[0]
    g = h // (Hq // Hkv)
    seg = max(i for i in range(len(ln)) if off[i] <= t)
    j0, jr = off[seg], off[seg] + ln[seg]
    if t >= jr:
        return np.zeros(D)
    j1 = t + 1 if causal else jr
    qv = e4m3_decode_torch(q[t, h * D:(h + 1) * D]) * sq[h, t]
    kv = e4m3_decode_torch(k[j0:j1, g * D:(g + 1) * D]) * sk[g, j0:j1][:, None]
    z = kv @ qv / math.sqrt(D)
    if mode == 1:
        y = z / math.log(2.0)
        p = np.exp2(y - math.ceil(y.max()))
    else:
        p = np.exp(z - z.max())
    l = p.sum()
    vv = e4m3_decode_torch(vT[g * D:(g + 1) * D, j0:j1]).T * sv[np.arange(j0, j1) // 128, g * D:(g + 1) * D]
    o = np.zeros(D)
    for b0 in range((j0 // 128) * 128, j1, 128):
        lo, hi = max(b0, j0), min(b0 + 128, j1)
        pb = p[lo - j0:hi - j0]
        s = pow2_scale(pb.max()) if mode == 1 else pb.max() / 448.0
        codes = torch.from_numpy((pb / s).astype(np.float32)).to(torch.float8_e4m3fn)
        phat = codes.to(torch.float64).numpy() * s
        o += phat @ vv[lo - j0:hi - j0]
    return o / l


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("causal", [True, False])
def test_brute_force_tiny(orc, causal, mode):
    Hq, Hkv, T = 4, 2, 512
    q, sq, k, sk, vT, sv = make_case(orc, T, Hq, Hkv, 3, mode=mode)
    off, ln = [0, 256, 512], [200, 256]          # a padded segment and a full one
    rows = [(t, h) for t in (0, 1, 77, 128, 199, 200, 255, 256, 300, 511) for h in range(Hq)]
    rt = [r[0] for r in rows]
    rh = [r[1] for r in rows]
    O, oa, of = orc.attention_fwd_rows(q, sq, k, sk, vT, sv, Hq, Hkv, off, ln, causal, rt, rh, mode)
    for i, (t, h) in enumerate(rows):
        ref = brute_force(q, sq, k, sk, vT, sv, Hq, Hkv, off, ln, causal, t, h, mode)
        np.testing.assert_allclose(O[i], ref, rtol=0, atol=1e-12 * (1 + oa[i].max()))
    # padding query rows are zero
    pad = [i for i, (t, _) in enumerate(rows) if 200 <= t < 256]
    assert np.all(O[pad] == 0)


def test_single_key_is_v(orc):
    """The first causal row sees one key: p = 1, its block amax maps to 448
    exactly (code 0x7E, p^ = 1), so O equals that key's dequantized V."""
    q, sq, k, sk, vT, sv = make_case(orc, 128, 1, 1, 5)
    O, _, of = orc.attention_fwd_rows(q, sq, k, sk, vT, sv, 1, 1, [0, 128], [128], True, [0], [0])
    vhat = np.array([orc.e4m3_decode(c) for c in vT[:, 0]]) * sv[0, :]
    assert np.array_equal(O[0], vhat)
    assert np.all(of == 0)


def test_identical_keys_average_v(orc):
    """All keys equal: every logit equal, p = 1 everywhere, O = mean of V^."""
    T = 256
    q, sq, k, sk, vT, sv = make_case(orc, T, 1, 1, 6)
    k[:] = k[0]
    sk[:] = sk[:, :1]
    O, _, _ = orc.attention_fwd_rows(q, sq, k, sk, vT, sv, 1, 1, [0, T], [T], False, [5, 200], [0, 0])
    dec = np.array([orc.e4m3_decode(c) for c in range(256)])
    vhat = dec[vT].T * sv[np.arange(T) // 128]
    for i in range(2):
        np.testing.assert_allclose(O[i], vhat.mean(axis=0), rtol=1e-13, atol=1e-15)


def test_dominating_key(orc):
    """One key's logit exceeds the others' by 60: their p / s = 448 e^-60 is
    far below the smallest E4M3 step, so they quantize to 0 and O is that
    key's V^ exactly."""
    T = 128
    q, sq, k, sk, vT, sv = make_case(orc, T, 1, 1, 7)
    k[:] = k[0]
    sk[:] = sk[:, :1]
    dec = np.array([orc.e4m3_decode(c) for c in range(256)])
    zb = (dec[q[9]] * sq[0, 9]) @ (dec[k[0]] * float(sk[0, 0])) / math.sqrt(D)
    sk[0, 40] = np.float32(sk[0, 0] * (1 + 60.0 / zb))     # z_40 = z_b + 60
    O, _, _ = orc.attention_fwd_rows(q, sq, k, sk, vT, sv, 1, 1, [0, T], [T], False, [9], [0])
    vhat = dec[vT[:, 40]] * sv[0]
    np.testing.assert_allclose(O[0], vhat, rtol=1e-12, atol=0)


def test_block_below_the_scale_range(orc):
    """A 128-key block far below the row's maximum: one key at e^-745 (p the
    smallest subnormal double), the others at e^-800 (p = 0), so amax / 448
    underflows to zero.  That block counts as all-zero (scale 1, every code
    0), as it does in fp32, where all its p are exactly 0; dividing its
    zero p by the underflowed scale would give 0/0.  Closed form: the other
    block holds the one key with p = 1 (code 0x7E against s = 1/448, p^ = 1)
    and keys at e^-745, so O = that key's V^ exactly."""
    T = 256
    dec = np.array([orc.e4m3_decode(c) for c in range(256)])
    one, m_one, two = 0x38, 0xB8, 0x40                  # E4M3 codes of 1, -1, 2
    assert (dec[one], dec[m_one], dec[two]) == (1.0, -1.0, 2.0)
    q = np.full((T, D), one, np.uint8)
    sq = np.full((1, T), 1.0 / 128, np.float32)          # q^ . k^ s_q = k^: z_j = k^_j s_kj / sqrt(128)
    k = np.full((T, D), m_one, np.uint8)
    sk = np.full((1, T), np.float32(745.0 * math.sqrt(D)), np.float32)   # z_j ~ -745
    sk[0, 1:128] = np.float32(800.0 * math.sqrt(D))     # z_j ~ -800: p = 0 in double
    k[128] = one
    sk[0, 128] = np.float32(1e-3)                         # z_128 ~ 0: the row's maximum
    vT = np.full((D, T), one, np.uint8)
    vT[:, 128] = two
    sv = np.ones((T // 128, D), np.float32)
    O, oa, of = orc.attention_fwd_rows(q, sq, k, sk, vT, sv, 1, 1, [0, T], [T], False, [3], [0])
    assert np.all(np.isfinite(O)) and np.all(np.isfinite(oa)) and np.all(np.isfinite(of))
    assert np.array_equal(O[0], np.full(D, 2.0))


def test_gqa_equals_replicated_heads(orc):
    Hq, Hkv, T = 4, 2, 256
    q, sq, k, sk, vT, sv = make_case(orc, T, Hq, Hkv, 8)
    # replicate each KV head for its two query heads
    rep = [0, 0, 1, 1]
    k4 = np.concatenate([k[:, g * D:(g + 1) * D] for g in rep], axis=1)
    sk4 = sk[rep]
    vT4 = np.concatenate([vT[g * D:(g + 1) * D] for g in rep], axis=0)
    sv4 = np.concatenate([sv[:, g * D:(g + 1) * D] for g in rep], axis=1)
    rt, rh = [3, 100, 255, 3], [0, 1, 2, 3]
    a = orc.attention_fwd_rows(q, sq, k, sk, vT, sv, Hq, Hkv, [0, T], [T], True, rt, rh)
    b = orc.attention_fwd_rows(q, sq, k4, sk4, vT4, sv4, Hq, Hq, [0, T], [T], True, rt, rh)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_causal_ignores_later_keys(orc):
    T = 384
    q, sq, k, sk, vT, sv = make_case(orc, T, 1, 1, 9)
    rt, rh = [10, 130, 200], [0, 0, 0]
    a, _, _ = orc.attention_fwd_rows(q, sq, k, sk, vT, sv, 1, 1, [0, T], [T], True, rt, rh)
    k2, vT2 = k.copy(), vT.copy()
    k2[201:] = 0x38
    vT2[:, 201:] = 0x38
    b, _, _ = orc.attention_fwd_rows(q, sq, k2, sk, vT2, sv, 1, 1, [0, T], [T], True, rt, rh)
    assert np.array_equal(a, b)
    c, _, _ = orc.attention_fwd_rows(q, sq, k2, sk, vT2, sv, 1, 1, [0, T], [T], False, rt, rh)
    d, _, _ = orc.attention_fwd_rows(q, sq, k, sk, vT, sv, 1, 1, [0, T], [T], False, rt, rh)
    assert not np.array_equal(c, d)


def test_packed_segments_are_independent(orc):
    """Two sequences packed into one batch give each sequence's own result."""
    q, sq, k, sk, vT, sv = make_case(orc, 512, 2, 1, 10)
    off, ln = [0, 256, 512], [180, 256]
    rt, rh = [0, 150, 179, 256, 400, 511], [0, 1, 0, 1, 0, 1]
    both, _, _ = orc.attention_fwd_rows(q, sq, k, sk, vT, sv, 2, 1, off, ln, True, rt, rh)
    first, _, _ = orc.attention_fwd_rows(q[:256], sq[:, :256], k[:256], sk[:, :256],
                                         np.ascontiguousarray(vT[:, :256]), sv[:2], 2, 1,
                                         [0, 256], [180], True, rt[:3], rh[:3])
    second, _, _ = orc.attention_fwd_rows(q[256:], sq[:, 256:], k[256:], sk[:, 256:],
                                          np.ascontiguousarray(vT[:, 256:]), sv[2:], 2, 1,
                                          [0, 256], [256], True, [t - 256 for t in rt[3:]], rh[3:])
    assert np.array_equal(both[:3], first) and np.array_equal(both[3:], second)


def test_flip_allowance_marks_midpoints(orc):
    """A key whose p / s sits on the E4M3 midpoint between 416 and 448 (432,
    i.e. p = 432/448 of the block maximum) is ambiguous: either code is a
    correct rounding for a kernel whose p carries fp32 error, and the oracle
    adds one E4M3 step (32 * s * |v^|) to the allowance; moved off the
    midpoint it adds nothing."""
    T = 128
    q, sq, k, sk, vT, sv = make_case(orc, T, 1, 1, 11)
    k[:] = k[0]
    sk[:] = sk[:, :1]
    dec = np.array([orc.e4m3_decode(c) for c in range(256)])
    zq = (dec[q[0]] * sq[0, 0]) @ (dec[k[0]] * float(sk[0, 0])) / math.sqrt(D)
    # key 1's logit is z + ln(432/448): p_1 / s = 432 up to the fp32 scale
    sk[0, 1] = np.float32(sk[0, 0] * (1 + math.log(432.0 / 448.0) / zq))
    O, oa, of = orc.attention_fwd_rows(q, sq, k, sk, vT, sv, 1, 1, [0, T], [T], False, [0], [0])
    z = (dec[q[0]] * sq[0, 0]) @ (dec[k] * sk[0][:, None]).T / math.sqrt(D)
    p = np.exp(z - z.max())
    assert abs(p[1] / p.max() * 448.0 - 432.0) < 1e-3
    vhat1 = dec[vT[:, 1]] * sv[0]
    np.testing.assert_allclose(of[0], 32.0 * (p.max() / 448.0) * np.abs(vhat1) / p.sum(), rtol=1e-9)
    # off the midpoint: no allowance
    sk[0, 1] = np.float32(sk[0, 0] * (1 + math.log(420.0 / 448.0) / zq))
    _, _, of1 = orc.attention_fwd_rows(q, sq, k, sk, vT, sv, 1, 1, [0, T], [T], False, [0], [0])
    assert np.all(of1 == 0)


def test_single_key_pow2_closed_form(orc):
    """Power-of-2 mode, one key: p = 2^(y - ceil(y)) with y = z log2 e, so
    p lies in (1/2, 1]; its block scale is 2^-8 for p > 448 2^-9 = 0.875 and
    2^-9 otherwise, and O = v^ * E4M3(p / s) * s / p."""
    for seed in range(12, 20):
        q, sq, k, sk, vT, sv = make_case(orc, 128, 1, 1, seed, mode=1)
        O, _, _ = orc.attention_fwd_rows(q, sq, k, sk, vT, sv, 1, 1, [0, 128], [128], True, [0], [0], 1)
        dec = np.array([orc.e4m3_decode(c) for c in range(256)])
        z = float((dec[q[0]] * sq[0, 0]) @ (dec[k[0]] * sk[0, 0])) / math.sqrt(D)
        y = z / math.log(2.0)
        p = 2.0 ** (y - math.ceil(y))
        s = 2.0 ** -8 if p > 0.875 else 2.0 ** -9
        code = torch.tensor([p / s], dtype=torch.float32).to(torch.float8_e4m3fn).to(torch.float64).item()
        vhat = dec[vT[:, 0]] * sv[0, :]
        np.testing.assert_allclose(O[0], vhat * (code * s / p), rtol=1e-13, atol=0)


def _pow2_row(orc, seed, targets):
    """One causal row (t = len(targets) - 1) of a power-of-2 case whose key
    logits are placed, through the key scales, so that key i has
    p_i = targets[i] (p against the integer reference of the largest).  The
    keys repeat the query's codes, so every product of the dot product is
    positive and the oracle's logit error bound (and with it the midpoint
    allowance) stays near 1e-4 relative."""
    T = 128
    q, sq, k, sk, vT, sv = make_case(orc, T, 1, 1, seed, mode=1)
    dec = np.array([orc.e4m3_decode(c) for c in range(256)])
    t = len(targets) - 1
    k[:t + 1] = q[t]      # every product of the dot product positive: tight logit error bounds
    qk = float((dec[q[t]] * sq[0, t]) @ dec[k[0]]) / math.sqrt(D) / math.log(2.0)   # y per unit key scale
    top = 5.0 + math.log2(max(targets))          # ceil(top) = 5: reference 2^5
    for i, pt in enumerate(targets):
        sk[0, i] = np.float32((5.0 + math.log2(pt)) / qk)
    O, oa, of = orc.attention_fwd_rows(q, sq, k, sk, vT, sv, 1, 1, [0, T], [T], True, [t], [0], 1)
    y = np.array([qk * float(sk[0, i]) for i in range(t + 1)])
    p = 2.0 ** (y - math.ceil(y.max()))
    vhat = dec[vT[:, :t + 1]].T * sv[0][None, :]
    assert math.ceil(top) == 5
    return O[0], of[0], p, vhat


def test_pow2_boundary_single_key(orc):
    """Power-of-2 mode, one key with p = 448 2^-9 = 0.875 (to fp32 accuracy):
    amax / 448 sits on the boundary between the scales 2^-9 and 2^-8, and a
    kernel's fp32 p may pick either; both codes (448 under 2^-9, 224 under
    2^-8) decode to 0.875, so the allowance is 0 and O = v^ 0.875 / p."""
    O, of, p, vhat = _pow2_row(orc, 21, [0.875])
    assert abs(p[0] / 0.875 - 1) < 1e-6
    assert np.all(of == 0)
    np.testing.assert_allclose(O, vhat[0] * 0.875 / p[0], rtol=1e-12, atol=0)


def test_pow2_boundary_subnormal_allowance(orc):
    """Power-of-2 mode, two keys: the block maximum p_0 = 0.875 sits on a
    scale boundary and p_1 = 4.6 2^-18 is tiny.  Under 2^-9, p_1 / s = 4.6
    2^-9 is an E4M3 subnormal and rounds to 5 2^-9; under 2^-8 it is 2.3 2^-9
    and rounds to 2 2^-9.  The dequantized values differ by 2^-18, and the
    allowance of output channel d is that difference times |v^_1[d]| / l."""
    O, of, p, vhat = _pow2_row(orc, 23, [0.875, 4.6 * 2.0 ** -18])
    assert abs(p[0] / 0.875 - 1) < 1e-6 and abs(p[1] / (4.6 * 2.0 ** -18) - 1) < 1e-5
    np.testing.assert_allclose(of, 2.0 ** -18 * np.abs(vhat[1]) / p.sum(), rtol=1e-9, atol=0)


@pytest.mark.parametrize("mode", [0, 1])
def test_gqa_and_causality_both_modes(orc, mode):
    """GQA equals replicated KV heads, and causal rows ignore later keys, in
    either scale mode."""
    Hq, Hkv, T = 4, 2, 256
    q, sq, k, sk, vT, sv = make_case(orc, T, Hq, Hkv, 22, mode=mode)
    rep = [0, 0, 1, 1]
    k4 = np.concatenate([k[:, g * D:(g + 1) * D] for g in rep], axis=1)
    vT4 = np.concatenate([vT[g * D:(g + 1) * D] for g in rep], axis=0)
    sv4 = np.concatenate([sv[:, g * D:(g + 1) * D] for g in rep], axis=1)
    rt, rh = [3, 100, 255, 3], [0, 1, 2, 3]
    a = orc.attention_fwd_rows(q, sq, k, sk, vT, sv, Hq, Hkv, [0, T], [T], True, rt, rh, mode)
    b = orc.attention_fwd_rows(q, sq, k4, sk[rep], vT4, sv4, Hq, Hq, [0, T], [T], True, rt, rh, mode)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    k2, vT2 = k.copy(), vT.copy()
    k2[101:] = 0x38
    vT2[:, 101:] = 0x38
    c = orc.attention_fwd_rows(q, sq, k2, sk, vT2, sv, Hq, Hkv, [0, T], [T], True, [3, 100], [0, 1], mode)
    assert np.array_equal(c[0], a[0][:2])

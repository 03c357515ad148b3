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


def quant_rows(x, orc):
    """1x128 row blocks (per token and head) with the oracle's quantizer."""
    q, s, _, _ = orc.quant_act_1x128(x.view(torch.int16).numpy().view(np.uint16), 0, colwise=False)
    return q, s


def quant_v(x, orc):
    """V's column-wise copy: codes [H*128, T], scales [T/128, H*128]."""
    _, _, qc, sc = orc.quant_act_1x128(x.view(torch.int16).numpy().view(np.uint16), 0)
    return qc, sc


def make_case(orc, T, Hq, Hkv, seed, qscale=1.0):
    g = torch.Generator().manual_seed(seed)
    Q = (torch.randn((T, Hq * D), generator=g) * qscale).to(torch.bfloat16)
    K = torch.randn((T, Hkv * D), generator=g).to(torch.bfloat16)
    V = torch.randn((T, Hkv * D), generator=g).to(torch.bfloat16)
    q, sq = quant_rows(Q, orc)
    k, sk = quant_rows(K, orc)
    vT, sv = quant_v(V, orc)
    return q, sq, k, sk, vT, sv


def e4m3_decode_torch(codes):
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def brute_force(q, sq, k, sk, vT, sv, Hq, Hkv, off, ln, causal, t, h):
    """Independent restatement: torch's E4M3 decode and cast, numpy softmax."""
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
    p = np.exp(z - z.max())
    l = p.sum()
    vv = e4m3_decode_torch(vT[g * D:(g + 1) * D, j0:j1]).T * sv[np.arange(j0, j1) // 128, g * D:(g + 1) * D]
    o = np.zeros(D)
    for b0 in range((j0 // 128) * 128, j1, 128):
        lo, hi = max(b0, j0), min(b0 + 128, j1)
        pb = p[lo - j0:hi - j0]
        s = pb.max() / 448.0
        codes = torch.from_numpy((pb / s).astype(np.float32)).to(torch.float8_e4m3fn)
        phat = codes.to(torch.float64).numpy() * s
        o += phat @ vv[lo - j0:hi - j0]
    return o / l


@pytest.mark.parametrize("causal", [True, False])
def test_brute_force_tiny(orc, causal):
    Hq, Hkv, T = 4, 2, 512
    q, sq, k, sk, vT, sv = make_case(orc, T, Hq, Hkv, 3)
    off, ln = [0, 256, 512], [200, 256]          # a padded segment and a full one
    rows = [(t, h) for t in (0, 1, 77, 128, 199, 200, 255, 256, 300, 511) for h in range(Hq)]
    rt = [r[0] for r in rows]
    rh = [r[1] for r in rows]
    O, oa, of = orc.attention_fwd_rows(q, sq, k, sk, vT, sv, Hq, Hkv, off, ln, causal, rt, rh)
    for i, (t, h) in enumerate(rows):
        ref = brute_force(q, sq, k, sk, vT, sv, Hq, Hkv, off, ln, causal, t, h)
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

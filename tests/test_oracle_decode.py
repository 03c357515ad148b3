"""Pins of the oracle's FP8 KV-cache decode attention reference (CPU only).

Method: "NVIDIA NeMo RL erreicht 48% ..." section "Leistungsgewinne in der
Praxis": the recipe extends FP8 to the KV cache and the attention
operations of generation.  Reading: the cache holds K and V as the
row-wise 1x128 quantization of the token matrix (one E4M3 code row and one
fp32 scale per token and KV head); the new token's query stays bf16; the
softmax and P.V are exact (fp64 in the oracle).  Each pin holds by
construction or by the mathematics, independently of the oracle's code: an
independent brute force built on torch's E4M3 decode, closed forms and
invariants."""
import math

import numpy as np
import pytest
import torch

D = 128


def bf16_bits(x):
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def make_cache(orc, B, Hq, Hkv, Lmax, seed, kscale=1.0):
    """Random bf16 query [B, Hq*128] and a cache [B*Lmax, Hkv*128] quantized
    row-wise by the oracle's own 1x128 quantizer."""
    g = torch.Generator().manual_seed(seed)
    Q = torch.randn((B, Hq * D), generator=g)
    K = torch.randn((B * Lmax, Hkv * D), generator=g) * kscale
    V = torch.randn((B * Lmax, Hkv * D), generator=g)
    k, sk, _, _ = orc.quant_act_1x128(bf16_bits(K), 0, colwise=False)
    v, sv, _, _ = orc.quant_act_1x128(bf16_bits(V), 0, colwise=False)
    return bf16_bits(Q), k, sk, v, sv


def brute_force(qb, k, sk, v, sv, Hq, Hkv, lens, Lmax):
    """Independent restatement: torch's float8_e4m3fn decode of the codes,
    numpy fp64 softmax and sum, rows looped in Python."""
    dec = lambda c: torch.from_numpy(np.ascontiguousarray(c)).view(torch.float8_e4m3fn).double().numpy()  # noqa: E731
    qf = torch.from_numpy(qb.view(np.int16)).view(torch.bfloat16).double().numpy()
    B, G = qb.shape[0], Hq // Hkv
    out = np.zeros((B, Hq, D))
    for b in range(B):
        L = lens[b]
        if L == 0:
            continue
        rows = b * Lmax + np.arange(L)
        for h in range(Hq):
            gk = h // G
            kh = dec(k[rows, gk * D:(gk + 1) * D]) * sk[gk, rows][:, None].astype(np.float64)
            vh = dec(v[rows, gk * D:(gk + 1) * D]) * sv[gk, rows][:, None].astype(np.float64)
            z = kh @ qf[b, h * D:(h + 1) * D] / math.sqrt(D)
            p = np.exp(z - z.max())
            out[b, h] = p @ vh / p.sum()
    return out


@pytest.mark.parametrize("Hq,Hkv", [(1, 1), (4, 2), (8, 1), (32, 8)])
def test_brute_force(orc, Hq, Hkv):
    B, Lmax = 3, 256
    lens = [1, 200, 256]
    qb, k, sk, v, sv = make_cache(orc, B, Hq, Hkv, Lmax, 11 + Hq)
    O, oa, oe = orc.attention_decode(qb, k, sk, v, sv, Hq, Hkv, lens, Lmax)
    ref = brute_force(qb, k, sk, v, sv, Hq, Hkv, lens, Lmax)
    np.testing.assert_allclose(O, ref, rtol=1e-12, atol=1e-13)
    assert np.all(oa >= np.abs(O) - 1e-12) and np.all(oe >= 0)


def test_single_key_is_v(orc):
    """A one-token cache: p = 1, so O is that token's dequantized V."""
    qb, k, sk, v, sv = make_cache(orc, 2, 2, 1, 128, 3)
    O, _, _ = orc.attention_decode(qb, k, sk, v, sv, 2, 1, [1, 1], 128)
    for b in range(2):
        vhat = np.array([orc.e4m3_decode(c) for c in v[b * 128]]) * sv[0, b * 128]
        assert np.array_equal(O[b, 0], vhat) and np.array_equal(O[b, 1], vhat)


def test_identical_keys_average_v(orc):
    """All cached keys equal: equal logits, O = the mean of the V rows."""
    Lmax = 128
    qb, k, sk, v, sv = make_cache(orc, 1, 1, 1, Lmax, 4)
    k[:] = k[0]
    sk[:] = sk[0, 0]
    L = 77
    O, _, _ = orc.attention_decode(qb, k, sk, v, sv, 1, 1, [L], Lmax)
    dec = np.array([orc.e4m3_decode(c) for c in range(256)])
    vhat = dec[v[:L]] * sv[0, :L, None]
    np.testing.assert_allclose(O[0, 0], vhat.mean(axis=0), rtol=1e-13, atol=1e-15)


def test_dominating_key(orc):
    """One key's logit exceeds the others' by 60: O is its V^ up to e^-60."""
    Lmax = 128
    qb, k, sk, v, sv = make_cache(orc, 1, 1, 1, Lmax, 5)
    k[:] = k[0]
    sk[:] = sk[0, 0]
    dec = np.array([orc.e4m3_decode(c) for c in range(256)])
    qf = torch.from_numpy(qb.view(np.int16)).view(torch.bfloat16).double().numpy()[0]
    z0 = (dec[k[0]] * float(sk[0, 0])) @ qf / math.sqrt(D)
    sk[0, 40] = np.float32(sk[0, 0] * (1 + 60.0 / z0))       # z_40 = z_0 + 60
    O, _, _ = orc.attention_decode(qb, k, sk, v, sv, 1, 1, [100], Lmax)
    vhat = dec[v[40]] * sv[0, 40]
    np.testing.assert_allclose(O[0, 0], vhat, rtol=1e-20, atol=1e-24 * np.abs(dec[v[:100]] * sv[0, :100, None]).max())


def test_gqa_equals_replicated_kv_heads(orc):
    """Hq = 4 over Hkv = 2 equals Hq = 4 over 4 KV heads where heads 2i and
    2i + 1 each get a copy of KV head i."""
    B, Lmax = 2, 128
    qb, k, sk, v, sv = make_cache(orc, B, 4, 2, Lmax, 6)
    rep = lambda c: np.concatenate([c[:, :D], c[:, :D], c[:, D:], c[:, D:]], axis=1)  # noqa: E731
    sk4 = np.stack([sk[0], sk[0], sk[1], sk[1]])
    sv4 = np.stack([sv[0], sv[0], sv[1], sv[1]])
    lens = [128, 57]
    O2, _, _ = orc.attention_decode(qb, k, sk, v, sv, 4, 2, lens, Lmax)
    O4, _, _ = orc.attention_decode(qb, rep(k), sk4, rep(v), sv4, 4, 4, lens, Lmax)
    assert np.array_equal(O2, O4)


def test_empty_cache_and_tokens_past_the_length(orc):
    """len = 0 gives zeros; cache rows past a sequence's length change
    nothing."""
    B, Lmax = 2, 256
    qb, k, sk, v, sv = make_cache(orc, B, 2, 2, Lmax, 7)
    O, oa, oe = orc.attention_decode(qb, k, sk, v, sv, 2, 2, [0, 130], Lmax)
    assert np.all(O[0] == 0) and np.all(oa[0] == 0) and np.all(oe[0] == 0)
    k2, v2 = k.copy(), v.copy()
    k2[Lmax + 130:] = 0x7E
    v2[Lmax + 130:] = 0xFE
    sk2 = sk.copy()
    sk2[:, Lmax + 130:] = 1e30
    O2, _, _ = orc.attention_decode(qb, k2, sk2, v2, sv, 2, 2, [0, 130], Lmax)
    assert np.array_equal(O, O2)


def test_error_allowance_scales_with_the_logits(orc):
    """The fp32 allowance grows with the logits' magnitude: keys scaled by
    2^10 give a larger oerr / oabs ratio than unscaled ones."""
    B, Lmax = 1, 128
    small = make_cache(orc, B, 1, 1, Lmax, 8)
    large = make_cache(orc, B, 1, 1, Lmax, 8, kscale=2.0 ** 10)
    _, oa1, oe1 = orc.attention_decode(*small, 1, 1, [128], Lmax)
    _, oa2, oe2 = orc.attention_decode(*large, 1, 1, [128], Lmax)
    r1, r2 = (oe1 / oa1).max(), (oe2 / oa2).max()
    assert 0 < r1 < r2 and r1 < 1e-3

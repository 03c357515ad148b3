"""GPU parity of the FP8 KV-cache decode attention against the oracle.

Method: "NVIDIA NeMo RL erreicht 48% ..." section "Leistungsgewinne in der
Praxis" (FP8 KV cache and attention in generation); workload shapes from
"NeMo-RL v0.3 mit Megatron-Core ..." (Llama 3.1 8B: 32 query heads, 8
key/value heads of 128; 16K-token contexts).  The cache is made by the
library's own row-wise 1x128 quantizer (one scale per token and KV head),
in both scale modes; the query is bf16.  Gate (fp32 kernel against the
fp64 reference): |o - O| <= 2^-10 sum_j p_j |v^_j| / l + 4 dz sum_j p_j
|v^_j| / l + 1 bf16 ulp, dz the oracle's bound on the fp32 logit error."""
import numpy as np
import pytest
import torch

import workloads
from util import bits

pytestmark = pytest.mark.gpu
DEV = "cuda"
D = 128
REL = 2.0 ** -10


def make_cache(fb, K, V, mode):
    T, Hkv = K.shape[0], K.shape[1] // D
    e = lambda *s, dt=torch.uint8: torch.empty(s, dtype=dt, device=DEV)  # noqa: E731
    k, sk, v, sv = e(T, Hkv * D), e(Hkv, T, dt=torch.float32), e(T, Hkv * D), e(Hkv, T, dt=torch.float32)
    fb.fp8bw_quant_act_1x128(K, mode, k, sk)
    fb.fp8bw_quant_act_1x128(V, mode, v, sv)
    return k, sk, v, sv


def run_and_check(fb, orc, Q, k, sk, v, sv, lens, Lmax, check_rows=None):
    B, Hq = Q.shape[0], Q.shape[1] // D
    Hkv = k.shape[1] // D
    o = torch.full((B, Hq * D), float("nan"), dtype=torch.bfloat16, device=DEV)
    fb.fp8bw_attention_decode(Q, k, sk, v, sv, o, torch.tensor(lens, dtype=torch.int32, device=DEV), Lmax)
    torch.cuda.synchronize()
    assert fb.fp8bw_last_device_error() == 0
    O, oa, oe = orc.attention_decode(bits(Q), k.cpu().numpy(), sk.cpu().numpy(), v.cpu().numpy(),
                                     sv.cpu().numpy(), Hq, Hkv, lens, Lmax)
    got = bits(o).reshape(B, Hq, D)
    sel = slice(None) if check_rows is None else check_rows
    bad, worst = orc.check_tol_attn(got[sel], O[sel], oa[sel], oe[sel], rel=REL)
    assert bad == 0, worst
    for b in range(B):
        if lens[b] == 0:
            assert torch.all(o[b] == 0)
    return o


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("heads", [(2, 2), (4, 2), (8, 2), (8, 1)])
def test_decode_all_rows(fb, orc, heads, mode):
    """Every (sequence, head) row, group sizes 1, 2, 4 and 8; lengths 0, 1,
    tile edges (31, 32, 33), a slice edge (255, 256, 257) and the whole
    cache (512)."""
    g = torch.Generator(device="cpu").manual_seed(40 + heads[0] + heads[1])
    Hq, Hkv = heads
    lens = [0, 1, 31, 32, 33, 255, 256, 257, 512]
    B, Lmax = len(lens), 512
    Q = torch.randn((B, Hq * D), generator=g).to(torch.bfloat16).to(DEV)
    K = torch.randn((B * Lmax, Hkv * D), generator=g).to(torch.bfloat16).to(DEV)
    V = torch.randn((B * Lmax, Hkv * D), generator=g).to(torch.bfloat16).to(DEV)
    run_and_check(fb, orc, Q, *make_cache(fb, K, V, mode), lens, Lmax)


@pytest.mark.parametrize("heads", [(32, 8), (8, 1)])
@pytest.mark.parametrize("mode", [0, 1])
def test_decode_long_cache_spread_scales(fb, orc, mode, heads):
    """16K-token caches (Llama-3.1-8B heads: 32 query over 8 KV; and eight
    query heads over one KV head), keys whose rows are scaled by
    2^-10 .. 2^8 and queries by up to 2^4, so logits range over orders of
    magnitude; every row checked."""
    g = torch.Generator(device="cpu").manual_seed(44)
    (Hq, Hkv), Lmax = heads, 16384
    lens = [16384, 9000, 1, 12345]
    B = len(lens)
    Q = torch.randn((B, Hq * D), generator=g) * (2.0 ** torch.randint(0, 5, (B, 1), generator=g))
    K = torch.randn((B * Lmax, Hkv * D), generator=g)
    K *= 2.0 ** torch.randint(-10, 9, (B * Lmax, 1), generator=g).float()
    V = torch.randn((B * Lmax, Hkv * D), generator=g)
    Q, K, V = (x.to(torch.bfloat16).to(DEV) for x in (Q, K, V))
    run_and_check(fb, orc, Q, *make_cache(fb, K, V, mode), lens, Lmax)


def test_decode_rollout_batch_sampled(fb, orc):
    """The benchmark's launch: 64 sequences of a 16K-token cache with the
    seeded length mix, 32 query / 8 KV heads; rows of 12 sequences (the
    shortest, the longest and random ones) checked."""
    lens, Lmax = workloads.decode_lengths(0)
    B, Hq, Hkv = len(lens), 32, 8
    Q = workloads.normal_bf16((B, Hq * D), 1.0, 51, DEV)
    K = workloads.normal_bf16((B * Lmax, Hkv * D), 1.0, 52, DEV)
    V = workloads.normal_bf16((B * Lmax, Hkv * D), 1.0, 53, DEV)
    k, sk, v, sv = make_cache(fb, K, V, 0)
    rng = np.random.default_rng(5)
    pick = sorted(set([int(np.argmin(lens)), int(np.argmax(lens))] + [int(x) for x in rng.choice(B, 10, replace=False)]))
    # the oracle on the picked sequences only (their cache rows, lengths kept)
    o = torch.full((B, Hq * D), float("nan"), dtype=torch.bfloat16, device=DEV)
    fb.fp8bw_attention_decode(Q, k, sk, v, sv, o, torch.tensor(lens, dtype=torch.int32, device=DEV), Lmax)
    torch.cuda.synchronize()
    assert fb.fp8bw_last_device_error() == 0
    rows = torch.cat([torch.arange(b * Lmax, (b + 1) * Lmax) for b in pick]).to(DEV)
    sub = lambda c: c[rows].cpu().numpy()  # noqa: E731
    subs = lambda s: s[:, rows].cpu().numpy()  # noqa: E731
    O, oa, oe = orc.attention_decode(bits(Q[pick]), sub(k), subs(sk), sub(v), subs(sv), Hq, Hkv,
                                     [lens[b] for b in pick], Lmax)
    got = bits(o[pick]).reshape(len(pick), Hq, D)
    bad, worst = orc.check_tol_attn(got, O, oa, oe, rel=REL)
    assert bad == 0, worst


def test_decode_rejects_bad_length(fb, orc):
    """A length above Lmax latches FP8BW_ERR_DEVICE_CHECK; that sequence's
    output is not written and the others are still correct."""
    g = torch.Generator(device="cpu").manual_seed(46)
    Hq, Hkv, Lmax = 4, 2, 256
    B = 3
    Q = torch.randn((B, Hq * D), generator=g).to(torch.bfloat16).to(DEV)
    K = torch.randn((B * Lmax, Hkv * D), generator=g).to(torch.bfloat16).to(DEV)
    V = torch.randn((B * Lmax, Hkv * D), generator=g).to(torch.bfloat16).to(DEV)
    k, sk, v, sv = make_cache(fb, K, V, 0)
    o = torch.full((B, Hq * D), 3.0, dtype=torch.bfloat16, device=DEV)
    fb.fp8bw_attention_decode(Q, k, sk, v, sv, o, torch.tensor([100, Lmax + 1, 7], dtype=torch.int32, device=DEV),
                              Lmax)
    assert fb.fp8bw_last_device_error() == 6
    assert torch.all(o[1] == 3.0)
    O, oa, oe = orc.attention_decode(bits(Q), k.cpu().numpy(), sk.cpu().numpy(), v.cpu().numpy(),
                                     sv.cpu().numpy(), Hq, Hkv, [100, 0, 7], Lmax)
    got = bits(o).reshape(B, Hq, D)
    for b in (0, 2):
        bad, worst = orc.check_tol_attn(got[b], O[b], oa[b], oe[b], rel=REL)
        assert bad == 0, worst
    assert fb.fp8bw_last_device_error() == 0

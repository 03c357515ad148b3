"""GPU parity of the FP8 attention forward against the oracle.

Method: "NVIDIA NeMo RL erreicht 48% ..." section "Leistungsgewinne in der
Praxis" (FP8 KV cache and attention); workload shapes from "NeMo-RL v0.3
mit Megatron-Core ..." (Llama 3.1 8B: 32 query heads, 8 key/value heads of
128; sequence packing with 16K-token contexts).  Q, K and V are quantized
by the library's own activation quantizer (Q, K row-wise: one scale per
token and head; V's column-wise copy), then attended with
fp8bw_attention_fwd; the oracle recomputes (token, head) rows in fp64 and
the gate is |o - O| <= 1e-2 sum|p^ v^| / l + midpoint allowance + 1 bf16 ulp."""
import numpy as np
import pytest
import torch

import workloads
from util import bits

pytestmark = pytest.mark.gpu
DEV = "cuda"
D = 128


def quantize_qkv(fb, Q, K, V, mode=0):
    T = Q.shape[0]
    Hq, Hkv = Q.shape[1] // D, K.shape[1] // D
    e = lambda *s, dt=torch.uint8: torch.empty(s, dtype=dt, device=DEV)  # noqa: E731
    q, sq = e(T, Hq * D), e(Hq, T, dt=torch.float32)
    k, sk = e(T, Hkv * D), e(Hkv, T, dt=torch.float32)
    vrow, svrow = e(T, Hkv * D), e(Hkv, T, dt=torch.float32)
    vT, sv = e(Hkv * D, T), e(T // 128, Hkv * D, dt=torch.float32)
    fb.fp8bw_quant_act_1x128(Q, mode, q, sq)
    fb.fp8bw_quant_act_1x128(K, mode, k, sk)
    fb.fp8bw_quant_act_1x128(V, mode, vrow, svrow, vT, sv)
    return q, sq, k, sk, vT, sv


def run_and_check(fb, orc, Q, K, V, off, ln, causal, rows, mode=0):
    T = Q.shape[0]
    Hq, Hkv = Q.shape[1] // D, K.shape[1] // D
    ops = quantize_qkv(fb, Q, K, V, mode)
    o = torch.full((T, Hq * D), float("nan"), dtype=torch.bfloat16, device=DEV)
    offd = torch.tensor(off, dtype=torch.int32, device=DEV)
    lnd = torch.tensor(ln, dtype=torch.int32, device=DEV)
    fb.fp8bw_attention_fwd(*ops, o, offd, lnd, causal, mode)
    torch.cuda.synchronize()
    assert fb.fp8bw_last_device_error() == 0
    host = [t.cpu().numpy() for t in ops]
    rt = np.array([r[0] for r in rows], np.int64)
    rh = np.array([r[1] for r in rows], np.int32)
    O, oa, of = orc.attention_fwd_rows(*host, Hq, Hkv, off, ln, causal, rt, rh, mode)
    ob = bits(o)
    got = np.stack([ob[t, h * D:(h + 1) * D] for t, h in rows])
    bad, worst = orc.check_tol_attn(got, O, oa, of)
    assert bad == 0, worst
    return o


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("causal", [1, 0])
def test_attention_tiny_all_rows(fb, orc, causal, mode):
    """T = 512, 4 query heads over 2 KV heads, a padded segment (200 real of
    256) and a full one; every (token, head) row is checked, and padding
    rows are exact zeros."""
    g = torch.Generator(device="cpu").manual_seed(1)
    T, Hq, Hkv = 512, 4, 2
    Q = torch.randn((T, Hq * D), generator=g).to(torch.bfloat16).to(DEV)
    K = torch.randn((T, Hkv * D), generator=g).to(torch.bfloat16).to(DEV)
    V = torch.randn((T, Hkv * D), generator=g).to(torch.bfloat16).to(DEV)
    off, ln = [0, 256, 512], [200, 256]
    rows = [(t, h) for t in range(T) for h in range(Hq)]
    o = run_and_check(fb, orc, Q, K, V, off, ln, causal, rows, mode)
    assert torch.all(o[200:256] == 0)


@pytest.mark.parametrize("heads", [(2, 2), (4, 2), (3, 1), (8, 1)])
@pytest.mark.parametrize("mode", [0, 1])
def test_attention_ragged_segments(fb, orc, mode, heads):
    """Odd lengths, an empty segment, a one-token sequence and tokens past
    the last segment (zeros); Hq = Hkv (no grouping), two query heads per
    KV head (the two-head kernels), three (an odd group: the one-head
    kernels) and eight (four head pairs of one KV group); scales spread over
    orders of magnitude (some rows scaled by 2^-20, some by 2^12)."""
    g = torch.Generator(device="cpu").manual_seed(2)
    T, (Hq, Hkv) = 1024, heads
    Q = torch.randn((T, Hq * D), generator=g)
    Q[::7] *= 2.0 ** -20
    Q[3::11] *= 2.0 ** 12
    K = torch.randn((T, Hkv * D), generator=g)
    K[5::13] *= 2.0 ** -10
    V = torch.randn((T, Hkv * D), generator=g)
    Q, K, V = (x.to(torch.bfloat16).to(DEV) for x in (Q, K, V))
    off, ln = [0, 384, 384, 512, 640, 896], [301, 0, 1, 128, 255]
    rows = [(t, h) for t in list(range(0, 400)) + list(range(500, 1024, 3)) for h in range(Hq)]
    o = run_and_check(fb, orc, Q, K, V, off, ln, 1, rows, mode)
    assert torch.all(o[896:] == 0) and torch.all(o[301:384] == 0) and torch.all(o[385:512] == 0)


@pytest.mark.parametrize("mode", [0, 1])
def test_attention_llama8b_packed_full_size(fb, orc, mode):
    """Llama-3.1-8B-like attention (32 query heads, 8 KV heads of 128) over
    the packed long-sequence batch (4 sequences, 32768 tokens, each padded
    to a multiple of 128), causal, in the benchmark's launch configuration.
    Checked rows: the first, last and random rows of every sequence, rows
    at block boundaries, for all heads of some of them; padding rows zero."""
    T, Hq, Hkv = workloads.PACKED_TOKENS, 32, 8
    off, ln = workloads.packed_segments(0)
    Q = workloads.normal_bf16((T, Hq * D), 1.0, 31, DEV)
    K = workloads.normal_bf16((T, Hkv * D), 1.0, 32, DEV)
    V = workloads.normal_bf16((T, Hkv * D), 1.0, 33, DEV)
    rng = np.random.default_rng(3)
    rows = []
    for s in range(len(ln)):
        a, n = off[s], ln[s]
        for t in [a, a + 1, a + 127, a + 128, a + n - 1] + [a + int(x) for x in rng.integers(0, n, 8)]:
            rows += [(t, int(h)) for h in rng.choice(Hq, 4, replace=False)]
        rows += [(a + n - 1, h) for h in range(Hq)]
    o = run_and_check(fb, orc, Q, K, V, off, ln, 1, sorted(set(rows)), mode)
    for s in range(len(ln)):
        if off[s] + ln[s] < off[s + 1]:
            assert torch.all(o[off[s] + ln[s]:off[s + 1]] == 0)


def test_attention_bad_offsets(fb, orc):
    """Offsets that are not multiples of 128 are rejected on the device:
    nothing is written and FP8BW_ERR_DEVICE_CHECK is latched."""
    T, H = 256, 1
    Q = torch.randn((T, H * D), device=DEV).to(torch.bfloat16)
    ops = quantize_qkv(fb, Q, Q, Q)
    o = torch.full((T, H * D), 3.0, dtype=torch.bfloat16, device=DEV)
    off = torch.tensor([0, 100, 256], dtype=torch.int32, device=DEV)
    ln = torch.tensor([100, 100], dtype=torch.int32, device=DEV)
    fb.fp8bw_attention_fwd(*ops, o, off, ln, 1)
    assert fb.fp8bw_last_device_error() == 6
    assert torch.all(o == 3.0)
    assert fb.fp8bw_last_device_error() == 0


@pytest.mark.parametrize("hq", [1, 2])
def test_attention_pow2_rejects_other_scales(fb, orc, hq):
    """Power-of-2 mode with scales from the FP32 rule (not powers of two):
    the kernel latches FP8BW_ERR_DEVICE_CHECK (o is undefined); the same
    operands in FP32 mode are fine.  One KV head with one query head, and
    with two (the two-head kernel)."""
    T = 256
    g = torch.Generator(device="cpu").manual_seed(5)
    Q = torch.randn((T, hq * D), generator=g).to(torch.bfloat16).to(DEV)
    KV = Q[:, :D].contiguous()
    ops = quantize_qkv(fb, Q, KV, KV, 0)
    o = torch.empty((T, hq * D), dtype=torch.bfloat16, device=DEV)
    off = torch.tensor([0, T], dtype=torch.int32, device=DEV)
    ln = torch.tensor([T], dtype=torch.int32, device=DEV)
    fb.fp8bw_attention_fwd(*ops, o, off, ln, 1, 1)
    assert fb.fp8bw_last_device_error() == 6
    fb.fp8bw_attention_fwd(*ops, o, off, ln, 1, 0)
    assert fb.fp8bw_last_device_error() == 0

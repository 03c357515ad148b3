"""GPU parity of the GEMM with the quantizing epilogue (fp8bw_gemm_quant).

Method: "NVIDIA NeMo RL erreicht 48% ..." sections "Der technische
Durchbruch" (1x128 activation blocks) and "Leistungsgewinne in der Praxis"
(quantization-kernel overhead): a GEMM whose output is the next FP8 GEMM's
operand writes that operand directly.

Checks, per kind and output scale rule:
  * D (the bf16 result the epilogue quantizes) is within the GEMM gate of
    the oracle's fp64 reference, and equals fp8bw_gemm's bf16 output bit for
    bit (the same promotion kernel);
  * the dequantized codes are within the gate plus the E4M3 rounding bound
    (half a step: 2^-4 of |D| for normal codes, 2^-10 of the block scale
    below) of the oracle's reference;
  * the codes and scales equal, bit for bit, fp8bw_quant_act_1x128 applied
    to the same D (the quantizer's own kernel, itself bit-exact against the
    oracle in test_gpu_quant.py)."""
import numpy as np
import pytest
import torch

import workloads
from util import act_buffers, bits, weight_buffers

pytestmark = pytest.mark.gpu
DEV = "cuda"


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def operands(fb, kind, M, N, K, seed):
    """Quantized operands of one GEMM of the given kind and sizes (M, N, K the
    GEMM's own sizes), from seeded bf16 tensors quantized by the library."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    if kind == 0:        # Y[M,N] = X[M,K] W[N,K]^T
        X = torch.randn((M, K), generator=g).to(torch.bfloat16).to(DEV)
        W = (torch.randn((N, K), generator=g) * 0.02).to(torch.bfloat16).to(DEV)
        qa, sa, _, _ = act_buffers(M, K, DEV, colwise=False)
        fb.fp8bw_quant_act_1x128(X, 0, qa, sa)
        qw, sw, _ = weight_buffers(N, K, DEV, transposed=False)
        fb.fp8bw_quant_weight_128x128(W, 0, qw, sw)
        return qa, sa, qw, sw
    if kind == 1:        # dX[M,N] = dY[M,K] W[K,N]: B = qT of W [K_layer=N... ]
        dY = (torch.randn((M, K), generator=g) * 1e-3).to(torch.bfloat16).to(DEV)
        W = (torch.randn((K, N), generator=g) * 0.02).to(torch.bfloat16).to(DEV)
        qa, sa, _, _ = act_buffers(M, K, DEV, colwise=False)
        fb.fp8bw_quant_act_1x128(dY, 0, qa, sa)
        qw, sw, qwT = weight_buffers(K, N, DEV)
        fb.fp8bw_quant_weight_128x128(W, 0, qw, sw, qwT)
        return qa, sa, qwT, sw
    # wgrad: dW[M,N] = dY^T[M, K=tokens] X[K=tokens, N]
    dY = (torch.randn((K, M), generator=g) * 1e-3).to(torch.bfloat16).to(DEV)
    X = torch.randn((K, N), generator=g).to(torch.bfloat16).to(DEV)
    _, _, qdc, sdc = act_buffers(K, M, DEV)
    _, _, qxc, sxc = act_buffers(K, N, DEV)
    fb.fp8bw_quant_act_1x128(dY, 0, *act_buffers(K, M, DEV, colwise=False)[:2], qdc, sdc)
    fb.fp8bw_quant_act_1x128(X, 0, *act_buffers(K, N, DEV, colwise=False)[:2], qxc, sxc)
    return qdc, sdc, qxc, sxc


def run_case(fb, orc, kind, M, N, K, mode, seed, tiles=None):
    A, sA, B, sB = operands(fb, kind, M, N, K, seed)
    q_row, s_row, q_col, s_col = act_buffers(M, N, DEV)
    D = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    fb.fp8bw_gemm_quant(kind, A, sA, B, sB, q_row, s_row, q_col, s_col, D=D, mode=mode)
    Dref = torch.empty_like(D)
    fb.fp8bw_gemm(kind, A, sA, B, sB, Dref, 0)
    r_row, rs_row, r_col, rs_col = act_buffers(M, N, DEV)
    fb.fp8bw_quant_act_1x128(D, mode, r_row, rs_row, r_col, rs_col)
    # row-wise only, without D
    o_row, os_row, _, _ = act_buffers(M, N, DEV, colwise=False)
    fb.fp8bw_gemm_quant(kind, A, sA, B, sB, o_row, os_row, mode=mode)
    torch.cuda.synchronize()
    assert fb.fp8bw_last_device_error() == 0
    assert torch.equal(D.view(torch.int16), Dref.view(torch.int16))
    assert torch.equal(q_row, r_row) and torch.equal(q_col, r_col)
    assert torch.equal(s_row.view(torch.int32), rs_row.view(torch.int32))
    assert torch.equal(s_col.view(torch.int32), rs_col.view(torch.int32))
    assert torch.equal(o_row, q_row) and torch.equal(os_row.view(torch.int32), s_row.view(torch.int32))
    # against the oracle
    Ah, sAh, Bh, sBh = (t.cpu().numpy() for t in (A, sA, B, sB))
    Db, qr, sr = bits(D), q_row.cpu().numpy(), s_row.cpu().numpy()
    dec = np.array([orc.e4m3_decode(c) for c in range(256)])
    if tiles is None:
        tiles = [(m0, n0) for m0 in range(0, M, 128) for n0 in range(0, N, 128)]
    for (m0, n0) in tiles:
        y, ya = orc.gemm_ref_tile(kind, Ah, sAh, Bh, sBh, m0, m0 + 128, n0, n0 + 128)
        bad, worst = orc.check_tol(np.ascontiguousarray(Db[m0:m0 + 128, n0:n0 + 128]), y, ya)
        assert bad == 0, ("D", m0, n0, worst)
        s = sr[n0 // 128, m0:m0 + 128].astype(np.float64)[:, None]
        xq = dec[qr[m0:m0 + 128, n0:n0 + 128]] * s
        dval = (Db[m0:m0 + 128, n0:n0 + 128].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        allow = 1e-2 * ya + np.array([[orc.bf16_ulp(v) for v in row] for row in y]) + \
            2.0 ** -4 * np.abs(dval) + 2.0 ** -10 * s
        assert np.all(np.abs(xq - y) <= allow), ("codes", m0, n0)


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("kind", [0, 1, 2])
def test_gemm_quant_small(fb, orc, kind, mode):
    """Every tile of a 384 x 640 result (the pair tile's second CTA past M,
    the last tile's second column half past N), K = 512."""
    run_case(fb, orc, kind, 384, 640, 512, mode, seed=10 * kind + mode)


@pytest.mark.parametrize("mode", [0, 1])
def test_gemm_quant_many_tiles(fb, orc, mode):
    """More pair tiles than CTA pairs, so every pair runs the epilogue's
    shared tile several times: dgrad of the o_proj shape at 8192 tokens,
    sampled 128x128 tiles checked against the oracle, all bits against the
    unfused path."""
    rng = np.random.default_rng(4 + mode)
    M, N, K = workloads.LLAMA8B_TOKENS, 4096, 4096
    tiles = [(0, 0), (M - 128, N - 128)] + [(128 * int(rng.integers(0, M // 128)), 128 * int(rng.integers(0, N // 128)))
                                            for _ in range(6)]
    run_case(fb, orc, 1, M, N, K, mode, seed=77, tiles=tiles)

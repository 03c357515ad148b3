"""GPU parity of the blockwise FP8 GEMMs (fprop / dgrad / wgrad) and of the
BF16 comparison GEMM against the oracle's fp64 reference.

Method: "NVIDIA NeMo RL erreicht 48% ..." section "Der technische
Durchbruch": FP8 linear layers on 1x128 / 128x128 blockwise-scaled E4M3
operands.  Acceptance: |y - y_ref| <= 1e-2 * sum_k |a_k b_k| + 1 bf16 ulp(y_ref),
y_ref the fp64 product of the dequantized operands.  The operands come from
the oracle's quantizer, so these tests do not depend on the GPU quantizers.
"""
import numpy as np
import pytest
import torch

import workloads
from util import bits

pytestmark = pytest.mark.gpu
DEV = "cuda"


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def gpu_gemm(fb, kind, A, sA, B, sB, mode=0):
    M, N = A.shape[0], B.shape[0]
    D = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    fb.fp8bw_gemm(kind, dev(A), dev(sA), dev(B), dev(sB), D, mode)
    torch.cuda.synchronize()
    assert fb.fp8bw_last_device_error() == 0
    return bits(D)


def operands(orc, X, W, dY, mode):
    """Quantized operands of the three GEMMs of one linear layer."""
    qx, sx, qxc, sxc = orc.quant_act_1x128(bits(X), mode)
    qw, sw, qwT = orc.quant_weight_128x128(bits(W), mode)
    qd, sd, qdc, sdc = orc.quant_act_1x128(bits(dY), mode)
    return {
        0: (qx, sx, qw, sw),          # fprop:  Y  = X W^T
        1: (qd, sd, qwT, sw),         # dgrad:  dX = dY W
        2: (qdc, sdc, qxc, sxc),      # wgrad:  dW = dY^T X
    }


def check(orc, y, kind, A, sA, B, sB):
    yr, ya = orc.gemm_ref_tile(kind, A, sA, B, sB, 0, A.shape[0], 0, B.shape[0])
    bad, worst = orc.check_tol(y, yr, ya)
    assert bad == 0, f"kind {kind}: {bad} elements out of tolerance (worst ratio {worst:.3g})"
    return worst


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("kind", [0, 1, 2])
def test_tiny_layer(fb, orc, kind, mode):
    X, W, dY = workloads.tiny(0)
    ops = operands(orc, X, W, dY, mode)[kind]
    y = gpu_gemm(fb, kind, *ops, mode=mode)
    check(orc, y, kind, *ops)
    # FP32 accumulation and promotion leave the result far inside the 1%
    # gate: within 1e-3 * sum|ab| + 1 ulp (bf16 output rounding dominates).
    yr, ya = orc.gemm_ref_tile(kind, *ops, 0, ops[0].shape[0], 0, ops[2].shape[0])
    bad, worst = orc.check_tol(y, yr, ya, rel=1e-3)
    assert bad == 0, worst


def rand_ops(rng, M, N, K, kind):
    A = rng.integers(0, 0x7E, (M, K), dtype=np.uint8) | (rng.integers(0, 2, (M, K), dtype=np.uint8) << 7)
    B = rng.integers(0, 0x7E, (N, K), dtype=np.uint8) | (rng.integers(0, 2, (N, K), dtype=np.uint8) << 7)
    nK = K // 128
    sA = (2.0 ** rng.uniform(-10, 4, (nK, M))).astype(np.float32)
    shp = {0: (N // 128, nK), 1: (nK, N // 128), 2: (nK, N)}[kind]
    sB = (2.0 ** rng.uniform(-10, 4, shp)).astype(np.float32)
    return A, sA, B, sB


@pytest.mark.parametrize("kind", [0, 1, 2])
@pytest.mark.parametrize("MNK", [(128, 128, 128), (384, 640, 384), (256, 384, 1024), (640, 256, 256)])
def test_shapes(fb, orc, kind, MNK):
    rng = np.random.default_rng(hash((kind,) + MNK) % 2**32)
    ops = rand_ops(rng, *MNK, kind)
    y = gpu_gemm(fb, kind, *ops)
    check(orc, y, kind, *ops)


@pytest.mark.parametrize("kind", [0, 1, 2])
def test_small_integers_exact(fb, orc, kind):
    rng = np.random.default_rng(21 + kind)
    pool = np.array([0x00, 0x38, 0x40, 0x44, 0xB8, 0xC0], np.uint8)   # 0, 1, 2, 3, -1, -2
    M, N, K = 256, 384, 256
    A = rng.choice(pool, (M, K))
    B = rng.choice(pool, (N, K))
    sA = np.ones((K // 128, M), np.float32)
    sB = {0: np.ones((N // 128, K // 128)), 1: np.ones((K // 128, N // 128)),
          2: np.ones((K // 128, N))}[kind].astype(np.float32)
    y = gpu_gemm(fb, kind, A, sA, B, sB)
    yr, _ = orc.gemm_ref_tile(kind, A, sA, B, sB, 0, M, 0, N)
    # integer sums are exact in fp32, so the only rounding is the final bf16
    want = torch.from_numpy(yr).float().to(torch.bfloat16).double().numpy()
    got = torch.from_numpy(y.view(np.int16)).view(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(got, want)


def test_identity_and_zero_rows(fb, orc):
    rng = np.random.default_rng(2)
    M = N = K = 256
    A, sA, _, _ = rand_ops(rng, M, N, K, 0)
    A[128:] = 0
    B = np.zeros((N, K), np.uint8)
    np.fill_diagonal(B, 0x38)
    sB = np.ones((N // 128, K // 128), np.float32)
    y = gpu_gemm(fb, 0, A, sA, B, sB)
    got = torch.from_numpy(y.view(np.int16)).view(torch.bfloat16).float().numpy()
    yr, _ = orc.gemm_ref_tile(0, A, sA, B, sB, 0, M, 0, N)
    want = torch.from_numpy(yr).float().to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(got, want)
    assert np.all(got[128:] == 0)


def test_ldd(fb, orc):
    rng = np.random.default_rng(4)
    A, sA, B, sB = rand_ops(rng, 256, 256, 256, 0)
    Dbig = torch.zeros((256, 512), dtype=torch.bfloat16, device=DEV)
    D = Dbig[:, 128:384]
    fb.fp8bw_gemm(0, dev(A), dev(sA), dev(B), dev(sB), D)
    torch.cuda.synchronize()
    check(orc, bits(D), 0, A, sA, B, sB)
    assert torch.all(Dbig[:, :128] == 0) and torch.all(Dbig[:, 384:] == 0)


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("kind", [0, 1, 2])
def test_ldd_16_byte_rows(fb, orc, kind, mode):
    """Rows of D only 16-byte aligned (ldd = N + 8) and a 128-column tail
    (N = 384 is not a multiple of the 256-wide tile): nothing outside the
    N columns is written."""
    rng = np.random.default_rng(40 + kind + 3 * mode)
    M, N, K = 256, 384, 256
    ops = rand_ops(rng, M, N, K, kind)
    if mode == 1:
        ops = pow2_scales(ops)
    Dbig = torch.full((M, N + 8), float("nan"), dtype=torch.bfloat16, device=DEV)
    D = Dbig[:, :N]
    fb.fp8bw_gemm(kind, *(dev(x) for x in ops), D, mode)
    torch.cuda.synchronize()
    assert fb.fp8bw_last_device_error() == 0
    check(orc, bits(D), kind, *ops)
    assert torch.isnan(Dbig[:, N:].float()).all()


@pytest.mark.parametrize("MNK", [(256, 512, 512), (128, 384, 256)])
def test_bf16_gemm(fb, orc, MNK):
    M, N, K = MNK
    g = torch.Generator().manual_seed(M + N + K)
    A = torch.randn((M, K), generator=g).to(torch.bfloat16)
    B = torch.randn((N, K), generator=g).to(torch.bfloat16)
    D = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    fb.fp8bw_gemm_bf16(A.to(DEV), B.to(DEV), D)
    torch.cuda.synchronize()
    yr, ya = orc.gemm_bf16_ref_tile(bits(A), bits(B), 0, M, 0, N)
    bad, worst = orc.check_tol(bits(D), yr, ya, rel=1e-3)
    assert bad == 0, worst


def test_bf16_gemm_many_tiles(fb, orc):
    """More 256x256 pair tiles than CTA pairs (each pair runs several tiles,
    both TMEM accumulators in turn), M and N with a 128-wide remainder:
    sampled 128x128 tiles, corners included."""
    M, N, K = 4224, 4224, 1024
    g = torch.Generator().manual_seed(99)
    A = torch.randn((M, K), generator=g).to(torch.bfloat16)
    B = torch.randn((N, K), generator=g).to(torch.bfloat16)
    D = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    fb.fp8bw_gemm_bf16(A.to(DEV), B.to(DEV), D)
    torch.cuda.synchronize()
    Db, Ab, Bb = bits(D), bits(A), bits(B)
    rng = np.random.default_rng(5)
    tiles = [(0, 0), (M - 128, N - 128), (M - 128, 0), (0, N - 128)]
    tiles += [(128 * int(rng.integers(0, M // 128)), 128 * int(rng.integers(0, N // 128))) for _ in range(6)]
    for (m0, n0) in tiles:
        yr, ya = orc.gemm_bf16_ref_tile(Ab, Bb, m0, m0 + 128, n0, n0 + 128)
        bad, worst = orc.check_tol(np.ascontiguousarray(Db[m0:m0 + 128, n0:n0 + 128]), yr, ya, rel=1e-3)
        assert bad == 0, (m0, n0, worst)


def test_bounded_wait_timeout_is_reported(fb, orc):
    """Failure path: a producer that never fills one K-chunk makes the GEMM's
    bounded waits run out; the call comes back with FP8BW_ERR_TIMEOUT and
    the context stays usable for the next (correct) GEMM."""
    rng = np.random.default_rng(12)
    A, sA, B, sB = rand_ops(rng, 256, 256, 512, 0)
    D = torch.zeros((256, 256), dtype=torch.bfloat16, device=DEV)
    fb.fp8bw_testing_stall_next_gemm(1)
    fb.fp8bw_gemm(0, dev(A), dev(sA), dev(B), dev(sB), D)
    assert fb.fp8bw_last_device_error() == 5          # FP8BW_ERR_TIMEOUT
    assert fb.fp8bw_last_device_error() == 0          # cleared
    y = gpu_gemm(fb, 0, A, sA, B, sB)
    check(orc, y, 0, A, sA, B, sB)


def rand_ops_pow2(rng, M, N, K, kind):
    A, _, B, _ = rand_ops(rng, M, N, K, kind)
    nK = K // 128
    sA = (2.0 ** rng.integers(-20, 6, (nK, M))).astype(np.float32)
    shp = {0: (N // 128, nK), 1: (nK, N // 128), 2: (nK, N)}[kind]
    sB = (2.0 ** rng.integers(-20, 6, shp)).astype(np.float32)
    return A, sA, B, sB


@pytest.mark.parametrize("kind", [0, 1, 2])
@pytest.mark.parametrize("MNK", [(128, 128, 128), (384, 640, 384), (256, 384, 1024)])
def test_shapes_pow2(fb, orc, kind, MNK):
    """Power-of-2 scales (the tensor core's block-scaled MMA applies them)."""
    rng = np.random.default_rng(hash((kind, 7) + MNK) % 2**32)
    ops = rand_ops_pow2(rng, *MNK, kind)
    y = gpu_gemm(fb, kind, *ops, mode=1)
    check(orc, y, kind, *ops)
    yr, ya = orc.gemm_ref_tile(kind, *ops, 0, MNK[0], 0, MNK[1])
    assert orc.check_tol(y, yr, ya, rel=1e-3)[0] == 0


def test_pow2_mode_rejects_other_scales(fb, orc):
    """A scale that is not a power of two in FP8BW_SCALE_POW2 mode is latched
    as FP8BW_ERR_DEVICE_CHECK."""
    rng = np.random.default_rng(1)
    A, sA, B, sB = rand_ops_pow2(rng, 128, 256, 256, 0)
    sA[1, 5] = 0.75
    D = torch.zeros((128, 256), dtype=torch.bfloat16, device=DEV)
    fb.fp8bw_gemm(0, dev(A), dev(sA), dev(B), dev(sB), D, 1)
    assert fb.fp8bw_last_device_error() == 6


def pow2_scales(ops):
    """The same operands with every scale rounded to a power of two."""
    A, sA, B, sB = ops
    r = lambda s: (2.0 ** np.round(np.log2(s))).astype(np.float32)  # noqa: E731
    return A, r(sA), B, r(sB)


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("kind", [0, 1, 2])
def test_gemm_f32_store_and_accumulate(fb, orc, kind, mode):
    """fp32 output (fp8bw_gemm_f32): a plain store into a strided buffer
    (columns past N untouched), then two accumulations onto a prior D, as for
    two micro-batches into an fp32 main gradient.  384 x 640 x 384: pair tiles
    with a ragged 128-row tail and a 128-column tail."""
    rng = np.random.default_rng(100 + 3 * kind + mode)
    M, N, K = 384, 640, 384
    ops = rand_ops(rng, M, N, K, kind)
    if mode == 1:
        ops = pow2_scales(ops)
    yr, ya = orc.gemm_ref_tile(kind, *ops, 0, M, 0, N)
    A, sA, B, sB = (dev(x) for x in ops)
    Dbig = torch.full((M, N + 64), float("nan"), dtype=torch.float32, device=DEV)
    D = Dbig[:, :N]
    fb.fp8bw_gemm_f32(kind, A, sA, B, sB, D, accumulate=False, mode=mode)
    torch.cuda.synchronize()
    assert fb.fp8bw_last_device_error() == 0
    bad, worst = orc.check_tol_f32(D.cpu().numpy(), yr, ya)
    assert bad == 0, worst
    assert torch.isnan(Dbig[:, N:]).all()
    D0 = (rng.standard_normal((M, N)) * np.abs(yr).mean()).astype(np.float32)
    Dacc = dev(D0)
    for _ in range(2):
        fb.fp8bw_gemm_f32(kind, A, sA, B, sB, Dacc, accumulate=True, mode=mode)
    torch.cuda.synchronize()
    assert fb.fp8bw_last_device_error() == 0
    bad, worst = orc.check_tol_f32(Dacc.cpu().numpy(), D0.astype(np.float64) + 2 * yr, 2 * ya)
    assert bad == 0, worst



@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("kind", [1, 2])
def test_e5m2_gradient_gemms(fb, orc, kind, mode):
    """dgrad / wgrad with E5M2 activation gradients (quantized by the oracle
    with the E5M2 rule) against E4M3 weights / activations: fp8bw_gemm_fmt
    within tolerance of the oracle's reference decoding A as E5M2."""
    X, W, dY = workloads.tiny(3)
    qx, sx, qxc, sxc = orc.quant_act_1x128(bits(X), mode)
    qw, sw, qwT = orc.quant_weight_128x128(bits(W), mode)
    qd, sd, qdc, sdc = orc.quant_act_1x128(bits(dY), mode, fmt=orc.FMT_E5M2)
    A, sA, B, sB = (qd, sd, qwT, sw) if kind == 1 else (qdc, sdc, qxc, sxc)
    M, N = A.shape[0], B.shape[0]
    D = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    fb.fp8bw_gemm_fmt(kind, dev(A), dev(sA), fb.FP8BW_FMT_E5M2, dev(B), dev(sB), fb.FP8BW_FMT_E4M3, D, mode)
    torch.cuda.synchronize()
    assert fb.fp8bw_last_device_error() == 0
    yr, ya = orc.gemm_ref_tile(kind, A, sA, B, sB, 0, M, 0, N, fa=orc.FMT_E5M2)
    bad, worst = orc.check_tol(bits(D), yr, ya)
    assert bad == 0, worst
    # read as E4M3 the same bytes give a different product: the format is used
    yr4, _ = orc.gemm_ref_tile(kind, A, sA, B, sB, 0, M, 0, N)
    assert not np.allclose(yr4, yr)

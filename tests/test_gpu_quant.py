"""GPU parity of the quantizers against the oracle: bytes and scale bits
must be identical.  Method: "NVIDIA NeMo RL erreicht 48% ..." section "Der
technische Durchbruch" (1x128 activation / 128x128 weight blocks, E4M3) and
"Leistungsgewinne in der Praxis" (per-step requantization)."""
import numpy as np
import pytest
import torch

import workloads
from util import act_buffers, assert_bytes_equal, bits, f32, from_bits, u8, weight_buffers

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_act(fb, x, mode, colwise=True):
    M, K = x.shape
    q_row, s_row, q_col, s_col = act_buffers(M, K, DEV, colwise)
    fb.fp8bw_quant_act_1x128(x, mode, q_row, s_row, q_col, s_col)
    torch.cuda.synchronize()
    return q_row, s_row, q_col, s_col


def check_act(fb, orc, x_cpu, mode, colwise=True):
    x = x_cpu.to(DEV)
    q_row, s_row, q_col, s_col = run_act(fb, x, mode, colwise)
    oq, os_, oqc, osc = orc.quant_act_1x128(bits(x_cpu), mode, colwise)
    assert_bytes_equal(u8(q_row), oq, "q_row")
    assert_bytes_equal(f32(s_row).view(np.uint32), os_.view(np.uint32), "s_row")
    if colwise:
        assert_bytes_equal(u8(q_col), oqc, "q_col")
        assert_bytes_equal(f32(s_col).view(np.uint32), osc.view(np.uint32), "s_col")


@pytest.mark.parametrize("mode", [0, 1])
def test_act_tiny(fb, orc, mode):
    X, _, dY = workloads.tiny(0)
    check_act(fb, orc, X, mode)
    check_act(fb, orc, dY, mode)
    check_act(fb, orc, X, mode, colwise=False)


@pytest.mark.parametrize("mode", [0, 1])
def test_act_shapes_and_edges(fb, orc, mode):
    g = torch.Generator().manual_seed(5)
    # single tile, several tiles with an odd tile count in both directions
    for M, K in [(128, 128), (384, 640), (640, 384)]:
        x = (torch.randn((M, K), generator=g) * 3).to(torch.bfloat16)
        check_act(fb, orc, x, mode)
    # edge blocks: all zero, -0, tiny (subnormal) values, huge values, mixed
    x = torch.zeros((256, 384), dtype=torch.float32)
    x[128:, :128] = -0.0
    x[:128, 128:256] = torch.randn((128, 128), generator=g) * 1e-39     # bf16 subnormals
    x[128:, 128:256] = torch.randn((128, 128), generator=g).clamp(-3, 3) * 1.1e38
    x[:, 256:] = torch.randn((256, 128), generator=g)
    x[5, 300] = 1e-30
    x[7, 301] = -2.0 ** -133
    x = x.to(torch.bfloat16)
    x[128:, :128] = -0.0
    check_act(fb, orc, x, mode)


def test_act_leading_dim(fb, orc):
    g = torch.Generator().manual_seed(9)
    big = torch.randn((256, 512 + 64), generator=g).to(torch.bfloat16).to(DEV)
    x = big[:, :512]
    q_row, s_row, q_col, s_col = act_buffers(256, 512, DEV)
    fb.fp8bw_quant_act_1x128(x, 0, q_row, s_row, q_col, s_col)
    torch.cuda.synchronize()
    oq, os_, oqc, osc = orc.quant_act_1x128(bits(x.cpu()), 0)
    assert_bytes_equal(u8(q_row), oq, "q_row")
    assert_bytes_equal(u8(q_col), oqc, "q_col")
    assert_bytes_equal(f32(s_col).view(np.uint32), osc.view(np.uint32), "s_col")


@pytest.mark.parametrize("mode", [0, 1])
def test_weight_tiny(fb, orc, mode):
    _, W, _ = workloads.tiny(0)
    q, s, qT = weight_buffers(*W.shape, DEV)
    fb.fp8bw_quant_weight_128x128(W.to(DEV), mode, q, s, qT)
    torch.cuda.synchronize()
    oq, os_, oqT = orc.quant_weight_128x128(bits(W), mode)
    assert_bytes_equal(u8(q), oq, "q")
    assert_bytes_equal(f32(s).view(np.uint32), os_.view(np.uint32), "s")
    assert_bytes_equal(u8(qT), oqT, "qT")


@pytest.mark.parametrize("mode", [0, 1])
def test_requant_batch(fb, orc, mode):
    g = torch.Generator().manual_seed(3)
    shapes = [(256, 384), (128, 128), (384, 256), (512, 128)]
    Ws = [(torch.randn(s, generator=g) * 0.02).to(torch.bfloat16).to(DEV) for s in shapes]
    Ws[1].zero_()
    outs = [weight_buffers(*w.shape, DEV, transposed=(i != 2)) for i, w in enumerate(Ws)]
    fb.fp8bw_requant_weights([(w, q, s, qT) for w, (q, s, qT) in zip(Ws, outs)], mode)
    torch.cuda.synchronize()
    for i, (w, (q, s, qT)) in enumerate(zip(Ws, outs)):
        oq, os_, oqT = orc.quant_weight_128x128(bits(w.cpu()), mode)
        assert_bytes_equal(u8(q), oq, f"q[{i}]")
        assert_bytes_equal(f32(s).view(np.uint32), os_.view(np.uint32), f"s[{i}]")
        if qT is not None:
            assert_bytes_equal(u8(qT), oqT, f"qT[{i}]")


@pytest.mark.parametrize("mode", [0, 1])
def test_act_e5m2(fb, orc, mode):
    """E5M2 codes (the gradient format of the per-tensor recipe, "FP8
    Trainingsinfrastructuur", "Het landschap van numerieke precisie") with
    the 57344 scale rule: bit-exact against the oracle, including zero, -0,
    subnormal and huge blocks."""
    _, _, dY = workloads.tiny(0)
    g = torch.Generator().manual_seed(12)
    edge = torch.zeros((256, 384), dtype=torch.float32)
    edge[:128, 128:256] = torch.randn((128, 128), generator=g) * 1e-39
    edge[128:, 128:256] = torch.randn((128, 128), generator=g).clamp(-3, 3) * 1.1e38
    edge[:, 256:] = torch.randn((256, 128), generator=g) * 1e-3
    edge = edge.to(torch.bfloat16)
    edge[128:, :128] = -0.0
    for x_cpu in (dY, edge):
        x = x_cpu.to(DEV)
        M, K = x.shape
        q_row, s_row, q_col, s_col = act_buffers(M, K, DEV)
        fb.fp8bw_quant_act_1x128_fmt(x, mode, fb.FP8BW_FMT_E5M2, q_row, s_row, q_col, s_col)
        torch.cuda.synchronize()
        oq, os_, oqc, osc = orc.quant_act_1x128(bits(x_cpu), mode, fmt=orc.FMT_E5M2)
        assert_bytes_equal(u8(q_row), oq, "q_row")
        assert_bytes_equal(f32(s_row).view(np.uint32), os_.view(np.uint32), "s_row")
        assert_bytes_equal(u8(q_col), oqc, "q_col")
        assert_bytes_equal(f32(s_col).view(np.uint32), osc.view(np.uint32), "s_col")


def _every_amax_input(seed):
    """[32768, 128] bf16: row i < 32639 is one 1x128 block whose magnitude
    maximum is the positive bf16 with bit pattern i + 1 (placed at column
    i % 128, sign random); the other elements have random magnitudes at or
    below it and random signs.  Rows past 32639 are zero."""
    rng = np.random.default_rng(seed)
    n = 0x7F7F
    top = np.arange(1, n + 1, dtype=np.uint32)
    x = np.zeros((32768, 128), np.uint16)
    mags = (rng.random((n, 128)) * (top[:, None] + 1)).astype(np.uint32)
    mags = np.minimum(mags, top[:, None])
    mags[np.arange(n), np.arange(n) % 128] = top
    signs = rng.integers(0, 2, (n, 128), dtype=np.uint32) << 15
    x[:n] = (mags | signs).astype(np.uint16)
    return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16), top


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("mode", [0, 1])
def test_act_every_bf16_amax(fb, orc, mode, fmt):
    """Every positive finite bf16 block amax through the activation
    quantizer: the row scales equal amax / qmax (one IEEE binary32 division)
    or the power-of-2 rule, and codes and scales of both copies are
    bit-exact against the oracle."""
    x_cpu, top = _every_amax_input(21 + fmt)
    x = x_cpu.to(DEV)
    M, K = x.shape
    q_row, s_row, q_col, s_col = act_buffers(M, K, DEV)
    fb.fp8bw_quant_act_1x128_fmt(x, mode, fmt, q_row, s_row, q_col, s_col)
    torch.cuda.synchronize()
    assert fb.fp8bw_last_device_error() == 0
    qmax = np.float32(448.0 if fmt == 0 else 57344.0)
    amax = (top << 16).view(np.float32)
    got = f32(s_row)[0, : len(top)]
    if mode == 0:
        assert np.array_equal(got.view(np.uint32), (amax / qmax).view(np.uint32))
    else:
        assert np.array_equal(got, np.array([orc.block_scale_fmt(float(a), 1, fmt) for a in amax],
                                            np.float32))
    oq, os_, oqc, osc = orc.quant_act_1x128(bits(x_cpu), mode, fmt=fmt)
    assert_bytes_equal(u8(q_row), oq, "q_row")
    assert_bytes_equal(f32(s_row).view(np.uint32), os_.view(np.uint32), "s_row")
    assert_bytes_equal(u8(q_col), oqc, "q_col")
    assert_bytes_equal(f32(s_col).view(np.uint32), osc.view(np.uint32), "s_col")

"""GPU parity of the per-tensor delayed-scaling quantizer against the oracle
(bytes, scale, amax and history bits identical) and of the per-tensor HYBRID
recipe's GEMMs (E4M3 forward, E5M2 gradients) through the blockwise GEMMs
with constant scale grids.  Recipe: "FP8 Trainingsinfrastructuur", sections
"Transformer Engine: de softwarebasis" and "Scaling-strategieën en
stabiliteit"."""
import numpy as np
import pytest
import torch

from util import assert_bytes_equal, bits, f32, u8

pytestmark = pytest.mark.gpu
DEV = "cuda"
E4M3, E5M2 = 0, 1


def run(fb, x, fmt, mode, hist, colwise=True, grid_len=0):
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.uint8, device=DEV)
    qT = torch.empty((K, M), dtype=torch.uint8, device=DEV) if colwise else None
    scale = torch.full((1,), -1.0, dtype=torch.float32, device=DEV)
    amax = torch.full((1,), -1.0, dtype=torch.float32, device=DEV)
    grid = torch.zeros((grid_len,), dtype=torch.float32, device=DEV) if grid_len else None
    fb.fp8bw_quant_tensor_delayed(x, fmt, mode, hist, q, qT, scale, amax, grid)
    torch.cuda.synchronize()
    assert fb.fp8bw_last_device_error() == 0
    return q, qT, scale, amax, grid


def check_step(fb, orc, x_cpu, fmt, mode, hist_dev, hist_cpu, colwise=True):
    q, qT, scale, amax, grid = run(fb, x_cpu.to(DEV), fmt, mode, hist_dev, colwise, grid_len=1000)
    oq, oqT, os_, oam, oh = orc.quant_tensor_delayed(bits(x_cpu), hist_cpu, mode, fmt, colwise)
    assert f32(scale).view(np.uint32)[0] == np.float32(os_).view(np.uint32)
    assert f32(amax).view(np.uint32)[0] == np.float32(oam).view(np.uint32)
    assert_bytes_equal(f32(hist_dev).view(np.uint32), oh.view(np.uint32), "history")
    assert np.all(f32(grid).view(np.uint32) == np.float32(os_).view(np.uint32))
    assert_bytes_equal(u8(q), oq, "q")
    if colwise:
        assert_bytes_equal(u8(qT), oqT, "qT")
    return oh


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
@pytest.mark.parametrize("mode", [0, 1])
def test_history_steps_bit_exact(fb, orc, fmt, mode):
    # 640 tiles: more than one grid-stride round on 148 SMs x 4 CTAs
    g = torch.Generator().manual_seed(21 + fmt + 2 * mode)
    M, K = 4096, 2560
    H = 3
    hist_cpu = np.zeros(H, np.float32)
    hist = torch.zeros(H, dtype=torch.float32, device=DEV)
    # magnitudes: a first step with no history (s = 1), a jump that
    # outgrows the history (saturation), a drop, and an outlier row
    for step, mag in enumerate([0.5, 8.0, 0.03, 2.0]):
        x = (torch.randn((M, K), generator=g) * mag)
        if step == 3:
            x[77, :] *= 300.0
        x = x.to(torch.bfloat16)
        hist_cpu = check_step(fb, orc, x, fmt, mode, hist, hist_cpu)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_shapes_rowwise_only_and_edges(fb, orc, fmt):
    g = torch.Generator().manual_seed(3)
    for M, K in [(128, 128), (384, 640), (640, 384)]:
        hist_cpu = np.array([1.5, 0.25], np.float32)
        hist = torch.from_numpy(hist_cpu.copy()).to(DEV)
        x = (torch.randn((M, K), generator=g) * 0.7).to(torch.bfloat16)
        check_step(fb, orc, x, fmt, 0, hist, hist_cpu)
        hist = torch.from_numpy(hist_cpu.copy()).to(DEV)
        check_step(fb, orc, x, fmt, 1, hist, hist_cpu, colwise=False)
    # subnormal, zero, -0 and huge values with a history that is far off
    x = torch.zeros((256, 256), dtype=torch.float32)
    x[:128, :128] = torch.randn((128, 128), generator=g) * 1e-39
    x[128:, 128:] = torch.randn((128, 128), generator=g).clamp(-3, 3) * 1.1e38
    x[5, 200] = -2.0 ** -133
    x = x.to(torch.bfloat16)
    x[200:, :64] = -0.0
    for h in ([0.0], [1e-30], [3e38], [7.0, float("nan")]):
        hist_cpu = np.array(h, np.float32)
        check_step(fb, orc, x, fmt, 0, torch.from_numpy(hist_cpu.copy()).to(DEV), hist_cpu)
        check_step(fb, orc, x, fmt, 1, torch.from_numpy(hist_cpu.copy()).to(DEV), hist_cpu)


def test_nan_is_not_an_amax(fb, orc):
    x = torch.ones((128, 256), dtype=torch.bfloat16)
    x[3, 4] = float("nan")
    x[9, 9] = -5.0
    hist = torch.tensor([2.0], dtype=torch.float32, device=DEV)
    q, _, scale, amax, _ = run(fb, x.to(DEV), E4M3, 0, hist)
    assert float(amax) == 5.0 and float(hist[0]) == 5.0
    oq, _, os_, _, _ = orc.quant_tensor_delayed(bits(x), np.array([2.0], np.float32), 0)
    got = u8(q)
    assert got[3, 4] & 0x7F == 0x7F
    got[3, 4] = oq[3, 4]
    assert_bytes_equal(got, oq, "q")


def test_empty_tensor_still_sets_scale_and_pushes(fb, orc):
    x = torch.empty((0, 256), dtype=torch.bfloat16, device=DEV)
    hist = torch.tensor([3.0, 9.0], dtype=torch.float32, device=DEV)
    q, qT, scale, amax, grid = run(fb, x, E4M3, 0, hist, grid_len=300)
    assert float(scale) == float(np.float32(9.0) / np.float32(448.0))
    assert float(amax) == 0.0
    assert f32(hist).tolist() == [0.0, 3.0]
    assert np.all(f32(grid) == f32(scale)[0])


def test_full_size_dy_gate_up_sampled(fb, orc):
    # dY of the gate_up layer at 8192 tokens: [8192, 28672]
    M, K = 8192, 28672
    g = torch.Generator(device=DEV).manual_seed(8)
    x = (torch.randn((M, K), generator=g, device=DEV) * 1e-3).to(torch.bfloat16)
    hist_cpu = np.array([0.004, 0.006, 0.005], np.float32)
    hist = torch.from_numpy(hist_cpu.copy()).to(DEV)
    q, qT, scale, amax, _ = run(fb, x, E5M2, 0, hist)
    assert torch.equal(qT, q.t())
    rows = np.linspace(0, M - 1, 48).astype(np.int64)
    xs = x[torch.from_numpy(rows).to(DEV)].cpu()
    oq, _, os_, _, _ = orc.quant_tensor_delayed(bits(xs), hist_cpu, 0, E5M2, transposed=False)
    assert f32(scale)[0] == os_
    assert_bytes_equal(u8(q[torch.from_numpy(rows).to(DEV)]), oq, "sampled rows")
    # no NaN in x: the largest |x| is the largest magnitude bit pattern
    top = np.array([(bits(x) & 0x7FFF).max()], np.uint32)
    want_amax = (top << 16).view(np.float32)[0]
    assert f32(amax)[0] == want_amax and f32(hist)[0] == want_amax


@pytest.mark.parametrize("mode", [0, 1])
def test_hybrid_recipe_gemms(fb, orc, mode):
    # The per-tensor HYBRID recipe: X and W in E4M3, dY in E5M2, every operand
    # with one delayed scale, the three GEMMs through the blockwise GEMMs with
    # constant scale grids.
    g = torch.Generator().manual_seed(13)
    M, N, K = 384, 256, 512
    X = (torch.randn((M, K), generator=g)).to(torch.bfloat16)
    W = (torch.randn((N, K), generator=g) * 0.02).to(torch.bfloat16)
    dY = (torch.randn((M, N), generator=g) * 1e-4).to(torch.bfloat16)
    ops = {}
    for name, t, fmt, grid_len, h in [("x", X, E4M3, M * K // 128, 4.5),
                                      ("w", W, E4M3, N * K // 16384, 0.09),
                                      ("dy", dY, E5M2, M * N // 128, 3e-4)]:
        hist_cpu = np.array([h, h / 2], np.float32)
        hist = torch.from_numpy(hist_cpu.copy()).to(DEV)
        q, qT, scale, amax, grid = run(fb, t.to(DEV), fmt, mode, hist, grid_len=grid_len)
        oq, oqT, os_, _, _ = orc.quant_tensor_delayed(bits(t), hist_cpu, mode, fmt)
        assert_bytes_equal(u8(q), oq, name)
        ops[name] = (q, qT, grid, oq, oqT, np.full(grid_len, os_, np.float32), fmt)
    qx, qxT, gx, oqx, oqxT, ogx, _ = ops["x"]
    qw, qwT, gw, oqw, oqwT, ogw, _ = ops["w"]
    qd, qdT, gd, oqd, oqdT, ogd, _ = ops["dy"]
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=DEV)
    dW = torch.empty((N, K), dtype=torch.bfloat16, device=DEV)
    fb.fp8bw_gemm_fmt(fb.FP8BW_FPROP, qx, gx, E4M3, qw, gw, E4M3, Y, mode)
    fb.fp8bw_gemm_fmt(fb.FP8BW_DGRAD, qd, gd, E5M2, qwT, gw, E4M3, dX, mode)
    fb.fp8bw_gemm_fmt(fb.FP8BW_WGRAD, qdT, gd, E5M2, qxT, gx, E4M3, dW, mode)
    torch.cuda.synchronize()
    assert fb.fp8bw_last_device_error() == 0
    cases = [("fprop", Y, 0, oqx, ogx.reshape(K // 128, M), oqw, ogw.reshape(N // 128, K // 128), E4M3, E4M3),
             ("dgrad", dX, 1, oqd, ogd.reshape(N // 128, M), oqwT, ogw.reshape(K // 128, N // 128), E5M2, E4M3),
             ("wgrad", dW, 2, oqdT, ogd.reshape(M // 128, N), oqxT, ogx.reshape(M // 128, K), E5M2, E4M3)]
    for name, out, kind, A, sA, B, sB, fa, fbm in cases:
        yr, ya = orc.gemm_ref_tile(kind, A, sA, B, sB, 0, A.shape[0], 0, B.shape[0], fa=fa, fb=fbm)
        bad, worst = orc.check_tol(bits(out), yr, ya)
        assert bad == 0, (name, bad, worst)

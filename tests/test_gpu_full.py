"""Full-size GPU parity, in the launch configurations the benchmark uses, in
both scale modes (FP32 scales on the promotion kernel, power-of-2 scales on
the tensor core's block-scaled MMA).

Workloads (seeded, synthetic, shaped like the pages' models — "NVIDIA NeMo
RL erreicht 48% ...": Llama 3.1 8B, scales recalibrated every step,
optional power-of-2 scales; "NeMo-RL v0.3 mit Megatron-Core ...": sequence
packing, 16K-token contexts):
  * Llama-3.1-8B-like linear layers, 8192 tokens, 0.1% outlier channels x50;
  * a packed long-sequence batch (4 sequences, 32768 tokens, Student-t
    activations, zero padding rows) on all four layer shapes;
  * the per-step requant sweep of 32 layers of those weights (Adam-like
    N(0, 1e-4^2) update, 10 steps).
The oracle recomputes sampled 128x128 quantizer tiles (bit-exact) and
sampled 128x128 GEMM output tiles (tolerance) one by one: the four corner
tiles, 16 seeded random tiles, tiles over outlier channels and tiles over
zero padding rows, for every GEMM."""
import numpy as np
import pytest
import torch

import workloads
from util import act_buffers, assert_bytes_equal, bits, weight_buffers

pytestmark = pytest.mark.gpu
DEV = "cuda"
T = 128          # side of a sampled tile
N_RANDOM = 16    # seeded random GEMM tiles per GEMM


def np_u8(t):
    return t.cpu().numpy()


def check_act_tiles(orc, x, q_row, s_row, q_col, s_col, tiles, mode=0):
    """Oracle on sampled 128x128 tiles of x (tile-aligned blocks are local)."""
    qr, sr, qc, sc = np_u8(q_row), s_row.cpu().numpy(), np_u8(q_col), s_col.cpu().numpy()
    for (m0, k0) in tiles:
        xt = bits(x[m0:m0 + 128, k0:k0 + 128])
        oq, os_, oqc, osc = orc.quant_act_1x128(xt, mode)
        assert_bytes_equal(qr[m0:m0 + 128, k0:k0 + 128], oq, f"q_row tile {m0},{k0}")
        assert_bytes_equal(sr[k0 // 128, m0:m0 + 128].view(np.uint32)[None], os_.view(np.uint32), "s_row")
        assert_bytes_equal(qc[k0:k0 + 128, m0:m0 + 128], oqc, f"q_col tile {m0},{k0}")
        assert_bytes_equal(sc[m0 // 128, k0:k0 + 128].view(np.uint32)[None], osc.view(np.uint32), "s_col")


def check_weight_blocks(orc, w, q, s, qT, blocks, mode=0):
    qh, sh = np_u8(q), s.cpu().numpy()
    qTh = np_u8(qT) if qT is not None else None
    for (n0, k0) in blocks:
        oq, os_, oqT = orc.quant_weight_128x128(bits(w[n0:n0 + 128, k0:k0 + 128]), mode)
        assert_bytes_equal(qh[n0:n0 + 128, k0:k0 + 128], oq, f"q block {n0},{k0}")
        assert sh[n0 // 128, k0 // 128].view(np.uint32) == os_.view(np.uint32)[0, 0]
        if qTh is not None:
            assert_bytes_equal(qTh[k0:k0 + 128, n0:n0 + 128], oqT, f"qT block {n0},{k0}")


def sample_tiles(rng, M, N, n, extra=()):
    t = [(0, 0), (M - 128, N - 128)] + list(extra)
    t += [(128 * int(rng.integers(0, M // 128)), 128 * int(rng.integers(0, N // 128))) for _ in range(n)]
    return t


def gemm_tiles(rng, M, N, rows=(), cols=()):
    """128x128 output tiles: the four corners, N_RANDOM seeded random tiles,
    a tile in the block row of every row in `rows` and in the block column
    of every column in `cols` (random along the other axis)."""
    t = [(0, 0), (M - T, N - T), (M - T, 0), (0, N - T)]
    t += [(T * int(rng.integers(0, M // T)), T * int(rng.integers(0, N // T))) for _ in range(N_RANDOM)]
    t += [((r // T) * T, T * int(rng.integers(0, N // T))) for r in rows]
    t += [(T * int(rng.integers(0, M // T)), (c // T) * T) for c in cols]
    return list(dict.fromkeys(t))


def check_gemm_tiles(orc, kind, A, sA, B, sB, D, tiles):
    """Every element of each 128x128 tile within the acceptance gate
    |y - y_ref| <= 1e-2 sum|a b| + 1 bf16 ulp(y_ref)."""
    Ah, sAh, Bh, sBh, Dh = np_u8(A), sA.cpu().numpy(), np_u8(B), sB.cpu().numpy(), bits(D)
    for (m0, n0) in tiles:
        y, ya = orc.gemm_ref_tile(kind, Ah, sAh, Bh, sBh, m0, m0 + T, n0, n0 + T)
        bad, worst = orc.check_tol(np.ascontiguousarray(Dh[m0:m0 + T, n0:n0 + T]), y, ya)
        assert bad == 0, (kind, m0, n0, worst)


def run_layer(fb, orc, X, W, dY, rng, mode=0, outlier_cols=(), pad_rows=()):
    M, K = X.shape
    N = W.shape[0]
    qx, sx, qxc, sxc = act_buffers(M, K, DEV)
    qd, sd, qdc, sdc = act_buffers(M, N, DEV)
    qw, sw, qwT = weight_buffers(N, K, DEV)
    fb.fp8bw_quant_act_1x128(X, mode, qx, sx, qxc, sxc)
    fb.fp8bw_quant_act_1x128(dY, mode, qd, sd, qdc, sdc)
    fb.fp8bw_requant_weights([(W, qw, sw, qwT)], mode)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=DEV)
    dW = torch.empty((N, K), dtype=torch.bfloat16, device=DEV)
    fb.fp8bw_gemm(0, qx, sx, qw, sw, Y, mode)
    fb.fp8bw_gemm(1, qd, sd, qwT, sw, dX, mode)
    fb.fp8bw_gemm(2, qdc, sdc, qxc, sxc, dW, mode)
    torch.cuda.synchronize()
    assert fb.fp8bw_last_device_error() == 0
    extra = [((r // 128) * 128, 128 * int(rng.integers(0, K // 128))) for r in pad_rows]
    extra += [(128 * int(rng.integers(0, M // 128)), (c // 128) * 128) for c in outlier_cols]
    check_act_tiles(orc, X, qx, sx, qxc, sxc, sample_tiles(rng, M, K, 6, extra), mode)
    check_act_tiles(orc, dY, qd, sd, qdc, sdc, sample_tiles(rng, M, N, 4), mode)
    check_weight_blocks(orc, W, qw, sw, qwT, sample_tiles(rng, N, K, 6), mode)
    check_gemm_tiles(orc, 0, qx, sx, qw, sw, Y, gemm_tiles(rng, M, N, rows=pad_rows))
    check_gemm_tiles(orc, 1, qd, sd, qwT, sw, dX, gemm_tiles(rng, M, K, rows=pad_rows, cols=outlier_cols))
    check_gemm_tiles(orc, 2, qdc, sdc, qxc, sxc, dW, gemm_tiles(rng, N, K, cols=outlier_cols))
    return Y, dX


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("name", [n for n, _, _ in workloads.LLAMA8B_LAYERS])
def test_llama8b_layer(fb, orc, name, mode):
    X, W, dY = workloads.llama_layer(name, seed=0, device=DEV)
    idx = [n for n, _, _ in workloads.LLAMA8B_LAYERS].index(name)
    K = workloads.LLAMA8B_LAYERS[idx][1]
    outl = workloads.outlier_channels(K, 0 * 1000 + idx * 10 + 1)
    rng = np.random.default_rng(idx + 10 * mode)
    run_layer(fb, orc, X, W, dY, rng, mode, outlier_cols=outl)


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("name", [n for n, _, _ in workloads.LLAMA8B_LAYERS])
def test_packed_long_sequence(fb, orc, name, mode):
    """4 packed sequences, 32768 tokens, heavy-tailed activations and zero
    padding rows on every Llama-like layer shape: padding rows give all-zero
    blocks (scale 1, zero codes) and exact zeros in fprop and dgrad."""
    idx = [n for n, _, _ in workloads.LLAMA8B_LAYERS].index(name)
    _, K, N = workloads.LLAMA8B_LAYERS[idx]
    mask = workloads.packed_rows_mask(0)
    X = workloads.packed_activations(K, 0, DEV)
    dY = workloads.packed_activations(N, 1, DEV, scale=1e-3)
    W = workloads.llama_weight(name, 0, device=DEV)
    pad = np.nonzero(~mask.numpy())[0]
    rng = np.random.default_rng(5 + idx + 10 * mode)
    pad_rows = sorted({int(pad[0]), int(pad[len(pad) // 2]), int(pad[-1])}) if pad.size else []
    Y, dX = run_layer(fb, orc, X, W, dY, rng, mode, pad_rows=pad_rows)
    if pad.size:
        rows = torch.from_numpy(pad).to(DEV)
        assert torch.all(Y[rows] == 0) and torch.all(dX[rows] == 0)


@pytest.mark.parametrize("mode", [0, 1])
def test_requant_sweep(fb, orc, mode):
    """32 layers x 4 weights (about 7B bf16 parameters), Adam-like update
    N(0, 1e-4^2) and one batched requant per step for 10 steps; step 0 and
    step 9 are checked on sampled blocks, and the batched call must equal the
    single-weight call bit for bit."""
    layers = 32
    names = [(n, K, N) for n, K, N in workloads.LLAMA8B_LAYERS]
    Ws, outs = [], []
    for l in range(layers):
        for (n, K, N) in names:
            Ws.append(workloads.llama_weight(n, l, device=DEV))
            outs.append(weight_buffers(N, K, DEV))
    items = [(w, q, s, qT) for w, (q, s, qT) in zip(Ws, outs)]
    rng = np.random.default_rng(9 + mode)
    for step in range(10):
        if step > 0:
            for i, w in enumerate(Ws):
                workloads.requant_update_(w, step, i // 4, i % 4)
        fb.fp8bw_requant_weights(items, mode)
        torch.cuda.synchronize()
        assert fb.fp8bw_last_device_error() == 0
        if step in (0, 9):
            for i in rng.choice(len(Ws), 6, replace=False):
                w, (q, s, qT) = Ws[i], outs[i]
                check_weight_blocks(orc, w, q, s, qT, sample_tiles(rng, *w.shape, 3), mode)
        else:
            i = int(rng.integers(0, len(Ws)))
            w, (q, s, qT) = Ws[i], outs[i]
            check_weight_blocks(orc, w, q, s, qT, sample_tiles(rng, *w.shape, 1), mode)
    # batched == single call, on two of the largest weights
    for i in (2, 6):
        q, s, qT = weight_buffers(*Ws[i].shape, DEV)
        fb.fp8bw_quant_weight_128x128(Ws[i], mode, q, s, qT)
        torch.cuda.synchronize()
        assert torch.equal(q, outs[i][0]) and torch.equal(qT, outs[i][2])
        assert torch.equal(s.view(torch.int32), outs[i][1].view(torch.int32))


def test_wgrad_accumulates_into_fp32_main_grad(fb, orc):
    """Gradient accumulation over two micro-batches of the down layer
    (8192 tokens each, 14336 -> 4096): dW of each is added to an fp32 main
    gradient by fp8bw_gemm_f32(accumulate); sampled 128x128 tiles are
    checked against main_grad0 + the fp64 references of both micro-batches."""
    name, K, N = workloads.LLAMA8B_LAYERS[3]
    M = workloads.LLAMA8B_TOKENS
    rng = np.random.default_rng(77)
    main = torch.randn((N, K), generator=torch.Generator(device=DEV).manual_seed(5), device=DEV) * 1e-2
    main0 = main.cpu().numpy().astype(np.float64)
    ops = []
    for mb in range(2):
        X, _, dY = workloads.llama_layer(name, seed=10 + mb, device=DEV, M=M)
        qx, sx, qxc, sxc = act_buffers(M, K, DEV)
        qd, sd, qdc, sdc = act_buffers(M, N, DEV)
        fb.fp8bw_quant_act_1x128(X, 0, qx, sx, qxc, sxc)
        fb.fp8bw_quant_act_1x128(dY, 0, qd, sd, qdc, sdc)
        fb.fp8bw_gemm_f32(2, qdc, sdc, qxc, sxc, main, accumulate=True)
        ops.append((qdc, sdc, qxc, sxc))
    torch.cuda.synchronize()
    assert fb.fp8bw_last_device_error() == 0
    got = main.cpu().numpy()
    host = [tuple(np_u8(t) if t.dtype == torch.uint8 else t.cpu().numpy() for t in o) for o in ops]
    for (m0, n0) in gemm_tiles(rng, N, K):
        ref = main0[m0:m0 + T, n0:n0 + T].copy()
        yabs = np.zeros((T, T))
        for A, sA, B, sB in host:
            y, ya = orc.gemm_ref_tile(2, A, sA, B, sB, m0, m0 + T, n0, n0 + T)
            ref += y
            yabs += ya
        bad, worst = orc.check_tol_f32(got[m0:m0 + T, n0:n0 + T], ref, yabs)
        assert bad == 0, (m0, n0, worst)

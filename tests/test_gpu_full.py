"""Full-size GPU parity, in the launch configurations the benchmark uses.

Workloads (seeded, synthetic, shaped like the pages' models — "NVIDIA NeMo
RL erreicht 48% ...": Llama 3.1 8B; "NeMo-RL v0.3 mit Megatron-Core ...":
sequence packing, 16K-token contexts):
  * Llama-3.1-8B-like linear layers, 8192 tokens, 0.1% outlier channels x50;
  * the per-step requant sweep of 32 layers of those weights (Adam-like
    N(0, 1e-4^2) update, 10 steps);
  * a packed long-sequence batch (4 sequences, 32768 tokens, Student-t
    activations, zero-padding blocks).
The oracle recomputes sampled 128x128 quantizer tiles (bit-exact) and
sampled 32x32 GEMM output tiles (tolerance) one by one."""
import numpy as np
import pytest
import torch

import workloads
from util import act_buffers, assert_bytes_equal, bits, weight_buffers

pytestmark = pytest.mark.gpu
DEV = "cuda"


def np_u8(t):
    return t.cpu().numpy()


def check_act_tiles(orc, x, q_row, s_row, q_col, s_col, tiles, mode=0):
    """Oracle on sampled 128x128 tiles of x (tile-aligned blocks are local)."""
    M, K = x.shape
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


def check_gemm_tiles(orc, kind, A, sA, B, sB, D, pts):
    """pts: (m0, n0) corners of 32x32 output tiles."""
    Ah, sAh, Bh, sBh, Dh = np_u8(A), sA.cpu().numpy(), np_u8(B), sB.cpu().numpy(), bits(D)
    for (m0, n0) in pts:
        y, ya = orc.gemm_ref_tile(kind, Ah, sAh, Bh, sBh, m0, m0 + 32, n0, n0 + 32)
        bad, worst = orc.check_tol(np.ascontiguousarray(Dh[m0:m0 + 32, n0:n0 + 32]), y, ya)
        assert bad == 0, (kind, m0, n0, worst)


def gemm_points(rng, M, N, n, extra_cols=()):
    p = [(0, 0), (M - 32, N - 32), (M - 32, 0), (0, N - 32)]
    p += [(32 * int(rng.integers(0, M // 32)), 32 * int(rng.integers(0, N // 32))) for _ in range(n)]
    p += [(32 * int(rng.integers(0, M // 32)), (c // 32) * 32) for c in extra_cols]
    return p


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
    check_act_tiles(orc, X, qx, sx, qxc, sxc, sample_tiles(rng, M, K, 6, extra))
    check_act_tiles(orc, dY, qd, sd, qdc, sdc, sample_tiles(rng, M, N, 4))
    check_weight_blocks(orc, W, qw, sw, qwT, sample_tiles(rng, N, K, 6))
    check_gemm_tiles(orc, 0, qx, sx, qw, sw, Y, gemm_points(rng, M, N, 5))
    check_gemm_tiles(orc, 1, qd, sd, qwT, sw, dX, gemm_points(rng, M, K, 5, outlier_cols))
    check_gemm_tiles(orc, 2, qdc, sdc, qxc, sxc, dW, gemm_points(rng, N, K, 5, outlier_cols))
    return Y, dX


@pytest.mark.parametrize("name", [n for n, _, _ in workloads.LLAMA8B_LAYERS])
def test_llama8b_layer(fb, orc, name):
    X, W, dY = workloads.llama_layer(name, seed=0, device=DEV)
    idx = [n for n, _, _ in workloads.LLAMA8B_LAYERS].index(name)
    K = workloads.LLAMA8B_LAYERS[idx][1]
    outl = workloads.outlier_channels(K, 0 * 1000 + idx * 10 + 1)
    rng = np.random.default_rng(idx)
    run_layer(fb, orc, X, W, dY, rng, outlier_cols=outl[:2])


def test_packed_long_sequence(fb, orc):
    """4 packed sequences, 32768 tokens, heavy-tailed activations and zero
    padding rows: padding rows give all-zero blocks (scale 1, zero codes) and
    exact zeros in the forward output."""
    name, K, N = workloads.LLAMA8B_LAYERS[0]
    M = workloads.PACKED_TOKENS
    mask = workloads.packed_rows_mask(0)
    X = workloads.packed_activations(K, 0, DEV)
    dY = workloads.packed_activations(N, 1, DEV, scale=1e-3)
    W = workloads.llama_weight(name, 0, device=DEV)
    pad = np.nonzero(~mask.numpy())[0]
    rng = np.random.default_rng(5)
    pad_rows = [int(pad[0]), int(pad[-1])] if pad.size else []
    Y, _ = run_layer(fb, orc, X, W, dY, rng, pad_rows=pad_rows)
    if pad.size:
        assert torch.all(Y[torch.from_numpy(pad).to(DEV)] == 0)


def test_requant_sweep(fb, orc):
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
    rng = np.random.default_rng(9)
    for step in range(10):
        if step > 0:
            for i, w in enumerate(Ws):
                workloads.requant_update_(w, step, i // 4, i % 4)
        fb.fp8bw_requant_weights(items, 0)
        torch.cuda.synchronize()
        assert fb.fp8bw_last_device_error() == 0
        if step in (0, 9):
            for i in rng.choice(len(Ws), 6, replace=False):
                w, (q, s, qT) = Ws[i], outs[i]
                check_weight_blocks(orc, w, q, s, qT, sample_tiles(rng, *w.shape, 3))
    # batched == single call, on two of the largest weights
    for i in (2, 6):
        q, s, qT = weight_buffers(*Ws[i].shape, DEV)
        fb.fp8bw_quant_weight_128x128(Ws[i], 0, q, s, qT)
        torch.cuda.synchronize()
        assert torch.equal(q, outs[i][0]) and torch.equal(qT, outs[i][2])
        assert torch.equal(s.view(torch.int32), outs[i][1].view(torch.int32))


def test_wgrad_accumulates_into_fp32_main_grad(fb, orc):
    """Gradient accumulation over two micro-batches of the down layer
    (8192 tokens each, 14336 -> 4096): dW of each is added to an fp32 main
    gradient by fp8bw_gemm_f32(accumulate); sampled 32x32 tiles are checked
    against main_grad0 + the fp64 references of both micro-batches."""
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
    for (m0, n0) in gemm_points(rng, N, K, 8):
        ref = main0[m0:m0 + 32, n0:n0 + 32].copy()
        yabs = np.zeros((32, 32))
        for A, sA, B, sB in host:
            y, ya = orc.gemm_ref_tile(2, A, sA, B, sB, m0, m0 + 32, n0, n0 + 32)
            ref += y
            yabs += ya
        bad, worst = orc.check_tol_f32(got[m0:m0 + 32, n0:n0 + 32], ref, yabs)
        assert bad == 0, (m0, n0, worst)

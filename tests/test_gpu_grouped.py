"""GPU parity of the grouped (mixture-of-experts) blockwise FP8 GEMM against
the oracle.  Method: "NVIDIA NeMo RL erreicht 48% ..." section
"Leistungsgewinne in der Praxis" (the recipe trains the Qwen3-30B MoE model
with the same FP8 linear layers).  Tokens are grouped by expert, each
segment zero-padded to a multiple of 128 rows."""
import numpy as np
import pytest
import torch

import workloads
from util import bits

pytestmark = pytest.mark.gpu
DEV = "cuda"


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def moe_case(orc, seed, lens, K, N, mode):
    """Permuted tokens (zero-padded segments), expert weights and dY, all
    quantized by the oracle.  Returns every operand the three GEMMs need."""
    g = torch.Generator().manual_seed(seed)
    pad = [((l + 127) // 128) * 128 for l in lens]
    off = np.concatenate([[0], np.cumsum(pad)]).astype(np.int32)
    Mtot = int(off[-1]) + 128          # a tail of rows beyond the last expert
    G = len(lens)
    X = torch.zeros((Mtot, K), dtype=torch.float32)
    dY = torch.zeros((Mtot, N), dtype=torch.float32)
    for e, l in enumerate(lens):
        X[off[e]:off[e] + l] = torch.randn((l, K), generator=g)
        dY[off[e]:off[e] + l] = torch.randn((l, N), generator=g) * 1e-3
    X, dY = X.to(torch.bfloat16), dY.to(torch.bfloat16)
    W = (torch.randn((G, N, K), generator=g) * 0.02).to(torch.bfloat16)
    qx, sx, qxc, sxc = orc.quant_act_1x128(bits(X), mode)
    qd, sd, qdc, sdc = orc.quant_act_1x128(bits(dY), mode)
    qw = np.empty((G, N, K), np.uint8)
    qwT = np.empty((G, K, N), np.uint8)
    sw = np.empty((G, N // 128, K // 128), np.float32)
    for e in range(G):
        qw[e], sw[e], qwT[e] = orc.quant_weight_128x128(bits(W[e]), mode)
    return dict(off=off, Mtot=Mtot, G=G, qx=qx, sx=sx, qxc=qxc, sxc=sxc, qd=qd, sd=sd, qdc=qdc,
                sdc=sdc, qw=qw, sw=sw, qwT=qwT)


def run_grouped(fb, kind, c, mode, D_shape):
    off = dev(c["off"])
    if kind == 0:
        A, sA, B, sB = c["qx"], c["sx"], c["qw"], c["sw"]
    elif kind == 1:
        A, sA, B, sB = c["qd"], c["sd"], c["qwT"], c["sw"]
    else:
        A, sA, B, sB = c["qdc"], c["sdc"], c["qxc"], c["sxc"]
    D = torch.full(D_shape, float("nan"), dtype=torch.bfloat16, device=DEV)
    fb.fp8bw_grouped_gemm(kind, off, dev(A), dev(sA), dev(B), dev(sB), D, mode)
    torch.cuda.synchronize()
    assert fb.fp8bw_last_device_error() == 0
    return D, (A, sA, B, sB)


@pytest.mark.parametrize("mode", [0, 1])
def test_grouped_small(fb, orc, mode):
    lens = [300, 0, 128, 1, 517, 0, 256, 77]          # empty experts and ragged segments
    K, N = 256, 384
    c = moe_case(orc, 11 + mode, lens, K, N, mode)
    off, Mtot, G = c["off"], c["Mtot"], c["G"]
    # fprop: Y = X W_g^T per segment;  dgrad: dX = dY W_g
    for kind, Nout, Kin in [(0, N, K), (1, K, N)]:
        D, ops = run_grouped(fb, kind, c, mode, (Mtot, Nout))
        y, ya = orc.grouped_gemm_ref_tile(kind, off, *ops, 0, 0, int(off[-1]), 0, Nout)
        bad, worst = orc.check_tol(bits(D)[:int(off[-1])], y, ya)
        assert bad == 0, (kind, worst)
        # rows past the last expert are not part of the result: untouched
        assert torch.isnan(D[int(off[-1]):].float()).all()
    # wgrad: dW_g = dY_g^T X_g over the expert's own tokens; empty experts -> 0
    D, ops = run_grouped(fb, 2, c, mode, (G, N, K))
    for e in range(G):
        y, ya = orc.grouped_gemm_ref_tile(2, off, *ops, e, 0, N, 0, K)
        bad, worst = orc.check_tol(bits(D[e]), y, ya)
        assert bad == 0, (e, worst)
        if lens[e] == 0:
            assert torch.all(D[e] == 0)


def test_grouped_bad_offsets(fb, orc):
    """Offsets that are not multiples of 128 are rejected on the device: the
    kernel writes nothing and latches FP8BW_ERR_DEVICE_CHECK."""
    lens = [128, 256]
    c = moe_case(orc, 3, lens, 128, 128, 0)
    bad = np.array([0, 100, 384], np.int32)
    D = torch.full((c["Mtot"], 128), 7.0, dtype=torch.bfloat16, device=DEV)
    fb.fp8bw_grouped_gemm(0, dev(bad), dev(c["qx"]), dev(c["sx"]), dev(c["qw"]), dev(c["sw"]), D, 0)
    assert fb.fp8bw_last_device_error() == 6
    assert torch.all(D == 7.0)
    assert fb.fp8bw_last_device_error() == 0   # the error word was cleared


MOE_SHAPES = {"gate_up": (workloads.MOE_HIDDEN, 2 * workloads.MOE_INTER),
              "down": (workloads.MOE_INTER, workloads.MOE_HIDDEN)}


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("layer", ["gate_up", "down"])
def test_grouped_moe_full_size_sampled(fb, orc, layer, mode):
    """Qwen3-30B-A3B-like expert layers (gate_up 2048 -> 1536 and down
    768 -> 2048, 128 experts, top-8 of 16384 tokens, Zipf(1.1) popularity)
    at full size, in the launch configuration the benchmark uses, in both
    scale modes: fprop, dgrad and wgrad.  Checked against the oracle: one
    128x128 output tile per expert for each GEMM (smallest and largest
    experts included), a tile over each expert's zero padding rows (exact
    zeros in fprop and dgrad), 16 seeded random tiles, and sampled
    quantizer tiles (bit-exact)."""
    r = workloads.moe_routing(0)
    G = workloads.MOE_EXPERTS
    K, N = MOE_SHAPES[layer]
    seeds = {"gate_up": (5, 6, 7), "down": (15, 16, 17)}[layer]
    X = workloads.moe_permuted(r, K, 1.0, seed=seeds[0], device=DEV)
    W = workloads.moe_experts(G, N, K, seed=seeds[1], device=DEV)
    dY = workloads.moe_permuted(r, N, 1e-3, seed=seeds[2], device=DEV)
    Mtot = r.m_total_pad
    u8, f32 = torch.uint8, torch.float32
    e = lambda *sh, dt=u8: torch.empty(sh, dtype=dt, device=DEV)  # noqa: E731
    qx, sx, qxc, sxc = e(Mtot, K), e(K // 128, Mtot, dt=f32), e(K, Mtot), e(Mtot // 128, K, dt=f32)
    qd, sd, qdc, sdc = e(Mtot, N), e(N // 128, Mtot, dt=f32), e(N, Mtot), e(Mtot // 128, N, dt=f32)
    qw, sw, qwT = e(G, N, K), e(G, N // 128, K // 128, dt=f32), e(G, K, N)
    fb.fp8bw_quant_act_1x128(X, mode, qx, sx, qxc, sxc)
    fb.fp8bw_quant_act_1x128(dY, mode, qd, sd, qdc, sdc)
    fb.fp8bw_requant_weights([(W[g], qw[g], sw[g], qwT[g]) for g in range(G)], mode)
    off = torch.tensor(r.offsets, dtype=torch.int32, device=DEV)
    bf = torch.bfloat16
    Y, dX, dW = e(Mtot, N, dt=bf), e(Mtot, K, dt=bf), e(G, N, K, dt=bf)
    fb.fp8bw_grouped_gemm(0, off, qx, sx, qw, sw, Y, mode)
    fb.fp8bw_grouped_gemm(1, off, qd, sd, qwT, sw, dX, mode)
    fb.fp8bw_grouped_gemm(2, off, qdc, sdc, qxc, sxc, dW, mode)
    torch.cuda.synchronize()
    assert fb.fp8bw_last_device_error() == 0

    rng = np.random.default_rng(100 + 10 * mode + (layer == "down"))
    counts = np.array(r.counts)
    offs = np.array(r.offsets, np.int32)
    h = lambda t: t.cpu().numpy()  # noqa: E731
    qx_h, sx_h, qxc_h, sxc_h = h(qx), h(sx), h(qxc), h(sxc)
    qd_h, sd_h, qdc_h, sdc_h = h(qd), h(sd), h(qdc), h(sdc)
    qw_h, sw_h, qwT_h = h(qw), h(sw), h(qwT)

    # quantizers: tiles at expert boundaries and random tiles, bit-exact
    for (m0, k0) in [(int(offs[g]), 0) for g in rng.choice(G, 4, replace=False) if counts[g]] + \
            [(128 * int(rng.integers(0, Mtot // 128)), 128 * int(rng.integers(0, K // 128)))]:
        oq, os_, oqc, osc = orc.quant_act_1x128(bits(X[m0:m0 + 128, k0:k0 + 128]), mode)
        assert np.array_equal(qx_h[m0:m0 + 128, k0:k0 + 128], oq)
        assert np.array_equal(qxc_h[k0:k0 + 128, m0:m0 + 128], oqc)
        assert np.array_equal(sx_h[k0 // 128, m0:m0 + 128].view(np.uint32), os_.view(np.uint32)[0])
        assert np.array_equal(sxc_h[m0 // 128, k0:k0 + 128].view(np.uint32), osc.view(np.uint32)[0])
    g = int(rng.integers(0, G))
    oq, os_, oqT = orc.quant_weight_128x128(bits(W[g]), mode)
    assert np.array_equal(qw_h[g], oq) and np.array_equal(qwT_h[g], oqT)
    assert np.array_equal(sw_h[g].view(np.uint32), os_.view(np.uint32))

    # fprop / dgrad: a tile per expert, a padding tile per padded expert,
    # random tiles over the routed rows
    for kind, D, (A, sA, B, sB), width in [(0, Y, (qx_h, sx_h, qw_h, sw_h), N),
                                           (1, dX, (qd_h, sd_h, qwT_h, sw_h), K)]:
        Dh = bits(D)
        rows = []
        for g in range(G):
            nblk = (offs[g + 1] - offs[g]) // 128
            if nblk == 0:
                continue
            rows.append(int(offs[g]) + 128 * int(rng.integers(0, nblk)))
            if counts[g] % 128:
                rows.append(int(offs[g + 1]) - 128)      # the block holding the padding rows
        rows += [128 * int(rng.integers(0, int(offs[-1]) // 128)) for _ in range(16)]
        for rb in dict.fromkeys(rows):
            cb = 128 * int(rng.integers(0, width // 128))
            y, ya = orc.grouped_gemm_ref_tile(kind, offs, A, sA, B, sB, 0, rb, rb + 128, cb, cb + 128)
            bad, worst = orc.check_tol(np.ascontiguousarray(Dh[rb:rb + 128, cb:cb + 128]), y, ya)
            assert bad == 0, (kind, rb, cb, worst)
        pad_rows = np.nonzero((r.row_token < 0).numpy())[0]
        if pad_rows.size:
            assert torch.all(D[torch.from_numpy(pad_rows).to(DEV)] == 0)

    # wgrad: one 128x128 tile of every expert's dW_g (contraction over the
    # expert's own tokens only), empty experts exact zeros
    dWh = bits(dW)
    for g in range(G):
        nb, kb = 128 * int(rng.integers(0, N // 128)), 128 * int(rng.integers(0, K // 128))
        y, ya = orc.grouped_gemm_ref_tile(2, offs, qdc_h, sdc_h, qxc_h, sxc_h, g, nb, nb + 128, kb, kb + 128)
        bad, worst = orc.check_tol(np.ascontiguousarray(dWh[g, nb:nb + 128, kb:kb + 128]), y, ya)
        assert bad == 0, (g, nb, kb, worst)
        if counts[g] == 0:
            assert torch.all(dW[g] == 0)


@pytest.mark.parametrize("mode", [0, 1])
def test_grouped_max_experts(fb, orc, mode):
    """FP8BW_MAX_EXPERTS (512) experts, most of them empty or a single
    128-row block (the per-expert pair-tile prefix spans 16 rounds of the
    device scan; odd block counts leave the second CTA of a pair idle)."""
    rng = np.random.default_rng(17 + mode)
    G = 512
    lens = [int(x) for x in rng.choice([0, 0, 1, 100, 130, 300], G)]
    K, N = 128, 256
    c = moe_case(orc, 23 + mode, lens, K, N, mode)
    off, Mtot = c["off"], c["Mtot"]
    for kind, Nout in [(0, N), (1, K)]:
        D, ops = run_grouped(fb, kind, c, mode, (Mtot, Nout))
        y, ya = orc.grouped_gemm_ref_tile(kind, off, *ops, 0, 0, int(off[-1]), 0, Nout)
        bad, worst = orc.check_tol(bits(D)[:int(off[-1])], y, ya)
        assert bad == 0, (kind, worst)
        assert torch.isnan(D[int(off[-1]):].float()).all()
    D, ops = run_grouped(fb, 2, c, mode, (G, N, K))
    Dh = bits(D)
    for e in rng.choice(G, 24, replace=False):
        y, ya = orc.grouped_gemm_ref_tile(2, off, *ops, int(e), 0, N, 0, K)
        bad, worst = orc.check_tol(Dh[e], y, ya)
        assert bad == 0, (int(e), worst)
        if lens[e] == 0:
            assert torch.all(D[e] == 0)


def test_degenerate_sizes(fb, orc):
    """K = 0 gives exact zeros (bf16 and fp32 stores) and leaves an fp32
    accumulator unchanged; M = 0 or N = 0 is a no-op."""
    p = torch.zeros(128 * 128, dtype=torch.uint8, device=DEV)
    s = torch.ones(128 * 128, dtype=torch.float32, device=DEV)
    r = fb.raw
    D = torch.full((128, 256), 5.0, dtype=torch.bfloat16, device=DEV)
    assert r.fp8bw_gemm(0, 128, 256, 0, p.data_ptr(), s.data_ptr(), p.data_ptr(), s.data_ptr(),
                        D.data_ptr(), 256, 0, None) == 0
    torch.cuda.synchronize()
    assert torch.all(D == 0)
    F = torch.full((128, 256), 5.0, dtype=torch.float32, device=DEV)
    assert r.fp8bw_gemm_f32(2, 128, 256, 0, p.data_ptr(), s.data_ptr(), p.data_ptr(), s.data_ptr(),
                            F.data_ptr(), 256, 1, 0, None) == 0
    torch.cuda.synchronize()
    assert torch.all(F == 5.0)
    assert r.fp8bw_gemm_f32(2, 128, 256, 0, p.data_ptr(), s.data_ptr(), p.data_ptr(), s.data_ptr(),
                            F.data_ptr(), 256, 0, 0, None) == 0
    torch.cuda.synchronize()
    assert torch.all(F == 0)
    D.fill_(5.0)
    assert r.fp8bw_gemm(0, 0, 256, 128, p.data_ptr(), s.data_ptr(), p.data_ptr(), s.data_ptr(),
                        D.data_ptr(), 256, 0, None) == 0
    assert r.fp8bw_quant_act_1x128(D.data_ptr(), 0, 128, 128, 0, p.data_ptr(), s.data_ptr(),
                                   None, None, None) == 0
    torch.cuda.synchronize()
    assert torch.all(D == 5.0)
    assert fb.fp8bw_last_device_error() == 0


@pytest.mark.parametrize("mode", [0, 1])
def test_grouped_wgrad_f32_accumulate(fb, orc, mode):
    """fp8bw_grouped_wgrad_f32: each expert's weight gradient stored in fp32,
    then added twice onto a prior fp32 main gradient [G][N][K] (empty experts
    add zeros)."""
    lens = [300, 0, 128, 1, 517, 0, 256, 77]
    K, N = 256, 384
    c = moe_case(orc, 31 + mode, lens, K, N, mode)
    off, G = c["off"], c["G"]
    A, sA, B, sB = c["qdc"], c["sdc"], c["qxc"], c["sxc"]
    offd = dev(off)
    Ad, sAd, Bd, sBd = dev(A), dev(sA), dev(B), dev(sB)
    D = torch.full((G, N, K), float("nan"), dtype=torch.float32, device=DEV)
    fb.fp8bw_grouped_wgrad_f32(offd, Ad, sAd, Bd, sBd, D, accumulate=False, mode=mode)
    torch.cuda.synchronize()
    assert fb.fp8bw_last_device_error() == 0
    rng = np.random.default_rng(8)
    D0 = (rng.standard_normal((G, N, K)) * 1e-3).astype(np.float32)
    Dacc = dev(D0)
    for _ in range(2):
        fb.fp8bw_grouped_wgrad_f32(offd, Ad, sAd, Bd, sBd, Dacc, accumulate=True, mode=mode)
    torch.cuda.synchronize()
    assert fb.fp8bw_last_device_error() == 0
    Dh, Dacch = D.cpu().numpy(), Dacc.cpu().numpy()
    for e in range(G):
        y, ya = orc.grouped_gemm_ref_tile(2, off, A, sA, B, sB, e, 0, N, 0, K)
        bad, worst = orc.check_tol_f32(Dh[e], y, ya)
        assert bad == 0, (e, worst)
        bad, worst = orc.check_tol_f32(Dacch[e], D0[e].astype(np.float64) + 2 * y, 2 * ya)
        assert bad == 0, (e, worst)
        if lens[e] == 0:
            assert np.all(Dh[e] == 0) and np.array_equal(Dacch[e], D0[e])

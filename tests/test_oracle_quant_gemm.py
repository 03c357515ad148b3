"""Pins for the oracle's quantizers and GEMM references (CPU only).

Sources (page titles, sections):
  * "NVIDIA NeMo RL erreicht 48% ...", "Der technische Durchbruch": E4M3 with
    one scale per 128x128 weight block and per 1x128 activation block; the
    linear layers run FP8 math.  "Leistungsgewinne in der Praxis": scales are
    recalibrated after every step; the recipe also covers the Qwen3-30B MoE.
Checks are hand-worked blocks, invariants, and brute force in numpy (an
independent decode through ml_dtypes / torch, scale expansion, fp64 matmul).
"""
import numpy as np
import pytest
import torch

import workloads


def bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def to_bits(a: np.ndarray) -> np.ndarray:
    return bits(torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16))


def dec(q: np.ndarray) -> np.ndarray:
    """Independent E4M3 decode through torch's float8 type."""
    return torch.from_numpy(np.ascontiguousarray(q)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


# --------------------------------------------------------- hand-worked ----
def test_pow2_block_amax_128(orc):
    # amax 128: 128 <= 448*2^-1 = 224 but > 448*2^-2 = 112, so s = 0.5.
    x = np.zeros((1, 128), np.float32)
    x[0, 0] = 128.0
    x[0, 1] = 3.0      # 3 / 0.5 = 6   -> 0x4C
    x[0, 2] = 100.0    # 100/0.5 = 200 -> tie 192|208 -> 0x74
    x[0, 3] = -1.0     # -2 -> 0xC0
    q, s, _, _ = orc.quant_act_1x128(to_bits(x), orc.MODE_POW2, colwise=False)
    assert s[0, 0] == 0.5
    assert q[0, 0] == 0x78  # 256 = 1.0*2^8: field 15 (0x78), mantissa 0
    assert q[0, 1] == 0x4C and q[0, 2] == 0x74 and q[0, 3] == 0xC0
    assert np.all(q[0, 4:] == 0)


@pytest.mark.parametrize("amax,s_exp", [(448.0, 1.0), (224.0, 0.5), (7.0, 2.0 ** -6)])
def test_fp32_exact_scales(orc, amax, s_exp):
    rng = np.random.default_rng(11)
    x = rng.uniform(-1, 1, (1, 128)).astype(np.float32) * amax
    x[0, 5] = amax
    xb = to_bits(x)
    q, s, _, _ = orc.quant_act_1x128(xb, orc.MODE_FP32, colwise=False)
    assert s[0, 0] == s_exp
    # s is a power of two, so q = E4M3(x / s) with an exact division
    xf = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).double().numpy()
    want = torch.from_numpy(xf / s_exp).to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(q, want)
    assert q[0, 5] == 0x7E


def test_single_one_block(orc):
    x = np.zeros((1, 128), np.float32)
    x[0, 17] = 1.0
    q, s, _, _ = orc.quant_act_1x128(to_bits(x), orc.MODE_FP32, colwise=False)
    assert s[0, 0] == np.float32(1.0) / np.float32(448.0)
    assert q[0, 17] == 0x7E and np.count_nonzero(q) == 1


def test_all_zero_block(orc):
    x = np.zeros((128, 256), np.float32)
    x[:, 128:] = 1.0
    for mode in (0, 1):
        q, s, qc, sc = orc.quant_act_1x128(to_bits(x), mode)
        assert s[0].view(np.uint32).tolist() == [0x3F800000] * 128
        assert np.all(q[:, :128] == 0) and not np.isnan(s).any()
        assert np.all(sc[0, :128] == 1.0) and np.all(qc[:128] == 0)
    # a block of -0 inputs: scale 1, every code 0x80 (the sign of zero is kept)
    z = np.full((128, 256), -0.0, np.float32)
    z[:, 128:] = 0.0
    q, s, qc, sc = orc.quant_act_1x128(to_bits(z), 0)
    assert np.all(q[:, :128] == 0x80) and np.all(q[:, 128:] == 0x00)
    assert np.all(s == 1.0) and np.all(sc == 1.0)
    assert np.all(qc[:128] == 0x80) and np.all(qc[128:] == 0x00)


# ----------------------------------------------------------- invariants ---
def test_amax_maps_to_448(orc):
    X, _, _ = workloads.tiny(0)
    xb = bits(X)
    xf = X.float().numpy()
    for mode in (0, 1):
        q, s, _, _ = orc.quant_act_1x128(xb, mode, colwise=False)
        M, K = xf.shape
        for m in range(0, M, 37):
            for kb in range(K // 128):
                blk = xf[m, kb * 128:(kb + 1) * 128]
                j = int(np.argmax(np.abs(blk)))
                if mode == 0:
                    assert q[m, kb * 128 + j] & 0x7F == 0x7E
                else:
                    # amax / s lies in (224, 448]; E4M3 rounding keeps it in [224, 448]
                    assert 224.0 < abs(blk[j]) / s[kb, m] <= 448.0
                    v = abs(dec(q[m, kb * 128 + j:kb * 128 + j + 1])[0])
                    assert 224.0 <= v <= 448.0


@pytest.mark.parametrize("mode", [0, 1])
def test_power_of_two_scaling_invariance(orc, mode):
    X, _, _ = workloads.tiny(0)
    xb = bits(X)
    q0, s0, qc0, sc0 = orc.quant_act_1x128(xb, mode)
    for j in (-3, 5):
        xj = bits((X.double() * 2.0 ** j).to(torch.bfloat16))
        q1, s1, qc1, sc1 = orc.quant_act_1x128(xj, mode)
        np.testing.assert_array_equal(q0, q1)
        np.testing.assert_array_equal(qc0, qc1)
        np.testing.assert_array_equal(s1, (s0.astype(np.float64) * 2.0 ** j).astype(np.float32))
        np.testing.assert_array_equal(sc1, (sc0.astype(np.float64) * 2.0 ** j).astype(np.float32))


def test_block_independence(orc):
    X, W, _ = workloads.tiny(0)
    xb = bits(X).copy()
    q0, s0, qc0, sc0 = orc.quant_act_1x128(xb, 0)
    xb2 = xb.copy()
    xb2[3, 130] = to_bits(np.array([[1000.0]]))[0, 0]
    q1, s1, qc1, sc1 = orc.quant_act_1x128(xb2, 0)
    # row block (3, kb=1) and column block (mb=0, k=130) change, nothing else
    dq = np.argwhere(q0 != q1)
    assert set(map(tuple, dq[:, :1].tolist())) == {(3,)}
    assert np.all((dq[:, 1] >= 128) & (dq[:, 1] < 256))
    ds = np.argwhere(s0 != s1)
    assert ds.tolist() == [[1, 3]]
    dqc = np.argwhere(qc0 != qc1)
    assert np.all(dqc[:, 0] == 130) and np.all(dqc[:, 1] < 128)
    assert np.argwhere(sc0 != sc1).tolist() == [[0, 130]]


def test_colwise_equals_rowwise_of_transpose(orc):
    X, _, dY = workloads.tiny(0)
    for T in (X, dY):
        for mode in (0, 1):
            _, _, qc, sc = orc.quant_act_1x128(bits(T), mode)
            qt, st, _, _ = orc.quant_act_1x128(bits(T.t().contiguous()), mode, colwise=False)
            np.testing.assert_array_equal(qc, qt)
            np.testing.assert_array_equal(sc, st)


@pytest.mark.parametrize("mode", [0, 1])
def test_weight_quant_invariants(orc, mode):
    _, W, _ = workloads.tiny(0)
    wb = bits(W)
    q, s, qT = orc.quant_weight_128x128(wb, mode)
    np.testing.assert_array_equal(qT, q.T)
    # the 128x128 scale is the largest of its rows' 1x128 scales (the scale
    # rule is monotone in amax), and codes follow E4M3(x / s)
    _, sr, _, _ = orc.quant_act_1x128(wb, mode, colwise=False)
    N, K = W.shape
    for nb in range(N // 128):
        for kb in range(K // 128):
            assert s[nb, kb] == sr[kb, nb * 128:(nb + 1) * 128].max()
    wf = W.float().numpy().astype(np.float32)
    sfull = np.repeat(np.repeat(s, 128, 0), 128, 1)
    t = (wf / sfull).astype(np.float32)
    np.testing.assert_array_equal(q, orc.e4m3_encode_array(t))


# ------------------------------------------------------------------ GEMM --
def _rand_operands(rng, M, N, K, kind, small_int=False):
    if small_int:
        # codes of small integers: 0x38 = 1, 0x40 = 2, 0x44 = 3, 0xB8 = -1
        pool = np.array([0x00, 0x38, 0x40, 0x44, 0xB8, 0xC0], np.uint8)
        A = rng.choice(pool, (M, K))
        B = rng.choice(pool, (N, K))
    else:
        A = rng.integers(0, 256, (M, K), dtype=np.uint8)
        B = rng.integers(0, 256, (N, K), dtype=np.uint8)
        A[(A & 0x7F) == 0x7F] = 0x00
        B[(B & 0x7F) == 0x7F] = 0x00
    nK = K // 128
    if small_int:
        sA = np.ones((nK, M), np.float32)
        sB = {0: np.ones((N // 128, nK)), 1: np.ones((nK, N // 128)), 2: np.ones((nK, N))}[kind].astype(np.float32)
    else:
        sA = (2.0 ** rng.uniform(-8, 2, (nK, M))).astype(np.float32)
        shp = {0: (N // 128, nK), 1: (nK, N // 128), 2: (nK, N)}[kind]
        sB = (2.0 ** rng.uniform(-8, 2, shp)).astype(np.float32)
    return A, sA, B, sB


def _brute(kind, A, sA, B, sB):
    M, K = A.shape
    N = B.shape[0]
    sa_full = np.repeat(sA.astype(np.float64), 128, axis=0).T          # [M, K]
    if kind == 0:
        sb_full = np.repeat(np.repeat(sB.astype(np.float64), 128, 0), 128, 1)   # [N, K]
    elif kind == 1:
        sb_full = np.repeat(np.repeat(sB.astype(np.float64).T, 128, 0), 128, 1)
    else:
        sb_full = np.repeat(sB.astype(np.float64), 128, axis=0).T
    a = dec(A) * sa_full
    b = dec(B) * sb_full
    return a @ b.T, np.abs(a) @ np.abs(b).T


@pytest.mark.parametrize("kind", [0, 1, 2])
def test_gemm_ref_brute_force(orc, kind):
    rng = np.random.default_rng(100 + kind)
    M, N, K = 128, 256, 384
    A, sA, B, sB = _rand_operands(rng, M, N, K, kind)
    y, ya = orc.gemm_ref_tile(kind, A, sA, B, sB, 0, M, 0, N)
    yb, yab = _brute(kind, A, sA, B, sB)
    np.testing.assert_allclose(y, yb, rtol=1e-12, atol=1e-12 * yab.max())
    np.testing.assert_allclose(ya, yab, rtol=1e-12)
    pm = rng.integers(0, M, 50)
    pn = rng.integers(0, N, 50)
    yp, _ = orc.gemm_ref_points(kind, A, sA, B, sB, pm, pn)
    np.testing.assert_array_equal(yp, y[pm, pn])


@pytest.mark.parametrize("kind", [0, 1, 2])
def test_gemm_small_integers_exact(orc, kind):
    rng = np.random.default_rng(7 + kind)
    A, sA, B, sB = _rand_operands(rng, 128, 128, 256, kind, small_int=True)
    y, _ = orc.gemm_ref_tile(kind, A, sA, B, sB, 0, 128, 0, 128)
    ai = np.round(dec(A)).astype(np.int64)
    bi = np.round(dec(B)).astype(np.int64)
    np.testing.assert_array_equal(y, (ai @ bi.T).astype(np.float64))


def test_gemm_identity(orc):
    rng = np.random.default_rng(3)
    M = K = N = 256
    A, sA, _, _ = _rand_operands(rng, M, N, K, 0)
    B = np.zeros((N, K), np.uint8)
    np.fill_diagonal(B, 0x38)
    sB = np.ones((N // 128, K // 128), np.float32)
    y, _ = orc.gemm_ref_tile(0, A, sA, B, sB, 0, M, 0, N)
    sa_full = np.repeat(sA.astype(np.float64), 128, axis=0).T
    np.testing.assert_array_equal(y, dec(A) * sa_full)


def test_gemm_zero_rows(orc):
    rng = np.random.default_rng(4)
    A, sA, B, sB = _rand_operands(rng, 256, 128, 256, 0)
    A[128:] = 0
    y, ya = orc.gemm_ref_tile(0, A, sA, B, sB, 128, 256, 0, 128)
    assert np.all(y == 0) and np.all(ya == 0)


def test_grouped_reference(orc):
    rng = np.random.default_rng(9)
    G, N, K = 4, 256, 256
    off = np.array([0, 256, 256, 384, 640], np.int32)     # expert 1 is empty
    Mtot = 768                                             # tail past off[G]
    A = rng.integers(0, 0x7E, (Mtot, K), dtype=np.uint8)
    sA = (2.0 ** rng.uniform(-4, 1, (K // 128, Mtot))).astype(np.float32)
    B = rng.integers(0, 0x7E, (G, N, K), dtype=np.uint8)
    sB = (2.0 ** rng.uniform(-4, 1, (G, N // 128, K // 128))).astype(np.float32)
    y, _ = orc.grouped_gemm_ref_tile(0, off, A, sA, B, sB, 0, 0, Mtot, 0, N)
    for g in range(G):
        r0, r1 = off[g], off[g + 1]
        if r1 == r0:
            continue
        yd, _ = _brute(0, A[r0:r1], np.ascontiguousarray(sA[:, r0:r1]), B[g], sB[g])
        np.testing.assert_allclose(y[r0:r1], yd, rtol=1e-12, atol=1e-9)
    assert np.all(y[off[G]:] == 0)
    # wgrad: dW_g contracts only expert g's tokens
    At = rng.integers(0, 0x7E, (N, Mtot), dtype=np.uint8)     # dY^T
    sAt = (2.0 ** rng.uniform(-4, 1, (Mtot // 128, N))).astype(np.float32)
    Bt = rng.integers(0, 0x7E, (K, Mtot), dtype=np.uint8)     # X^T
    sBt = (2.0 ** rng.uniform(-4, 1, (Mtot // 128, K))).astype(np.float32)
    for g in range(G):
        r0, r1 = off[g], off[g + 1]
        yw, _ = orc.grouped_gemm_ref_tile(2, off, At, sAt, Bt, sBt, g, 0, N, 0, K)
        if r1 == r0:
            assert np.all(yw == 0)
            continue
        yd, _ = _brute(2, np.ascontiguousarray(At[:, r0:r1]), np.ascontiguousarray(sAt[r0 // 128:r1 // 128]),
                       np.ascontiguousarray(Bt[:, r0:r1]), np.ascontiguousarray(sBt[r0 // 128:r1 // 128]))
        np.testing.assert_allclose(yw, yd, rtol=1e-12, atol=1e-9)


def test_bf16_reference(orc):
    rng = np.random.default_rng(5)
    a = rng.standard_normal((128, 256)).astype(np.float32)
    b = rng.standard_normal((64, 256)).astype(np.float32)
    ab, bb = to_bits(a), to_bits(b)
    y, _ = orc.gemm_bf16_ref_tile(ab, bb, 0, 128, 0, 64)
    af = torch.from_numpy(ab.view(np.int16)).view(torch.bfloat16).double().numpy()
    bf = torch.from_numpy(bb.view(np.int16)).view(torch.bfloat16).double().numpy()
    np.testing.assert_allclose(y, af @ bf.T, rtol=1e-12, atol=1e-12)


def test_check_tol_and_mimic(orc):
    X, W, _ = workloads.tiny(0)
    qx, sx, _, _ = orc.quant_act_1x128(bits(X), 0, colwise=False)
    qw, sw, _ = orc.quant_weight_128x128(bits(W), 0)
    y, ya = orc.gemm_ref_tile(0, qx, sx, qw, sw, 0, 128, 0, 128)
    yb = to_bits(y)
    assert orc.check_tol(yb, y, ya)[0] == 0
    mim = orc.gemm_mimic_tile(0, qx, sx, qw, sw, 0, 128, 0, 128)
    bad, worst = orc.check_tol(mim, y, ya)
    assert bad == 0 and worst < 0.2
    # a planted error well beyond the allowance is caught
    yp = y.copy()
    yp[5, 7] += 0.02 * ya[5, 7] + 1.0
    assert orc.check_tol(to_bits(yp), y, ya)[0] >= 1
    # a dropped K-chunk is caught (allowance is 1% of sum |a b|)
    qx2 = qx.copy()
    qx2[:, 128:256] = 0
    y2, _ = orc.gemm_ref_tile(0, qx2, sx, qw, sw, 0, 128, 0, 128)
    assert orc.check_tol(to_bits(y2), y, ya)[0] > 100


def test_check_tol_f32(orc):
    """The fp32-output gate: exact values and errors up to the allowance pass,
    anything beyond it (or NaN) fails."""
    yref = np.array([1.0, -3.0, 0.0, 1e-3])
    yabs = np.array([2.0, 3.0, 0.0, 1e-3])
    lim = orc.REL_TOL * yabs + orc.F32_ABS_REL * np.abs(yref)
    assert orc.check_tol_f32(yref, yref, yabs)[0] == 0
    assert orc.check_tol_f32(yref + 0.99 * lim, yref, yabs)[0] == 0
    bad, worst = orc.check_tol_f32(yref + 1.01 * lim * np.array([1, 0, 0, 1]), yref, yabs)
    assert bad == 2 and worst > 1.0
    assert orc.check_tol_f32(np.array([np.nan, -3.0, 0.0, 1e-3]), yref, yabs)[0] == 1
    assert orc.check_tol_f32(np.array([1.0, -3.0, 1e-30, 1e-3]), yref, yabs)[0] == 1  # zero allowance

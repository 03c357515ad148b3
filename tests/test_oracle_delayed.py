"""Pins of the oracle's per-tensor delayed scaling (CPU only).

"FP8 Trainingsinfrastructuur: Numerieke Precisie van de Volgende
Generatie", sections "Transformer Engine: de softwarebasis" (the recipe: a
history of 16 amax values, the "max" rule, margin 0, E4M3 forward and E5M2
backward) and "Scaling-strategieën en stabiliteit" (one scale per tensor;
delayed scaling takes it from statistics of earlier iterations, not of the
tensor being quantized)."""
import numpy as np
import pytest
import torch

import oracle as orc


def bits(x):
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


def spike(v, shape=(128, 256), at=(3, 77)):
    x = torch.zeros(shape, dtype=torch.bfloat16)
    x[at] = v
    return bits(x)


def test_history_sequence_hand_worked():
    # H = 4; each step's tensor holds one value, so its amax is that value.
    # Before step t the history holds the amax of steps t-1 .. t-4.
    H = 4
    amaxes = [3.0, 0.5, 7.0, 1.0, 2.0, 0.25, 0.125, 0.5]
    f = np.float32
    # the largest earlier amax at each step, worked by hand: none, 3, 3, 7,
    # 7, 7, 7 (steps 2..5), then 2 once 7 has left the window
    want = [f(1.0), f(3) / f(448), f(3) / f(448), f(7) / f(448), f(7) / f(448),
            f(7) / f(448), f(7) / f(448), f(2) / f(448)]
    hist = np.zeros(H, np.float32)
    for t, a in enumerate(amaxes):
        q, qT, s, am, hist = orc.quant_tensor_delayed(spike(a), hist, orc.MODE_FP32)
        assert s == want[t], (t, s, want[t])
        assert am == f(a)
    assert list(hist) == [0.5, 0.125, 0.25, 2.0]          # newest first


def test_history_of_length_one_is_the_previous_step():
    hist = np.zeros(1, np.float32)
    seen = []
    for a in [5.0, 0.75, 96.0]:
        _, _, s, _, hist = orc.quant_tensor_delayed(spike(a), hist, orc.MODE_POW2)
        seen.append(s)
    # POW2: smallest 2^e with amax <= 448 * 2^e: none -> 1; 5 -> 2^-6
    # (448/64 = 7 >= 5, 448/128 = 3.5 < 5); 0.75 -> 2^-9 (0.875 >= 0.75)
    assert seen == [1.0, 2.0 ** -6, 2.0 ** -9]


@pytest.mark.parametrize("fmt,tdt,qmax", [(orc.FMT_E4M3, torch.float8_e4m3fn, 448.0),
                                          (orc.FMT_E5M2, torch.float8_e5m2, 57344.0)])
@pytest.mark.parametrize("mode", [orc.MODE_FP32, orc.MODE_POW2])
def test_codes_match_torch_cast(fmt, tdt, qmax, mode):
    g = torch.Generator().manual_seed(5)
    x = (torch.randn((256, 384), generator=g) * 3.0).to(torch.bfloat16)
    x[7, :] *= 40.0                                    # an outlier row
    a = float(x.float().abs().max())
    # history above the current amax: nothing saturates
    hist = np.array([a * 0.5, a * 1.5, a * 0.25], np.float32)
    q, qT, s, am, _ = orc.quant_tensor_delayed(bits(x), hist, mode, fmt)
    assert am == np.float32(a)
    t = x.float() / torch.tensor(s, dtype=torch.float32)
    assert float(t.abs().max()) <= qmax
    ref = t.to(tdt).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)
    assert np.array_equal(qT, q.T)


@pytest.mark.parametrize("fmt,tdt,qmax", [(orc.FMT_E4M3, torch.float8_e4m3fn, 448.0),
                                          (orc.FMT_E5M2, torch.float8_e5m2, 57344.0)])
def test_tensor_outgrowing_its_history_saturates(fmt, tdt, qmax):
    g = torch.Generator().manual_seed(9)
    x = (torch.randn((128, 256), generator=g) * 2.0).to(torch.bfloat16)
    a = float(x.float().abs().max())
    hist = np.array([a / 8.0], np.float32)            # delayed amax 8x too small
    q, _, s, _, _ = orc.quant_tensor_delayed(bits(x), hist, orc.MODE_FP32, fmt)
    t = x.float() / torch.tensor(s, dtype=torch.float32)
    over = t.abs() >= qmax
    assert int(over.sum()) > 100
    # saturation then rounding: 448 and 57344 are grid points, so clamping
    # before the cast is the saturating round-to-nearest-even
    ref = t.clamp(-qmax, qmax).to(tdt).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)
    top = 0x7E if fmt == orc.FMT_E4M3 else 0x7B
    assert np.all((q[over.numpy()] & 0x7F) == top)


@pytest.mark.parametrize("mode", [orc.MODE_FP32, orc.MODE_POW2])
def test_own_amax_in_history_is_the_single_block_rule(mode):
    # With the tensor's own amax as the only history entry, one 128x128 tensor
    # is quantized exactly as the single block of the 128x128 weight rule.
    g = torch.Generator().manual_seed(2)
    w = (torch.randn((128, 128), generator=g) * 0.02).to(torch.bfloat16)
    wb = bits(w)
    hist = np.array([float(w.float().abs().max())], np.float32)
    q, qT, s, _, _ = orc.quant_tensor_delayed(wb, hist, mode)
    qw, sw, qwT = orc.quant_weight_128x128(wb, mode)
    assert s == sw[0, 0]
    assert np.array_equal(q, qw) and np.array_equal(qT, qwT)


def test_nan_wins_no_maximum():
    x = torch.zeros((128, 128), dtype=torch.bfloat16)
    x[0, 0], x[1, 1] = float("nan"), -6.0
    hist = np.array([np.nan, 3.0], np.float32)
    q, _, s, am, h = orc.quant_tensor_delayed(bits(x), hist, orc.MODE_FP32)
    assert am == 6.0 and s == np.float32(3) / np.float32(448)
    assert q[0, 0] == 0x7F
    assert h[0] == 6.0 and np.isnan(h[1])


def test_per_tensor_gemm_through_the_block_reference():
    # A per-tensor operand is a blockwise operand whose scale grid is constant;
    # the block reference then computes s_a * s_b * (A_codes . B_codes).
    rng = np.random.default_rng(4)
    M, N, K = 128, 256, 384
    A = rng.integers(0, 0x7E, (M, K), dtype=np.uint8) | (rng.integers(0, 2, (M, K), dtype=np.uint8) << 7)
    B = rng.integers(0, 0x7B, (N, K), dtype=np.uint8) | (rng.integers(0, 2, (N, K), dtype=np.uint8) << 7)
    sa, sb = np.float32(3.0 / 448), np.float32(0.01 / 57344)
    sA = np.full((K // 128, M), sa, np.float32)
    sB = np.full((N // 128, K // 128), sb, np.float32)
    y, yabs = orc.gemm_ref_tile(orc.FPROP, A, sA, B, sB, 0, M, 0, N, fa=orc.FMT_E4M3, fb=orc.FMT_E5M2)
    da = torch.from_numpy(A).view(torch.float8_e4m3fn).double().numpy()
    db = torch.from_numpy(B).view(torch.float8_e5m2).double().numpy()
    want = float(sa) * float(sb) * (da @ db.T)
    assert np.all(np.abs(y - want) <= 1e-12 * yabs)

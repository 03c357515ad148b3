"""Pins of the quantization-error study (oracle/quant_error.py), CPU only.

"FP8 Trainingsinfrastructuur ...", section "Scaling-strategieën en
stabiliteit": block scaling lowers the quantization error by 30-50 % against
per-tensor scaling.  The study's schemes are pinned to special cases where
they must agree with the method's quantizers, then the claim is checked on
activations with the workloads' outlier channels."""
import numpy as np
import torch

import workloads
from oracle import MODE_FP32, MODE_POW2
from oracle import quant_error as qe


def bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def test_tensor_scale_on_one_block_equals_blockwise():
    # a [1, 128] tensor is a single 1x128 block: per-tensor == blockwise (fp32 scale)
    g = torch.Generator().manual_seed(1)
    x = (torch.randn((1, 128), generator=g) * 7).to(torch.bfloat16)
    b = bits(torch.cat([x] * 128))  # 128 copies of the row: whole 128-row tiles
    xf = qe.bf16_bits_to_f32(b)
    assert np.array_equal(qe.dq_tensor(xf[:1]), qe.dq_blockwise_act(b, MODE_FP32)[:1])


def test_mx32_round_up_on_equal_blocks_equals_pow2_blockwise():
    # four 1x32 blocks with the same amax share one power-of-2 scale with the 1x128 block
    g = torch.Generator().manual_seed(2)
    x = torch.randn((128, 128), generator=g)
    x[:, ::32] = 5.0                      # every 32-block's amax is 5
    x = x.clamp(-4.9, 5.0).to(torch.bfloat16)
    b = bits(x)
    xf = qe.bf16_bits_to_f32(b)
    assert np.array_equal(qe.dq_mx32(xf, round_up=True), qe.dq_blockwise_act(b, MODE_POW2))
    # the floor rule puts 5 = 1.25 * 2^2 at 320 = 1.25 * 2^8: no saturation, same codes here
    assert np.array_equal(qe.dq_mx32(xf), qe.dq_blockwise_act(b, MODE_POW2))


def test_mx32_floor_rule_saturates_above_1p75():
    # amax = 1.875 * 2^0 -> floor exponent 0 - 8 -> 1.875 * 2^8 = 480 saturates to 448
    x = np.zeros((1, 32), np.float32)
    x[0, 0] = 1.875
    assert qe.dq_mx32(x)[0, 0] == 448.0 * 2.0 ** -8
    assert qe.dq_mx32(x, round_up=True)[0, 0] == 1.875


def test_gaussian_weights_scale_invariant():
    # no outliers: E4M3's relative spacing does not depend on the scale, so
    # one scale per tensor and per 128x128 block give the same error (within 2 %)
    W = workloads.normal_bf16((512, 512), 0.02, 3)
    e = qe.tensor_errors(bits(W), weight=True)
    assert abs(e["blockwise"] - e["tensor"]) < 0.02 * e["tensor"]


def test_block_scaling_beats_per_tensor_on_outlier_activations():
    X, W, _ = workloads.llama_layer("o_proj", seed=0, M=256)
    xb, wb = bits(X), bits(W)
    e = qe.tensor_errors(xb, weight=False)
    assert e["blockwise"] < 0.7 * e["tensor"]          # at least 30 % lower
    y = qe.gemm_errors(xb, wb, 128, 256)
    assert y["blockwise"] < y["tensor"]


def test_delayed_scaling_on_a_constant_tensor_is_current_scaling():
    # the same tensor every step: from step 1 on the history's maximum is the
    # tensor's own amax, so delayed and current per-tensor scaling coincide
    rows = qe.delayed_study(tokens=128, history=4, schedule=[1.0, 1.0, 1.0])
    for _, _, e in rows[1:]:
        assert e["delayed"] == e["tensor"] and e["saturated"] < 1e-4


def test_delayed_scaling_first_step_uses_unit_scale():
    # zero history: s = 1, so the codes are the plain E4M3 encodings of x
    X, _, _ = workloads.llama_layer("o_proj", seed=0, M=128)
    xb = bits(X)
    dq, h, _ = qe.dq_delayed(xb, np.zeros(4, np.float32))
    x = qe.bf16_bits_to_f32(xb)
    plain = qe.decode_table()[qe.e4m3_encode_array(np.ascontiguousarray(x))]
    assert np.array_equal(dq, plain)
    assert h[0] == np.abs(x).max() and np.all(h[1:] == 0)


def test_delayed_scaling_spike_saturates_then_recovers():
    # a 4x spike after steady steps: the delayed scale lags, the outlier
    # channels saturate and the error jumps; on the next step (back to the
    # old magnitude, history inflated by the spike) it is back near current
    # scaling, since E4M3's relative spacing does not depend on the scale
    rows = qe.delayed_study(tokens=128, history=4, schedule=[1.0, 1.0, 4.0, 1.0, 1.0])
    spike, after = rows[2][2], rows[3][2]
    assert spike["saturated"] > 0 and spike["delayed"] > 5 * spike["tensor"]
    assert after["delayed"] < 1.1 * after["tensor"]


def test_e5m2_per_tensor_on_one_block_equals_blockwise():
    g = torch.Generator().manual_seed(6)
    x = (torch.randn((1, 128), generator=g) * 1e-3).to(torch.bfloat16)
    b = bits(torch.cat([x] * 128))
    xf = qe.bf16_bits_to_f32(b)
    assert np.array_equal(qe.dq_tensor_fmt(xf[:1], qe.FMT_E5M2),
                          qe.dq_blockwise_act_fmt(b, qe.FMT_E5M2)[:1])


def test_e5m2_gradient_error_is_twice_e4m3():
    # one mantissa bit fewer doubles the grid spacing, hence the relative
    # rounding error of values in the normal range
    _, _, dY = workloads.llama_layer("o_proj", seed=0, M=128)
    db = bits(dY)
    d = qe.bf16_bits_to_f32(db)
    e4 = qe.rel_err(d, qe.dq_blockwise_act_fmt(db, qe.FMT_E4M3))
    e5 = qe.rel_err(d, qe.dq_blockwise_act_fmt(db, qe.FMT_E5M2))
    assert 1.8 < e5 / e4 < 2.2

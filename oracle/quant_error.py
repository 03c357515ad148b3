"""Quantization-error study — TEST INFRASTRUCTURE (CPU only, oracle codec).

"FP8 Trainingsinfrastructuur: Numerieke Precisie van de Volgende Generatie",
section "Scaling-strategieën en stabiliteit": block scaling lowers the
quantization error by 30-50 % against one scale per tensor.  This module
measures that on the seeded synthetic workloads, for several ways of
choosing E4M3 scales.  Every scheme divides in fp32 (IEEE, round to nearest) and
encodes with the oracle's E4M3 codec (round to nearest even, saturating):

  blockwise  the method itself: 1x128 blocks along K for activations and
             gradients, 128x128 blocks for weights, s = fp32(amax / 448)
             (or the power-of-2 scale), via the oracle's quantizers;
  tensor     one scale for the whole tensor, s = fp32(amax / 448);
  mx32       1x32 blocks along K with a power-of-two scale
             2^(floor(log2 amax) - 8), the shared-exponent rule of the OCP
             MX formats (8 is the exponent of E4M3's largest normal, 448 =
             1.75 * 2^8); values above 448 after scaling saturate;
  mx32_up    the same 1x32 blocks with the method's power-of-2 rule (the
             smallest 2^e with amax <= 448 * 2^e: nothing saturates).

Reported: the relative Frobenius error of each dequantized tensor against
its bf16 values, and of the product Y = X * W^T on a block of outputs
against the fp64 product of the bf16 operands.

Run ``python -m oracle.quant_error`` for the table of the Llama-3.1-8B-like
layers (config of 8192-token layers, sampled at 1024 tokens) and the packed
Student-t batch.

A second table follows one activation tensor over training steps whose
magnitude drifts, for the delayed per-tensor recipe of the same page
(section "Transformer Engine: de softwarebasis": a history of 16 amax
values, the "max" rule): its scale comes from earlier steps, so a tensor
that grows saturates and, after a spike, the inflated history wastes
dynamic range until the spike leaves the window.
"""
from __future__ import annotations

import numpy as np

from . import (FMT_E4M3, FMT_E5M2, MODE_FP32, MODE_POW2, e4m3_decode, e4m3_encode_array,
               e5m2_decode, e5m2_encode_array, quant_act_1x128, quant_tensor_delayed,
               quant_weight_128x128)

_TABLE = None


def decode_table() -> np.ndarray:
    """fp64 value of each of the 256 E4M3 codes (NaN for 0x7F, 0xFF)."""
    global _TABLE
    if _TABLE is None:
        _TABLE = np.array([e4m3_decode(c) for c in range(256)], np.float64)
    return _TABLE


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def dq_blockwise_act(bits: np.ndarray, mode: int) -> np.ndarray:
    """Dequantized 1x128 row-block quantization of a bf16 [M, K] tensor."""
    q, s, _, _ = quant_act_1x128(bits, mode, colwise=False)
    return decode_table()[q] * np.repeat(s.T.astype(np.float64), 128, axis=1)


def dq_blockwise_weight(bits: np.ndarray, mode: int) -> np.ndarray:
    """Dequantized 128x128 block quantization of a bf16 [N, K] weight."""
    q, s, _ = quant_weight_128x128(bits, mode, transposed=False)
    sf = np.repeat(np.repeat(s.astype(np.float64), 128, axis=0), 128, axis=1)
    return decode_table()[q] * sf


def dq_tensor(x: np.ndarray) -> np.ndarray:
    """One fp32 scale amax/448 for the whole tensor."""
    amax = np.float32(np.max(np.abs(x)))
    s = np.float32(amax / np.float32(448.0)) if amax > 0 else np.float32(1.0)
    codes = e4m3_encode_array(np.ascontiguousarray((x / s).astype(np.float32)))
    return decode_table()[codes] * np.float64(s)


def dq_mx32(x: np.ndarray, round_up: bool = False) -> np.ndarray:
    """1x32 blocks along the last axis, scale 2^(floor(log2 amax) - 8), or
    with `round_up` the smallest 2^e with amax <= 448 * 2^e."""
    R, C = x.shape
    xb = x.reshape(R, C // 32, 32)
    amax = np.max(np.abs(xb), axis=2)
    f, E = np.frexp(amax.astype(np.float64))     # amax = f * 2^E, f in [0.5, 1)
    e = E - 1 - 8                                # amax = (2f) * 2^(E-1), 2f in [1, 2)
    if round_up:
        e = e + (2 * f > 1.75)
    e = np.clip(e, -127, 127)
    X = np.where(amax > 0, np.ldexp(np.float32(1.0), e).astype(np.float32), np.float32(1.0))
    v = (xb / X[:, :, None]).astype(np.float32)    # exact: X is a power of two
    codes = e4m3_encode_array(np.ascontiguousarray(v))
    return (decode_table()[codes] * X[:, :, None].astype(np.float64)).reshape(R, C)


def rel_err(ref: np.ndarray, approx: np.ndarray) -> float:
    ref = ref.astype(np.float64)
    return float(np.linalg.norm(approx - ref) / np.linalg.norm(ref))


def tensor_errors(bits: np.ndarray, weight: bool) -> dict:
    """Relative errors of the four schemes on one bf16 tensor (uint16 bits)."""
    x = bf16_bits_to_f32(bits)
    blk = dq_blockwise_weight if weight else dq_blockwise_act
    return {"blockwise": rel_err(x, blk(bits, MODE_FP32)),
            "blockwise_pow2": rel_err(x, blk(bits, MODE_POW2)),
            "tensor": rel_err(x, dq_tensor(x)),
            "mx32": rel_err(x, dq_mx32(x)),
            "mx32_up": rel_err(x, dq_mx32(x, True))}


def gemm_errors(xbits: np.ndarray, wbits: np.ndarray, rows: int, cols: int) -> dict:
    """Relative error of Y = X W^T on the first rows x cols outputs."""
    x, w = bf16_bits_to_f32(xbits), bf16_bits_to_f32(wbits)
    ref = x[:rows].astype(np.float64) @ w[:cols].astype(np.float64).T
    out = {}
    xb, wb = dq_blockwise_act(xbits[:rows], MODE_FP32), dq_blockwise_weight(wbits[:cols], MODE_FP32)
    out["blockwise"] = rel_err(ref, xb @ wb.T)
    xb, wb = dq_blockwise_act(xbits[:rows], MODE_POW2), dq_blockwise_weight(wbits[:cols], MODE_POW2)
    out["blockwise_pow2"] = rel_err(ref, xb @ wb.T)
    # per-tensor scales come from the whole tensors, then the same block of outputs
    out["tensor"] = rel_err(ref, dq_tensor(x)[:rows] @ dq_tensor(w)[:cols].T)
    out["mx32"] = rel_err(ref, dq_mx32(x[:rows]) @ dq_mx32(w[:cols]).T)
    out["mx32_up"] = rel_err(ref, dq_mx32(x[:rows], True) @ dq_mx32(w[:cols], True).T)
    return out


def study(tokens: int = 1024, seed: int = 0) -> list:
    """Rows of (tensor name, errors) for the Llama-3.1-8B-like layers at
    `tokens` tokens and for the packed Student-t activations."""
    import torch

    import workloads

    def bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    rows = []
    for name, K, N in workloads.LLAMA8B_LAYERS:
        X, W, dY = workloads.llama_layer(name, seed=seed, M=tokens)
        xb, wb, db = bits(X), bits(W), bits(dY)
        rows.append((f"{name} X [{tokens},{K}]", tensor_errors(xb, False)))
        rows.append((f"{name} W [{N},{K}]", tensor_errors(wb, True)))
        rows.append((f"{name} dY [{tokens},{N}]", tensor_errors(db, False)))
        rows.append((f"{name} Y=XW^T [256,512]", gemm_errors(xb, wb, 256, 512)))
    P = workloads.packed_activations(4096, seed, total=tokens)
    rows.append((f"packed Student-t X [{tokens},4096]", tensor_errors(bits(P), False)))
    return rows


_TABLE5 = None


def decode_table_e5m2() -> np.ndarray:
    """fp64 value of each of the 256 E5M2 codes."""
    global _TABLE5
    if _TABLE5 is None:
        _TABLE5 = np.array([e5m2_decode(c) for c in range(256)], np.float64)
    return _TABLE5


def dq_blockwise_act_fmt(bits: np.ndarray, fmt: int) -> np.ndarray:
    """Dequantized 1x128 row blocks (fp32 scale) in E4M3 or E5M2."""
    q, s, _, _ = quant_act_1x128(bits, MODE_FP32, colwise=False, fmt=fmt)
    table = decode_table_e5m2() if fmt == FMT_E5M2 else decode_table()
    return table[q] * np.repeat(s.T.astype(np.float64), 128, axis=1)


def dq_tensor_fmt(x: np.ndarray, fmt: int) -> np.ndarray:
    """One fp32 scale amax/Q for the whole tensor, Q = 448 (E4M3) or 57344
    (E5M2)."""
    if fmt == FMT_E4M3:
        return dq_tensor(x)
    amax = np.float32(np.max(np.abs(x)))
    s = np.float32(amax / np.float32(57344.0)) if amax > 0 else np.float32(1.0)
    codes = e5m2_encode_array(np.ascontiguousarray((x / s).astype(np.float32)))
    return decode_table_e5m2()[codes] * np.float64(s)


def gradient_study(tokens: int = 256, seed: int = 0, cols: int = 512) -> list:
    """Rows of (layer, errors) for the gradient dY [tokens, N] of each
    Llama-like layer in four encodings (E4M3 / E5M2, 1x128 blocks / one
    scale per tensor, fp32 scales), and for the data gradient
    dX[:, :cols] = dY W[:, :cols] with W in 128x128 E4M3 blocks."""
    import torch

    import workloads

    def bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    rows = []
    for name, K, N in workloads.LLAMA8B_LAYERS:
        _, W, dY = workloads.llama_layer(name, seed=seed, M=tokens)
        db = bits(dY)
        d = bf16_bits_to_f32(db)
        w = bf16_bits_to_f32(bits(W))[:, :cols].astype(np.float64)
        wq = dq_blockwise_weight(bits(W[:, :cols]), MODE_FP32)
        ref = d.astype(np.float64) @ w
        e = {}
        for key, dq in [("block_e4m3", dq_blockwise_act_fmt(db, FMT_E4M3)),
                        ("block_e5m2", dq_blockwise_act_fmt(db, FMT_E5M2)),
                        ("tensor_e4m3", dq_tensor_fmt(d, FMT_E4M3)),
                        ("tensor_e5m2", dq_tensor_fmt(d, FMT_E5M2))]:
            e[key] = rel_err(d, dq)
            e["dX_" + key] = rel_err(ref, dq @ wq)
        rows.append((f"{name} dY [{tokens},{N}]", e))
    return rows


def dq_delayed(bits: np.ndarray, hist: np.ndarray):
    """Per-tensor delayed scaling (E4M3, fp32 scale) of a bf16 tensor with the
    given history.  Returns (dequantized tensor, new history, fraction of
    elements at the saturated code)."""
    q, _, s, _, h = quant_tensor_delayed(bits, hist, MODE_FP32, transposed=False)
    sat = float(np.mean((q & 0x7F) == 0x7E))
    return decode_table()[q] * np.float64(s), h, sat


def magnitude_schedule(steps: int = 40) -> list:
    """Per-step magnitude of the drifting tensor: 3 % growth per step, one
    4x spike at step 12, back on the trend after it."""
    return [1.03 ** t * (4.0 if t == 12 else 1.0) for t in range(steps)]


def delayed_study(tokens: int = 256, seed: int = 0, history: int = 16, schedule=None) -> list:
    """Rows of (step, magnitude, errors) for the o_proj input (with the
    workloads' outlier channels) scaled by `schedule` (default
    `magnitude_schedule()`): blockwise (current 1x128 scales), per-tensor
    current scaling, and per-tensor delayed scaling with a `history`-long
    amax history (zero at step 0)."""
    import torch

    import workloads

    X, _, _ = workloads.llama_layer("o_proj", seed=seed, M=tokens)
    base = X.float()
    hist = np.zeros(history, np.float32)
    rows = []
    for t, m in enumerate(magnitude_schedule() if schedule is None else schedule):
        xb = (base * m).to(torch.bfloat16).contiguous().view(torch.int16).numpy().view(np.uint16)
        x = bf16_bits_to_f32(xb)
        dq, hist, sat = dq_delayed(xb, hist)
        rows.append((t, m, {"blockwise": rel_err(x, dq_blockwise_act(xb, MODE_FP32)),
                            "tensor": rel_err(x, dq_tensor(x)),
                            "delayed": rel_err(x, dq), "saturated": sat}))
    return rows


def main():
    rows = study()
    print("| tensor | blockwise (fp32 s) | blockwise (pow2 s) | per-tensor | MX-32 (floor) | "
          "MX-32 (round up) | blockwise vs per-tensor |")
    print("|---|---|---|---|---|---|---|")
    for name, e in rows:
        red = 1.0 - e["blockwise"] / e["tensor"]
        print(f"| {name} | {e['blockwise']:.4f} | {e['blockwise_pow2']:.4f} | {e['tensor']:.4f} | "
              f"{e['mx32']:.4f} | {e['mx32_up']:.4f} | {100 * red:.0f} % lower |")
    print()
    print("| gradient | 1x128 E4M3 | 1x128 E5M2 | tensor E4M3 | tensor E5M2 | dX: 1x128 E4M3 | "
          "dX: 1x128 E5M2 | dX: tensor E4M3 | dX: tensor E5M2 |")
    print("|---|---|---|---|---|---|---|---|---|")
    for name, e in gradient_study():
        print(f"| {name} | {e['block_e4m3']:.4f} | {e['block_e5m2']:.4f} | {e['tensor_e4m3']:.4f} | "
              f"{e['tensor_e5m2']:.4f} | {e['dX_block_e4m3']:.4f} | {e['dX_block_e5m2']:.4f} | "
              f"{e['dX_tensor_e4m3']:.4f} | {e['dX_tensor_e5m2']:.4f} |")
    print()
    print("| step | magnitude | blockwise | per-tensor (current) | per-tensor (delayed, 16) | "
          "saturated (delayed) |")
    print("|---|---|---|---|---|---|")
    for t, m, e in delayed_study():
        print(f"| {t} | {m:.2f} | {e['blockwise']:.4f} | {e['tensor']:.4f} | {e['delayed']:.4f} | "
              f"{100 * e['saturated']:.3f} % |")


if __name__ == "__main__":
    main()

"""Python binding of libfp8bw.so, the blockwise-scaled FP8 linear layer for B200.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/fp8bw.h``.  Functions keep the
C names.  Each takes torch CUDA tensors (used for their device memory only),
derives sizes from their shapes, passes raw pointers, launches on the current
torch stream and raises ``Fp8bwError`` on a non-OK status.  There is no CPU
fallback: if the library is missing this module fails to import.

``raw`` is the ctypes handle with the C prototypes, for pointer-level calls.
The library is loaded on first use (``load()``), so that building it does not
require an already-built copy.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8bw.so")

FP8BW_OK = 0
FP8BW_SCALE_FP32, FP8BW_SCALE_POW2 = 0, 1
FP8BW_FPROP, FP8BW_DGRAD, FP8BW_WGRAD = 0, 1, 2
FP8BW_FMT_E4M3, FP8BW_FMT_E5M2 = 0, 1
FP8BW_REQUANT_MAX_PER_LAUNCH = 256
FP8BW_MAX_EXPERTS = 512
FP8BW_MAX_HISTORY = 1024
FP8BW_ATTN_MAX_SEGMENTS = 65536
FP8BW_ATTN_MAX_HEADS = 1024
STATUS = {0: "FP8BW_OK", 1: "FP8BW_ERR_INVALID_ARG", 2: "FP8BW_ERR_ALIGNMENT",
          3: "FP8BW_ERR_UNSUPPORTED_ARCH", 4: "FP8BW_ERR_CUDA", 5: "FP8BW_ERR_TIMEOUT",
          6: "FP8BW_ERR_DEVICE_CHECK", 7: "FP8BW_ERR_TOO_LARGE"}


class Fp8bwError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {STATUS.get(status, status)} ({status_string(status)})")


class fp8bw_weight_desc(ctypes.Structure):
    _fields_ = [("w", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("ldw", ctypes.c_int64), ("q", ctypes.c_void_p), ("s", ctypes.c_void_p),
                ("qT", ctypes.c_void_p)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m blockwise_scaled_fp8_fp8bw_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
    L.fp8bw_init.argtypes = [i32]
    L.fp8bw_status_string.argtypes = [i32]
    L.fp8bw_status_string.restype = ctypes.c_char_p
    L.fp8bw_last_device_error.argtypes = [vp]
    L.fp8bw_testing_stall_next_gemm.argtypes = [ctypes.c_int32]
    L.fp8bw_quant_act_1x128.argtypes = [vp, i64, i64, i64, i32, vp, vp, vp, vp, vp]
    L.fp8bw_quant_weight_128x128.argtypes = [vp, i64, i64, i64, i32, vp, vp, vp, vp]
    L.fp8bw_requant_weights.argtypes = [ctypes.POINTER(fp8bw_weight_desc), ctypes.c_int32, i32, vp]
    L.fp8bw_gemm.argtypes = [i32, i64, i64, i64, vp, vp, vp, vp, vp, i64, i32, vp]
    L.fp8bw_quant_act_1x128_fmt.argtypes = [vp, i64, i64, i64, i32, i32, vp, vp, vp, vp, vp]
    L.fp8bw_gemm_fmt.argtypes = [i32, i64, i64, i64, vp, vp, i32, vp, vp, i32, vp, i64, i32, vp]
    L.fp8bw_gemm_f32.argtypes = [i32, i64, i64, i64, vp, vp, vp, vp, vp, i64, ctypes.c_int32, i32, vp]
    L.fp8bw_grouped_gemm.argtypes = [i32, ctypes.c_int32, vp, i64, i64, i64, vp, vp, vp, vp, vp, i32, vp]
    L.fp8bw_grouped_wgrad_f32.argtypes = [ctypes.c_int32, vp, i64, i64, i64, vp, vp, vp, vp, vp,
                                          ctypes.c_int32, i32, vp]
    L.fp8bw_gemm_bf16.argtypes = [i64, i64, i64, vp, vp, vp, i64, vp]
    L.fp8bw_quant_tensor_delayed.argtypes = [vp, i64, i64, i64, i32, i32, vp, ctypes.c_int32, vp, vp,
                                             vp, vp, vp, i64, vp]
    L.fp8bw_gemm_quant.argtypes = [i32, i64, i64, i64, vp, vp, vp, vp, i32, vp, i64, vp, vp, vp, vp, vp]
    L.fp8bw_attention_fwd.argtypes = [i64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, vp, vp,
                                      ctypes.c_int32, ctypes.c_int32, vp, vp, vp, vp, vp, vp, vp, vp]
    L.fp8bw_attention_decode.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, i64, vp, vp, vp, vp,
                                         vp, vp, vp, vp]
    for f in ("fp8bw_init", "fp8bw_last_device_error", "fp8bw_testing_stall_next_gemm", "fp8bw_attention_fwd",
              "fp8bw_attention_decode",
              "fp8bw_gemm_quant",
              "fp8bw_quant_act_1x128", "fp8bw_quant_act_1x128_fmt", "fp8bw_gemm_fmt",
              "fp8bw_quant_weight_128x128", "fp8bw_requant_weights", "fp8bw_gemm",
              "fp8bw_gemm_f32", "fp8bw_grouped_gemm", "fp8bw_grouped_wgrad_f32", "fp8bw_gemm_bf16",
              "fp8bw_quant_tensor_delayed"):
        getattr(L, f).restype = i32
    return L


_raw = None


def load():
    """Loads libfp8bw.so (raises ImportError if it is missing or stale)."""
    global _raw
    if _raw is None:
        try:
            _raw = _load()
        except AttributeError as e:  # a symbol of the header is missing: stale build
            raise ImportError(f"{LIB_PATH} is stale ({e}); rebuild it") from e
    return _raw


def __getattr__(name):
    if name == "raw":
        return load()
    raise AttributeError(name)


def status_string(status: int) -> str:
    return load().fp8bw_status_string(int(status)).decode()


def _check(fn: str, status: int) -> None:
    if status != FP8BW_OK:
        raise Fp8bwError(fn, status)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


# --------------------------------------------------------------- calls ----
def fp8bw_init(device: int = 0) -> None:
    _check("fp8bw_init", load().fp8bw_init(int(device)))


def fp8bw_last_device_error(stream=None) -> int:
    """Status of the device error word (synchronizes the stream, clears it)."""
    return load().fp8bw_last_device_error(_stream(stream))


def fp8bw_testing_stall_next_gemm(chunk: int) -> None:
    """Testing hook: the next GEMM launch stalls at `chunk` and times out."""
    _check("fp8bw_testing_stall_next_gemm", load().fp8bw_testing_stall_next_gemm(int(chunk)))


def fp8bw_quant_act_1x128(x, mode, q_row, s_row, q_col=None, s_col=None, stream=None, K=None):
    """x [M, ldx] bf16 (first K columns); q_row [M,K] u8; s_row [K/128,M] f32;
    q_col [K,M] u8 / s_col [M/128,K] f32 or both None."""
    M, ldx = x.shape[0], x.stride(0)
    K = x.shape[1] if K is None else K
    _check("fp8bw_quant_act_1x128", load().fp8bw_quant_act_1x128(
        _ptr(x), M, K, ldx, int(mode), _ptr(q_row), _ptr(s_row), _ptr(q_col), _ptr(s_col),
        _stream(stream)))


def fp8bw_quant_act_1x128_fmt(x, mode, fmt, q_row, s_row, q_col=None, s_col=None, stream=None):
    """fp8bw_quant_act_1x128 with the element format (FP8BW_FMT_E4M3 / _E5M2)."""
    M, K = x.shape
    _check("fp8bw_quant_act_1x128_fmt", load().fp8bw_quant_act_1x128_fmt(
        _ptr(x), M, K, x.stride(0), int(mode), int(fmt), _ptr(q_row), _ptr(s_row), _ptr(q_col),
        _ptr(s_col), _stream(stream)))


def fp8bw_quant_tensor_delayed(x, fmt, mode, hist, q, qT, scale, amax, s_grid=None, stream=None):
    """Per-tensor delayed scaling.  x [M, ldx] bf16; hist [H] f32 (updated);
    q [M,K] u8; qT [K,M] u8 or None; scale, amax: 1-element f32 tensors;
    s_grid: f32 tensor filled with the scale, or None."""
    M, K = x.shape
    n = s_grid.numel() if s_grid is not None else 0
    _check("fp8bw_quant_tensor_delayed", load().fp8bw_quant_tensor_delayed(
        _ptr(x), M, K, x.stride(0), int(fmt), int(mode), _ptr(hist), hist.numel(), _ptr(q),
        _ptr(qT), _ptr(scale), _ptr(amax), _ptr(s_grid), n, _stream(stream)))


def fp8bw_quant_weight_128x128(w, mode, q, s, qT=None, stream=None):
    """w [N, ldw] bf16; q [N,K] u8; s [N/128,K/128] f32; qT [K,N] u8 or None."""
    N, K = w.shape
    _check("fp8bw_quant_weight_128x128", load().fp8bw_quant_weight_128x128(
        _ptr(w), N, K, w.stride(0), int(mode), _ptr(q), _ptr(s), _ptr(qT), _stream(stream)))


def fp8bw_requant_weights(items, mode, stream=None):
    """items: sequence of (w, q, s, qT-or-None) tensors."""
    n = len(items)
    arr = (fp8bw_weight_desc * max(n, 1))()
    for i, (w, q, s, qT) in enumerate(items):
        arr[i] = fp8bw_weight_desc(w.data_ptr(), w.shape[0], w.shape[1], w.stride(0), q.data_ptr(),
                                   s.data_ptr(), qT.data_ptr() if qT is not None else None)
    _check("fp8bw_requant_weights", load().fp8bw_requant_weights(arr, n, int(mode), _stream(stream)))


def fp8bw_gemm(kind, A, sA, B, sB, D, mode=FP8BW_SCALE_FP32, stream=None):
    """A [M,K] u8, sA [K/128,M]; B [N,K] u8, sB per kind; D [M, ldd>=N] bf16."""
    M, K = A.shape
    N = B.shape[0]
    _check("fp8bw_gemm", load().fp8bw_gemm(int(kind), M, N, K, _ptr(A), _ptr(sA), _ptr(B), _ptr(sB),
                                        _ptr(D), D.stride(0), int(mode), _stream(stream)))


def fp8bw_gemm_fmt(kind, A, sA, a_fmt, B, sB, b_fmt, D, mode=FP8BW_SCALE_FP32, stream=None):
    """fp8bw_gemm with the element formats of A and B given."""
    M, K = A.shape
    N = B.shape[0]
    _check("fp8bw_gemm_fmt", load().fp8bw_gemm_fmt(int(kind), M, N, K, _ptr(A), _ptr(sA), int(a_fmt),
                                                _ptr(B), _ptr(sB), int(b_fmt), _ptr(D), D.stride(0),
                                                int(mode), _stream(stream)))


def fp8bw_gemm_f32(kind, A, sA, B, sB, D, accumulate=False, mode=FP8BW_SCALE_FP32, stream=None):
    """As fp8bw_gemm with D [M, ldd>=N] fp32; accumulate: D += result."""
    M, K = A.shape
    N = B.shape[0]
    _check("fp8bw_gemm_f32", load().fp8bw_gemm_f32(int(kind), M, N, K, _ptr(A), _ptr(sA), _ptr(B), _ptr(sB),
                                                _ptr(D), D.stride(0), int(bool(accumulate)), int(mode),
                                                _stream(stream)))


def fp8bw_grouped_gemm(kind, offsets, A, sA, B, sB, D, mode=FP8BW_SCALE_FP32, stream=None):
    """offsets: device int32 [G+1].  FPROP/DGRAD: A [Mtot,K], B [G,N,K], D [Mtot,N].
    WGRAD: A [N,Mtot], B [K,Mtot], D [G,N,K]."""
    G = offsets.numel() - 1
    if kind == FP8BW_WGRAD:
        N, Mtot = A.shape
        K = B.shape[0]
    else:
        Mtot, K = A.shape
        N = B.shape[1]
    _check("fp8bw_grouped_gemm", load().fp8bw_grouped_gemm(
        int(kind), G, _ptr(offsets), Mtot, N, K, _ptr(A), _ptr(sA), _ptr(B), _ptr(sB), _ptr(D),
        int(mode), _stream(stream)))


def fp8bw_grouped_wgrad_f32(offsets, A, sA, B, sB, D, accumulate=False, mode=FP8BW_SCALE_FP32, stream=None):
    """offsets device int32 [G+1]; A [N,Mtot], B [K,Mtot]; D [G,N,K] fp32."""
    G = offsets.numel() - 1
    N, Mtot = A.shape
    K = B.shape[0]
    _check("fp8bw_grouped_wgrad_f32", load().fp8bw_grouped_wgrad_f32(
        G, _ptr(offsets), Mtot, N, K, _ptr(A), _ptr(sA), _ptr(B), _ptr(sB), _ptr(D),
        int(bool(accumulate)), int(mode), _stream(stream)))


def fp8bw_gemm_bf16(A, B, D, stream=None):
    """A [M,K] bf16, B [N,K] bf16, D [M, ldd>=N] bf16."""
    M, K = A.shape
    N = B.shape[0]
    _check("fp8bw_gemm_bf16", load().fp8bw_gemm_bf16(M, N, K, _ptr(A), _ptr(B), _ptr(D), D.stride(0),
                                                  _stream(stream)))


def fp8bw_attention_fwd(q, sq, k, sk, vT, sv, o, seg_off, seg_len, causal=True, mode=FP8BW_SCALE_FP32,
                        stream=None):
    """FP8 attention forward.  q [T, Hq*128] u8, sq [Hq, T]; k [T, Hkv*128] u8,
    sk [Hkv, T]; vT [Hkv*128, T] u8, sv [T/128, Hkv*128]; o [T, Hq*128] bf16;
    seg_off [nseg+1], seg_len [nseg]: device int32; mode: the scales' rule
    (FP8BW_SCALE_POW2: power-of-two scales, applied by the tensor core)."""
    T = q.shape[0]
    Hq, Hkv = q.shape[1] // 128, k.shape[1] // 128
    _check("fp8bw_attention_fwd", load().fp8bw_attention_fwd(
        T, Hq, Hkv, seg_len.numel(), _ptr(seg_off), _ptr(seg_len), int(bool(causal)), int(mode), _ptr(q), _ptr(sq),
        _ptr(k), _ptr(sk), _ptr(vT), _ptr(sv), _ptr(o), _stream(stream)))


def fp8bw_attention_decode(q, k, sk, v, sv, o, lens, Lmax, stream=None):
    """FP8 KV-cache decode attention.  q [B, Hq*128] bf16 (one new token per
    sequence); k, v [B*Lmax, Hkv*128] u8 cache codes, sk, sv [Hkv, B*Lmax]
    fp32 (one scale per token and KV head); lens [B] device int32; o [B,
    Hq*128] bf16."""
    B = q.shape[0]
    Hq, Hkv = q.shape[1] // 128, k.shape[1] // 128
    _check("fp8bw_attention_decode", load().fp8bw_attention_decode(
        B, Hq, Hkv, int(Lmax), _ptr(lens), _ptr(q), _ptr(k), _ptr(sk), _ptr(v), _ptr(sv), _ptr(o),
        _stream(stream)))


def fp8bw_gemm_quant(kind, A, sA, B, sB, q_row, s_row, q_col=None, s_col=None, D=None,
                     mode=FP8BW_SCALE_FP32, stream=None):
    """The GEMM with its bf16 output quantized in the epilogue (scale rule
    `mode`): q_row [M,N] u8, s_row [N/128,M]; q_col [N,M] / s_col [M/128,N] or
    None; D [M, ldd>=N] bf16 or None."""
    M, K = A.shape
    N = B.shape[0]
    _check("fp8bw_gemm_quant", load().fp8bw_gemm_quant(
        int(kind), M, N, K, _ptr(A), _ptr(sA), _ptr(B), _ptr(sB), int(mode), _ptr(D),
        D.stride(0) if D is not None else 0, _ptr(q_row), _ptr(s_row), _ptr(q_col), _ptr(s_col),
        _stream(stream)))

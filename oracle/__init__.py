"""Oracle for the blockwise-scaled FP8 linear layer — TEST INFRASTRUCTURE.

A ctypes front for ``oracle.cpp``, the plain CPU implementation the CUDA
library is checked against.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package; the library
itself never does, and it shares no code with the library.

Every array argument is a numpy array; bf16 tensors travel as their uint16
bit patterns.  Layouts match the C functions (see ``oracle.cpp``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")

MODE_FP32 = 0
MODE_POW2 = 1
FPROP, DGRAD, WGRAD = 0, 1, 2

_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.cpp into liboracle.so next to it (g++, IEEE float)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-ffp-contract=off",
               "-fopenmp", "-o", _LIB + ".tmp", _SRC]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        i64, i32, vp, dbl, flt = (ctypes.c_int64, ctypes.c_int, ctypes.c_void_p,
                                  ctypes.c_double, ctypes.c_float)
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_decode.restype = dbl
        L.orc_e4m3_encode.argtypes = [flt]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_block_scale.argtypes = [flt, i32]
        L.orc_block_scale.restype = flt
        L.orc_e5m2_decode.argtypes = [ctypes.c_uint8]
        L.orc_e5m2_decode.restype = dbl
        L.orc_e5m2_encode.argtypes = [flt]
        L.orc_e5m2_encode.restype = ctypes.c_uint8
        L.orc_e5m2_encode_array.argtypes = [vp, i64, vp]
        L.orc_block_scale_fmt.argtypes = [flt, i32, i32]
        L.orc_block_scale_fmt.restype = flt
        L.orc_quant_act_1x128_fmt.argtypes = [vp, i64, i64, i64, i32, i32, vp, vp, vp, vp]
        L.orc_quant_tensor_delayed.argtypes = [vp, i64, i64, i64, i32, i32, vp, i32, vp, vp,
                                               vp, vp]
        L.orc_gemm_ref_tile_fmt.argtypes = [i32, i32, i32, i64, i64, i64, vp, vp, vp, vp,
                                            i64, i64, i64, i64, vp, vp]
        L.orc_bf16_to_float.argtypes = [ctypes.c_uint16]
        L.orc_bf16_to_float.restype = flt
        L.orc_float_to_bf16.argtypes = [flt]
        L.orc_float_to_bf16.restype = ctypes.c_uint16
        L.orc_e4m3_encode_array.argtypes = [vp, i64, vp]
        L.orc_quant_act_1x128.argtypes = [vp, i64, i64, i64, i32, vp, vp, vp, vp]
        L.orc_quant_weight_128x128.argtypes = [vp, i64, i64, i64, i32, vp, vp, vp]
        L.orc_gemm_ref_tile.argtypes = [i32, i64, i64, i64, vp, vp, vp, vp,
                                        i64, i64, i64, i64, vp, vp]
        L.orc_gemm_ref_points.argtypes = [i32, i64, i64, i64, vp, vp, vp, vp,
                                          vp, vp, i64, vp, vp]
        L.orc_gemm_mimic_tile.argtypes = [i32, i64, i64, i64, vp, vp, vp, vp,
                                          i64, i64, i64, i64, vp]
        L.orc_grouped_gemm_ref_tile.argtypes = [i32, i32, vp, i64, i64, i64, vp, vp,
                                                vp, vp, i32, i64, i64, i64, i64, vp, vp]
        L.orc_gemm_bf16_ref_tile.argtypes = [i64, i64, i64, vp, vp, i64, i64, i64, i64,
                                             vp, vp]
        L.orc_bf16_ulp.argtypes = [dbl]
        L.orc_bf16_ulp.restype = dbl
        L.orc_check_tol.argtypes = [vp, vp, vp, i64, dbl, vp]
        L.orc_check_tol.restype = i64
        L.orc_attention_fwd_rows.argtypes = [i64, i32, i32, i32, vp, vp, i32, vp, vp, vp, vp,
                                             vp, vp, i64, vp, vp, vp, vp, vp, i32]
        L.orc_attention_decode.argtypes = [i32, i32, i32, i64, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.orc_set_threads.argtypes = [i32]
        L.orc_max_threads.restype = i32
        _lib = L
    return _lib


def _u16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def _u8(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint8, a.dtype
    return a


def _f32(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.float32, a.dtype
    return a


def set_threads(n: int) -> None:
    """Threads of the oracle's OpenMP loops (for timing; results do not depend on it)."""
    lib().orc_set_threads(int(n))


def max_threads() -> int:
    return int(lib().orc_max_threads())


# ----------------------------------------------------------------- scalars --
def e4m3_decode(code: int) -> float:
    return lib().orc_e4m3_decode(int(code))


def e4m3_encode(v: float) -> int:
    return int(lib().orc_e4m3_encode(float(v)))


def e4m3_encode_array(v: np.ndarray) -> np.ndarray:
    v = _f32(v)
    out = np.empty(v.shape, np.uint8)
    lib().orc_e4m3_encode_array(_p(v), v.size, _p(out))
    return out


def block_scale(amax: float, mode: int) -> float:
    return lib().orc_block_scale(float(amax), int(mode))


# Element formats: E4M3 (the method's) and E5M2 (the gradient format of the
# per-tensor recipe, "FP8 Trainingsinfrastructuur", "Het landschap van
# numerieke precisie").
FMT_E4M3, FMT_E5M2 = 0, 1


def e5m2_decode(code: int) -> float:
    return lib().orc_e5m2_decode(int(code))


def e5m2_encode(v: float) -> int:
    return int(lib().orc_e5m2_encode(float(v)))


def e5m2_encode_array(v: np.ndarray) -> np.ndarray:
    v = _f32(v)
    out = np.empty(v.shape, np.uint8)
    lib().orc_e5m2_encode_array(_p(v), v.size, _p(out))
    return out


def block_scale_fmt(amax: float, mode: int, fmt: int) -> float:
    return lib().orc_block_scale_fmt(float(amax), int(mode), int(fmt))


def bf16_ulp(v: float) -> float:
    return lib().orc_bf16_ulp(float(v))


# -------------------------------------------------------------- quantizers --
def quant_act_1x128(x_bits: np.ndarray, mode: int, colwise: bool = True, fmt: int = FMT_E4M3):
    """x_bits: uint16 [M, K].  Returns (q_row, s_row, q_col, s_col)."""
    x = _u16(x_bits)
    M, K = x.shape
    q_row = np.empty((M, K), np.uint8)
    s_row = np.empty((K // 128, M), np.float32)
    q_col = np.empty((K, M), np.uint8) if colwise else None
    s_col = np.empty((M // 128, K), np.float32) if colwise else None
    lib().orc_quant_act_1x128_fmt(_p(x), M, K, K, mode, fmt, _p(q_row), _p(s_row),
                                  _p(q_col) if colwise else None,
                                  _p(s_col) if colwise else None)
    return q_row, s_row, q_col, s_col


def quant_weight_128x128(w_bits: np.ndarray, mode: int, transposed: bool = True):
    """w_bits: uint16 [N, K].  Returns (q, s, qT)."""
    w = _u16(w_bits)
    N, K = w.shape
    q = np.empty((N, K), np.uint8)
    s = np.empty((N // 128, K // 128), np.float32)
    qT = np.empty((K, N), np.uint8) if transposed else None
    lib().orc_quant_weight_128x128(_p(w), N, K, K, mode, _p(q), _p(s),
                                   _p(qT) if transposed else None)
    return q, s, qT


def quant_tensor_delayed(x_bits: np.ndarray, hist: np.ndarray, mode: int,
                         fmt: int = FMT_E4M3, transposed: bool = True):
    """Per-tensor delayed scaling ("FP8 Trainingsinfrastructuur", sections
    "Transformer Engine: de softwarebasis" and "Scaling-strategieën en
    stabiliteit").  x_bits: uint16 [M, K]; hist: float32 [H], newest first
    (not modified).  Returns (q, qT, scale, amax, new_hist)."""
    x = _u16(x_bits)
    M, K = x.shape
    h = _f32(hist).copy()
    q = np.empty((M, K), np.uint8)
    qT = np.empty((K, M), np.uint8) if transposed else None
    sc = np.zeros(1, np.float32)
    am = np.zeros(1, np.float32)
    lib().orc_quant_tensor_delayed(_p(x), M, K, K, mode, fmt, _p(h), h.size, _p(q),
                                   _p(qT) if transposed else None, _p(sc), _p(am))
    return q, qT, np.float32(sc[0]), np.float32(am[0]), h


# ------------------------------------------------------------------- GEMMs --
def gemm_ref_tile(kind, A, sA, B, sB, m0, m1, n0, n1, fa=FMT_E4M3, fb=FMT_E4M3):
    """fp64 reference of rows [m0,m1) x cols [n0,n1); fa/fb the element
    formats of the A and B codes.  Returns (y, yabs)."""
    A, B, sA, sB = _u8(A), _u8(B), _f32(sA), _f32(sB)
    M, K = A.shape
    N = B.shape[0]
    y = np.empty((m1 - m0, n1 - n0), np.float64)
    ya = np.empty_like(y)
    lib().orc_gemm_ref_tile_fmt(kind, fa, fb, M, N, K, _p(A), _p(sA), _p(B), _p(sB),
                                m0, m1, n0, n1, _p(y), _p(ya))
    return y, ya


def gemm_ref_points(kind, A, sA, B, sB, pm, pn):
    A, B, sA, sB = _u8(A), _u8(B), _f32(sA), _f32(sB)
    M, K = A.shape
    N = B.shape[0]
    pm = np.ascontiguousarray(pm, np.int64)
    pn = np.ascontiguousarray(pn, np.int64)
    y = np.empty(pm.size, np.float64)
    ya = np.empty_like(y)
    lib().orc_gemm_ref_points(kind, M, N, K, _p(A), _p(sA), _p(B), _p(sB),
                              _p(pm), _p(pn), pm.size, _p(y), _p(ya))
    return y, ya


def gemm_mimic_tile(kind, A, sA, B, sB, m0, m1, n0, n1):
    A, B, sA, sB = _u8(A), _u8(B), _f32(sA), _f32(sB)
    M, K = A.shape
    N = B.shape[0]
    y = np.empty((m1 - m0, n1 - n0), np.uint16)
    lib().orc_gemm_mimic_tile(kind, M, N, K, _p(A), _p(sA), _p(B), _p(sB),
                              m0, m1, n0, n1, _p(y))
    return y


def grouped_gemm_ref_tile(kind, offsets, A, sA, B, sB, expert, m0, m1, n0, n1,
                          N=None, K=None):
    """Grouped reference.  kind 0/1: A [Mtot,K], B [G,N,K]; kind 2: A [N,Mtot],
    B [K,Mtot] and the output tile is of expert `expert`'s dW [N,K]."""
    A, B, sA, sB = _u8(A), _u8(B), _f32(sA), _f32(sB)
    off = np.ascontiguousarray(offsets, np.int32)
    G = off.size - 1
    if kind == 2:
        N, Mtot = A.shape
        K = B.shape[0]
    else:
        Mtot, K = A.shape
        N = B.shape[1]
    y = np.empty((m1 - m0, n1 - n0), np.float64)
    ya = np.empty_like(y)
    lib().orc_grouped_gemm_ref_tile(kind, G, _p(off), Mtot, N, K, _p(A), _p(sA),
                                    _p(B), _p(sB), int(expert), m0, m1, n0, n1,
                                    _p(y), _p(ya))
    return y, ya


def gemm_bf16_ref_tile(A_bits, B_bits, m0, m1, n0, n1):
    A, B = _u16(A_bits), _u16(B_bits)
    M, K = A.shape
    N = B.shape[0]
    y = np.empty((m1 - m0, n1 - n0), np.float64)
    ya = np.empty_like(y)
    lib().orc_gemm_bf16_ref_tile(M, N, K, _p(A), _p(B), m0, m1, n0, n1, _p(y), _p(ya))
    return y, ya


# GEMM acceptance: |y - y_ref| <= REL_TOL * sum_k |a_dq b_dq| + 1 bf16 ulp(y_ref)
REL_TOL = 1e-2


def check_tol(y_bits, yref, yabs, rel=REL_TOL):
    """Returns (violations, worst error/allowance ratio)."""
    y = _u16(y_bits).ravel()
    yref = np.ascontiguousarray(yref, np.float64).ravel()
    yabs = np.ascontiguousarray(yabs, np.float64).ravel()
    worst = np.zeros(1, np.float64)
    bad = lib().orc_check_tol(_p(y), _p(yref), _p(yabs), y.size, rel, _p(worst))
    return int(bad), float(worst[0])


# fp32-output acceptance: the GEMM gate with the bf16 output ulp replaced by
# 2^-22 |y_ref| (two fp32 roundings: the result and, when accumulating, the add)
F32_ABS_REL = 2.0 ** -22


def check_tol_f32(y, yref, yabs, rel=REL_TOL):
    """|y - y_ref| <= rel * yabs + 2^-22 |y_ref| elementwise (NaN fails).
    Returns (violations, worst error/allowance ratio)."""
    y = np.asarray(y, np.float64).ravel()
    yref = np.asarray(yref, np.float64).ravel()
    lim = rel * np.asarray(yabs, np.float64).ravel() + F32_ABS_REL * np.abs(yref)
    err = np.abs(y - yref)
    ok = err <= lim
    ratio = np.where(lim > 0, err / np.where(lim > 0, lim, 1.0), np.where(err > 0, np.inf, 0.0))
    worst = float(np.max(np.where(np.isnan(ratio), np.inf, ratio))) if ratio.size else 0.0
    return int(np.count_nonzero(~ok)), worst


# ------------------------------------------------------------- attention --
HEAD_DIM = 128


def attention_fwd_rows(q, sq, k, sk, vT, sv, Hq, Hkv, seg_off, seg_len, causal, rows_t, rows_h, mode=0):
    """FP8 attention forward reference ("NVIDIA NeMo RL erreicht 48% ...",
    "Leistungsgewinne in der Praxis": FP8 KV cache and attention) for the
    (token, head) rows given.  q [T, Hq*128] codes, sq [Hq, T]; k [T, Hkv*128],
    sk [Hkv, T]; vT [Hkv*128, T] codes of V's column-wise copy, sv
    [T/128, Hkv*128]; seg_off [nseg+1] (multiples of 128), seg_len [nseg].
    mode 0: P's block scale by the FP32 rule; mode 1: power-of-2 scales (P
    taken against an integer power-of-two reference maximum).
    Returns (O [n,128], oabs [n,128], oflip [n,128]) in fp64."""
    q, k, vT = _u8(q), _u8(k), _u8(vT)
    sq, sk, sv = _f32(sq), _f32(sk), _f32(sv)
    T = q.shape[0]
    off = np.ascontiguousarray(seg_off, np.int32)
    ln = np.ascontiguousarray(seg_len, np.int32)
    rt = np.ascontiguousarray(rows_t, np.int64)
    rh = np.ascontiguousarray(rows_h, np.int32)
    n = rt.size
    out = np.empty((n, HEAD_DIM), np.float64)
    oa = np.empty_like(out)
    of = np.empty_like(out)
    lib().orc_attention_fwd_rows(T, int(Hq), int(Hkv), ln.size, _p(off), _p(ln), int(bool(causal)),
                                 _p(q), _p(sq), _p(k), _p(sk), _p(vT), _p(sv), n, _p(rt), _p(rh),
                                 _p(out), _p(oa), _p(of), int(mode))
    return out, oa, of


def attention_decode(q_bits, k, sk, v, sv, Hq, Hkv, lens, Lmax):
    """FP8 KV-cache decode attention reference ("NVIDIA NeMo RL erreicht 48%
    ...", "Leistungsgewinne in der Praxis": FP8 KV cache and attention in
    generation): one bf16 query token per sequence, q_bits uint16 [B,
    Hq*128]; the cache k, v [B*Lmax, Hkv*128] E4M3 codes with scales sk, sv
    [Hkv, B*Lmax] (one per token and KV head); lens [B].  Returns (O, oabs,
    oerr), each [B, Hq, 128] fp64 (oerr: the fp32 logit-error allowance)."""
    q = _u16(q_bits)
    k, v = _u8(k), _u8(v)
    sk, sv = _f32(sk), _f32(sv)
    B = q.shape[0]
    ln = np.ascontiguousarray(lens, np.int32)
    out = np.empty((B, int(Hq), HEAD_DIM), np.float64)
    oa = np.empty_like(out)
    oe = np.empty_like(out)
    lib().orc_attention_decode(int(B), int(Hq), int(Hkv), int(Lmax), _p(ln), _p(q), _p(k), _p(sk),
                               _p(v), _p(sv), _p(out), _p(oa), _p(oe))
    return out, oa, oe


def check_tol_attn(y_bits, oref, oabs, oflip, rel=REL_TOL):
    """Attention gate: |y - O| <= rel * oabs + oflip + 1 bf16 ulp(O), with y
    bf16 bits.  Returns (violations, worst error/allowance ratio)."""
    y = _u16(y_bits).ravel()
    oref = np.ascontiguousarray(oref, np.float64).ravel()
    yabs = (np.ascontiguousarray(oabs, np.float64).ravel() +
            np.ascontiguousarray(oflip, np.float64).ravel() / rel)
    worst = np.zeros(1, np.float64)
    bad = lib().orc_check_tol(_p(y), _p(oref), _p(yabs), y.size, rel, _p(worst))
    return int(bad), float(worst[0])

"""The C-ABI library loads, exports every call its header declares, and
rejects invalid arguments on the host (no GPU needed: none of these calls
reaches the device)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8bw.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"FP8BW_API\s+[\w\s\*]+?\b(fp8bw_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from blockwise_scaled_fp8_fp8bw_b200 import build
    build.build()
    import blockwise_scaled_fp8_fp8bw_b200 as fb
    return fb


def test_header_declares_the_calls():
    names = _declared()
    for n in ["fp8bw_quant_act_1x128", "fp8bw_quant_weight_128x128", "fp8bw_requant_weights",
              "fp8bw_gemm", "fp8bw_grouped_gemm", "fp8bw_gemm_bf16", "fp8bw_init",
              "fp8bw_status_string", "fp8bw_last_device_error", "fp8bw_quant_tensor_delayed"]:
        assert n in names


def test_exports_every_declared_symbol(lib):
    so = ctypes.CDLL(lib.LIB_PATH)
    for n in _declared():
        assert hasattr(so, n), n


def test_status_strings(lib):
    for s in range(8):
        assert lib.status_string(s) and lib.status_string(s) != "unknown status"
    assert lib.status_string(99) == "unknown status"


def test_host_validation(lib):
    r = lib.raw
    p = ctypes.c_void_p(0x10000)      # 16-byte aligned, never dereferenced
    odd = ctypes.c_void_p(0x10008)    # misaligned
    N = None
    # null pointers
    assert r.fp8bw_gemm(0, 128, 128, 128, N, p, p, p, p, 128, 0, N) == 1
    assert r.fp8bw_quant_act_1x128(N, 128, 128, 128, 0, p, p, N, N, N) == 1
    # q_col without s_col
    assert r.fp8bw_quant_act_1x128(p, 128, 128, 128, 0, p, p, p, N, N) == 1
    # bad enums
    assert r.fp8bw_gemm(3, 128, 128, 128, p, p, p, p, p, 128, 0, N) == 1
    assert r.fp8bw_gemm(0, 128, 128, 128, p, p, p, p, p, 128, 2, N) == 1
    assert r.fp8bw_quant_weight_128x128(p, 128, 128, 128, 5, p, p, N, N) == 1
    # sizes not multiples of 128, misaligned pointers, bad leading dims
    assert r.fp8bw_gemm(0, 130, 128, 128, p, p, p, p, p, 128, 0, N) == 2
    assert r.fp8bw_gemm(0, 128, 128, 128, odd, p, p, p, p, 128, 0, N) == 2
    assert r.fp8bw_gemm(0, 128, 128, 128, p, p, p, p, p, 132, 0, N) == 2
    assert r.fp8bw_gemm(0, 128, 256, 128, p, p, p, p, p, 128, 0, N) == 1   # ldd < N
    assert r.fp8bw_quant_act_1x128(p, 128, 200, 256, 0, p, p, N, N, N) == 2
    assert r.fp8bw_quant_act_1x128(p, 128, 128, 100, 0, p, p, N, N, N) == 1   # ldx < K
    # activation codes leave in 32-byte stores: q_row / q_col 32-byte aligned
    p16 = ctypes.c_void_p(0x10010)
    assert r.fp8bw_quant_act_1x128(p, 128, 128, 128, 0, p16, p, N, N, N) == 2
    assert r.fp8bw_quant_act_1x128(p, 128, 128, 128, 0, p, p, p16, p, N) == 2
    assert r.fp8bw_quant_act_1x128_fmt(p, 128, 128, 128, 0, 1, p, p, p16, p, N) == 2
    assert r.fp8bw_gemm_bf16(128, 128, 100, p, p, p, 128, N) == 2
    # element formats: only E4M3 (0) and E5M2 (1)
    assert r.fp8bw_quant_act_1x128_fmt(p, 128, 128, 128, 0, 2, p, p, N, N, N) == 1
    assert r.fp8bw_gemm_fmt(1, 128, 128, 128, p, p, 2, p, p, 0, p, 128, 0, N) == 1
    assert r.fp8bw_gemm_fmt(1, 128, 128, 128, p, p, 1, p, p, 3, p, 128, 0, N) == 1
    # fp32 output: accumulate flag, 16-byte rows (ldd a multiple of 4), ldd >= N
    assert r.fp8bw_gemm_f32(2, 128, 128, 128, p, p, p, p, p, 128, 2, 0, N) == 1
    assert r.fp8bw_gemm_f32(2, 128, 128, 128, p, p, p, p, p, 130, 1, 0, N) == 2
    assert r.fp8bw_gemm_f32(2, 128, 256, 128, p, p, p, p, p, 128, 1, 0, N) == 1
    assert r.fp8bw_gemm_f32(2, 128, 128, 128, p, p, p, p, odd, 128, 1, 0, N) == 2
    # grouped: bad G, too many experts, misaligned offsets
    assert r.fp8bw_grouped_gemm(0, 0, p, 128, 128, 128, p, p, p, p, p, 0, N) == 1
    assert r.fp8bw_grouped_gemm(0, 2000, p, 128, 128, 128, p, p, p, p, p, 0, N) == 7
    assert r.fp8bw_grouped_gemm(0, 4, ctypes.c_void_p(0x10002), 128, 128, 128, p, p, p, p, p, 0, N) == 2
    # too large
    assert r.fp8bw_gemm(0, 1 << 31, 128, 128, p, p, p, p, p, 128, 0, N) == 7
    # requant: a bad descriptor anywhere rejects the whole batch
    d = (lib.fp8bw_weight_desc * 2)()
    d[0] = lib.fp8bw_weight_desc(0x10000, 128, 128, 128, 0x10000, 0x10000, None)
    d[1] = lib.fp8bw_weight_desc(0x10000, 128, 136, 136, 0x10000, 0x10000, None)
    assert r.fp8bw_requant_weights(d, 2, 0, N) == 2
    assert r.fp8bw_requant_weights(None, 1, 0, N) == 1
    # per-tensor delayed scaling: formats, history length, 32-byte operands,
    # ldx a multiple of 16, a grid length needs a grid
    q32, p16 = ctypes.c_void_p(0x10020), ctypes.c_void_p(0x10010)
    dl = r.fp8bw_quant_tensor_delayed
    assert dl(N, 128, 128, 128, 0, 0, p, 16, q32, N, p, p, N, 0, N) == 1
    assert dl(p, 128, 128, 128, 2, 0, p, 16, q32, N, p, p, N, 0, N) == 1
    assert dl(p, 128, 128, 128, 0, 2, p, 16, q32, N, p, p, N, 0, N) == 1
    assert dl(p, 128, 128, 128, 0, 0, p, 0, q32, N, p, p, N, 0, N) == 1
    assert dl(p, 128, 128, 128, 0, 0, p, 1025, q32, N, p, p, N, 0, N) == 1
    assert dl(p, 128, 128, 128, 0, 0, N, 16, q32, N, p, p, N, 0, N) == 1
    assert dl(p, 128, 128, 128, 0, 0, p, 16, q32, N, p, p, N, 64, N) == 1
    assert dl(p, 130, 128, 128, 0, 0, p, 16, q32, N, p, p, N, 0, N) == 2
    assert dl(p, 128, 128, 136, 0, 0, p, 16, q32, N, p, p, N, 0, N) == 2
    assert dl(p16, 128, 128, 128, 0, 0, p, 16, q32, N, p, p, N, 0, N) == 2
    assert dl(p, 128, 128, 128, 0, 0, p, 16, p16, N, p, p, N, 0, N) == 2
    assert dl(p, 128, 128, 128, 0, 0, p, 16, q32, p16, p, p, N, 0, N) == 2
    assert dl(p, 128, 128, 128, 0, 0, ctypes.c_void_p(0x10002), 16, q32, N, p, p, N, 0, N) == 2
    # KV-cache decode: null pointers, Hq not a multiple of Hkv, a group size
    # outside {1, 2, 4, 8}, Lmax 0 or not a multiple of 128, misaligned scales
    dec = r.fp8bw_attention_decode
    assert dec(2, 4, 2, 128, N, p, p, p, p, p, p, N) == 1
    assert dec(2, 6, 4, 128, p, p, p, p, p, p, p, N) == 1
    assert dec(2, 12, 4, 128, p, p, p, p, p, p, p, N) == 1
    assert dec(2, 32, 2, 128, p, p, p, p, p, p, p, N) == 1
    assert dec(2, 4, 2, 0, p, p, p, p, p, p, p, N) == 1
    assert dec(2, 4, 2, 200, p, p, p, p, p, p, p, N) == 2
    assert dec(2, 4, 2, 128, p, p, p, ctypes.c_void_p(0x10004), p, p, p, N) == 2
    # testing hook: only chunk >= -1 is accepted; -1 cancels
    assert r.fp8bw_testing_stall_next_gemm(-2) == 1
    assert r.fp8bw_testing_stall_next_gemm(-1) == 0


def _param_counts():
    """Parameter count of every FP8BW_API function in the header."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"FP8BW_API\s+[\w\s\*]+?\b(fp8bw_\w+)\s*\(([^)]*)\)", src):
        params = [p for p in m.group(2).split(",") if p.strip() and p.strip() != "void"]
        out[m.group(1)] = len(params)
    return out


def test_binding_argtypes_match_the_header(lib):
    """The ctypes binding declares, for every call it wraps, as many arguments
    as the header's prototype has (a drifted wrapper would shift arguments)."""
    raw = lib.load()
    counts = _param_counts()
    checked = 0
    for name, n in counts.items():
        fn = getattr(raw, name)
        if fn.argtypes is None:
            continue
        assert len(fn.argtypes) == n, (name, len(fn.argtypes), n)
        checked += 1
    assert checked >= 14

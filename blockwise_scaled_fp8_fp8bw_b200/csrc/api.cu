// C ABI of the library (declared in include/fp8bw.h): host-side argument
// validation, device checks and kernel launches.  Nothing here allocates
// device memory; no exception, abort or assert crosses the boundary.

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/fp8bw.h"

namespace fp8bw {
cudaError_t launch_quant_act(const void* x, int64_t M, int64_t K, int64_t ldx, int mode,
                             uint8_t* q_row, float* s_row, uint8_t* q_col, float* s_col,
                             int num_sms, cudaStream_t st, int fmt = 0);
cudaError_t launch_quant_weight(const void* w, int64_t N, int64_t K, int64_t ldw, int mode,
                                uint8_t* q, float* s, uint8_t* qT, cudaStream_t st);
cudaError_t launch_requant(const fp8bw_weight_desc* d, int32_t n, int mode, cudaStream_t st);
cudaError_t launch_gemm_fp8(int kind, bool grouped, int G, const int32_t* d_off, int64_t M,
                            int64_t N, int64_t K, const uint8_t* A, const float* sA,
                            const uint8_t* B, const float* sB, void* D, int64_t ldd, int mode,
                            int num_sms, cudaStream_t st, int out_mode, int a_fmt = 0, int b_fmt = 0);
cudaError_t launch_gemm_quant(int kind, int64_t M, int64_t N, int64_t K, const uint8_t* A, const float* sA,
                              const uint8_t* B, const float* sB, int qmode, void* D, int64_t ldd,
                              uint8_t* q_row, float* s_row, uint8_t* q_col, float* s_col, int num_sms,
                              cudaStream_t st);
cudaError_t launch_gemm_bf16(int64_t M, int64_t N, int64_t K, const void* A, const void* B,
                             void* D, int64_t ldd, int num_sms, cudaStream_t st);
cudaError_t launch_quant_tensor(const void* x, int64_t M, int64_t K, int64_t ldx, int mode,
                                int fmt, float* hist, int H, uint8_t* q, uint8_t* qT,
                                float* scale, float* amax, float* s_grid, int64_t s_grid_len,
                                int num_sms, cudaStream_t st);
cudaError_t launch_attention_fwd(int64_t T, int Hq, int Hkv, int nseg, const int32_t* d_off,
                                 const int32_t* d_len, int causal, int mode, const uint8_t* q, const float* sq,
                                 const uint8_t* k, const float* sk, const uint8_t* vT, const float* sv,
                                 void* o, cudaStream_t st);
cudaError_t gemm_read_clear_error(uint32_t* out, cudaStream_t st);
cudaError_t quant_read_clear_error(uint32_t* out, cudaStream_t st);
cudaError_t attn_read_clear_error(uint32_t* out, cudaStream_t st);
cudaError_t launch_attention_decode(int B, int Hq, int Hkv, int64_t Lmax, const int32_t* d_len,
                                    const void* q, const uint8_t* k, const float* sk, const uint8_t* v,
                                    const float* sv, void* o, cudaStream_t st);
cudaError_t dec_read_clear_error(uint32_t* out, cudaStream_t st);
extern int gemm_stall_chunk;
}  // namespace fp8bw

namespace {

constexpr int kMaxDevices = 64;
int g_sms[kMaxDevices];  // 0 = not initialised, -1 = unsupported

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// The activation quantizer writes its codes with 32-byte stores.
inline bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }
inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
inline bool mult128(int64_t v) { return v >= 0 && (v & 127) == 0; }
constexpr int64_t kMaxDim = int64_t(1) << 30;  // sizes index with 32-bit tile math

fp8bw_status init_device(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return FP8BW_ERR_INVALID_ARG;
  if (g_sms[dev] > 0) return FP8BW_OK;
  if (g_sms[dev] < 0) return FP8BW_ERR_UNSUPPORTED_ARCH;
  int major = 0, minor = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return FP8BW_ERR_CUDA;
  if (major != 10 || minor != 0) {
    g_sms[dev] = -1;
    return FP8BW_ERR_UNSUPPORTED_ARCH;
  }
  g_sms[dev] = sms;
  return FP8BW_OK;
}

fp8bw_status current(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FP8BW_ERR_CUDA;
  fp8bw_status s = init_device(dev);
  if (s == FP8BW_OK) *sms = g_sms[dev];
  return s;
}

inline fp8bw_status from_cuda(cudaError_t e) { return e == cudaSuccess ? FP8BW_OK : FP8BW_ERR_CUDA; }

fp8bw_status check_weight(const void* w, int64_t N, int64_t K, int64_t ldw, const uint8_t* q,
                          const float* s, const uint8_t* qT) {
  if (!w || !q || !s) return FP8BW_ERR_INVALID_ARG;
  if (N < 0 || K < 0 || ldw < K) return FP8BW_ERR_INVALID_ARG;
  if (N > kMaxDim || K > kMaxDim) return FP8BW_ERR_TOO_LARGE;
  if (!mult128(N) || !mult128(K) || (ldw & 7) != 0) return FP8BW_ERR_ALIGNMENT;
  if (!aligned16(w) || !aligned16(q) || !aligned16(s) || (qT && !aligned16(qT)))
    return FP8BW_ERR_ALIGNMENT;
  return FP8BW_OK;
}

}  // namespace

extern "C" {

FP8BW_API fp8bw_status fp8bw_init(int device) { return init_device(device); }

FP8BW_API const char* fp8bw_status_string(fp8bw_status s) {
  switch (s) {
    case FP8BW_OK: return "ok";
    case FP8BW_ERR_INVALID_ARG: return "invalid argument";
    case FP8BW_ERR_ALIGNMENT: return "size or pointer alignment";
    case FP8BW_ERR_UNSUPPORTED_ARCH: return "unsupported architecture (needs sm_100)";
    case FP8BW_ERR_CUDA: return "CUDA error";
    case FP8BW_ERR_TIMEOUT: return "device-side wait timed out";
    case FP8BW_ERR_DEVICE_CHECK: return "device-side argument check failed";
    case FP8BW_ERR_TOO_LARGE: return "size exceeds the supported maximum";
  }
  return "unknown status";
}

FP8BW_API fp8bw_status fp8bw_testing_stall_next_gemm(int32_t chunk) {
  if (chunk < -1) return FP8BW_ERR_INVALID_ARG;
  fp8bw::gemm_stall_chunk = chunk;
  return FP8BW_OK;
}

FP8BW_API fp8bw_status fp8bw_last_device_error(fp8bw_stream_t stream) {
  uint32_t v = 0, vq = 0, va = 0, vd = 0;
  const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (fp8bw::gemm_read_clear_error(&v, cs) != cudaSuccess) return FP8BW_ERR_CUDA;
  if (fp8bw::quant_read_clear_error(&vq, cs) != cudaSuccess) return FP8BW_ERR_CUDA;
  if (fp8bw::attn_read_clear_error(&va, cs) != cudaSuccess) return FP8BW_ERR_CUDA;
  if (fp8bw::dec_read_clear_error(&vd, cs) != cudaSuccess) return FP8BW_ERR_CUDA;
  v |= vq | va | vd;
  if (v & 1u) return FP8BW_ERR_TIMEOUT;
  if (v & 2u) return FP8BW_ERR_DEVICE_CHECK;
  return FP8BW_OK;
}

FP8BW_API fp8bw_status fp8bw_quant_act_1x128(const void* x, int64_t M, int64_t K, int64_t ldx,
                                   fp8bw_scale_mode mode, uint8_t* q_row, float* s_row,
                                   uint8_t* q_col, float* s_col, fp8bw_stream_t stream) {
  return fp8bw_quant_act_1x128_fmt(x, M, K, ldx, mode, FP8BW_FMT_E4M3, q_row, s_row, q_col, s_col,
                                   stream);
}

FP8BW_API fp8bw_status fp8bw_quant_act_1x128_fmt(const void* x, int64_t M, int64_t K, int64_t ldx,
                                       fp8bw_scale_mode mode, fp8bw_format fmt,
                                       uint8_t* q_row, float* s_row, uint8_t* q_col,
                                       float* s_col, fp8bw_stream_t stream) {
  if (fmt != FP8BW_FMT_E4M3 && fmt != FP8BW_FMT_E5M2) return FP8BW_ERR_INVALID_ARG;
  if (!x || !q_row || !s_row) return FP8BW_ERR_INVALID_ARG;
  if ((q_col == nullptr) != (s_col == nullptr)) return FP8BW_ERR_INVALID_ARG;
  if (mode != FP8BW_SCALE_FP32 && mode != FP8BW_SCALE_POW2) return FP8BW_ERR_INVALID_ARG;
  if (M < 0 || K < 0 || ldx < K) return FP8BW_ERR_INVALID_ARG;
  if (M > kMaxDim || K > kMaxDim || M / 128 > 65535) return FP8BW_ERR_TOO_LARGE;
  if (!mult128(M) || !mult128(K) || (ldx & 7) != 0) return FP8BW_ERR_ALIGNMENT;
  if (!aligned16(x) || !aligned32(q_row) || !aligned16(s_row) || (q_col && !aligned32(q_col)) ||
      (s_col && !aligned16(s_col)))
    return FP8BW_ERR_ALIGNMENT;
  int sms = 0;
  fp8bw_status s = current(&sms);
  if (s != FP8BW_OK) return s;
  if (M == 0 || K == 0) return FP8BW_OK;
  return from_cuda(fp8bw::launch_quant_act(x, M, K, ldx, mode, q_row, s_row, q_col, s_col, sms,
                                           reinterpret_cast<cudaStream_t>(stream), fmt));
}

FP8BW_API fp8bw_status fp8bw_quant_weight_128x128(const void* w, int64_t N, int64_t K, int64_t ldw,
                                        fp8bw_scale_mode mode, uint8_t* q, float* s, uint8_t* qT,
                                        fp8bw_stream_t stream) {
  if (mode != FP8BW_SCALE_FP32 && mode != FP8BW_SCALE_POW2) return FP8BW_ERR_INVALID_ARG;
  fp8bw_status st = check_weight(w, N, K, ldw, q, s, qT);
  if (st != FP8BW_OK) return st;
  if (N / 128 > 65535) return FP8BW_ERR_TOO_LARGE;
  int sms = 0;
  st = current(&sms);
  if (st != FP8BW_OK) return st;
  if (N == 0 || K == 0) return FP8BW_OK;
  return from_cuda(fp8bw::launch_quant_weight(w, N, K, ldw, mode, q, s, qT,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

FP8BW_API fp8bw_status fp8bw_requant_weights(const fp8bw_weight_desc* descs, int32_t n,
                                   fp8bw_scale_mode mode, fp8bw_stream_t stream) {
  if (n < 0 || (n > 0 && !descs)) return FP8BW_ERR_INVALID_ARG;
  if (mode != FP8BW_SCALE_FP32 && mode != FP8BW_SCALE_POW2) return FP8BW_ERR_INVALID_ARG;
  int64_t total = 0;
  for (int32_t i = 0; i < n; ++i) {
    const fp8bw_weight_desc& d = descs[i];
    fp8bw_status st = check_weight(d.w, d.N, d.K, d.ldw, d.q, d.s, d.qT);
    if (st != FP8BW_OK) return st;
    total += (d.N / 128) * (d.K / 128);
  }
  if (total > 0x7FFFFFFF) return FP8BW_ERR_TOO_LARGE;
  int sms = 0;
  fp8bw_status st = current(&sms);
  if (st != FP8BW_OK) return st;
  if (n == 0) return FP8BW_OK;
  return from_cuda(fp8bw::launch_requant(descs, n, mode, reinterpret_cast<cudaStream_t>(stream)));
}

FP8BW_API fp8bw_status fp8bw_gemm(fp8bw_gemm_kind kind, int64_t M, int64_t N, int64_t K, const uint8_t* A,
                        const float* sA, const uint8_t* B, const float* sB, void* D, int64_t ldd,
                        fp8bw_scale_mode mode, fp8bw_stream_t stream) {
  return fp8bw_gemm_fmt(kind, M, N, K, A, sA, FP8BW_FMT_E4M3, B, sB, FP8BW_FMT_E4M3, D, ldd, mode,
                        stream);
}

FP8BW_API fp8bw_status fp8bw_gemm_fmt(fp8bw_gemm_kind kind, int64_t M, int64_t N, int64_t K,
                            const uint8_t* A, const float* sA, fp8bw_format a_fmt,
                            const uint8_t* B, const float* sB, fp8bw_format b_fmt,
                            void* D, int64_t ldd, fp8bw_scale_mode mode,
                            fp8bw_stream_t stream) {
  if (kind != FP8BW_FPROP && kind != FP8BW_DGRAD && kind != FP8BW_WGRAD) return FP8BW_ERR_INVALID_ARG;
  if ((a_fmt != FP8BW_FMT_E4M3 && a_fmt != FP8BW_FMT_E5M2) ||
      (b_fmt != FP8BW_FMT_E4M3 && b_fmt != FP8BW_FMT_E5M2))
    return FP8BW_ERR_INVALID_ARG;
  if (mode != FP8BW_SCALE_FP32 && mode != FP8BW_SCALE_POW2) return FP8BW_ERR_INVALID_ARG;
  if (!A || !sA || !B || !sB || !D) return FP8BW_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || K < 0 || ldd < N) return FP8BW_ERR_INVALID_ARG;
  if (M > kMaxDim || N > kMaxDim || K > kMaxDim) return FP8BW_ERR_TOO_LARGE;
  if (!mult128(M) || !mult128(N) || !mult128(K) || (ldd & 7) != 0) return FP8BW_ERR_ALIGNMENT;
  if (!aligned16(A) || !aligned16(B) || !aligned16(D) || !aligned16(sA) || !aligned16(sB))
    return FP8BW_ERR_ALIGNMENT;
  int sms = 0;
  fp8bw_status st = current(&sms);
  if (st != FP8BW_OK) return st;
  if (M == 0 || N == 0) return FP8BW_OK;
  if (K == 0) return from_cuda(cudaMemset2DAsync(D, ldd * 2, 0, N * 2, M, reinterpret_cast<cudaStream_t>(stream)));
  return from_cuda(fp8bw::launch_gemm_fp8(kind, false, 0, nullptr, M, N, K, A, sA, B, sB, D, ldd,
                                          mode, sms, reinterpret_cast<cudaStream_t>(stream), 0,
                                          a_fmt, b_fmt));
}

FP8BW_API fp8bw_status fp8bw_gemm_f32(fp8bw_gemm_kind kind, int64_t M, int64_t N, int64_t K,
                            const uint8_t* A, const float* sA, const uint8_t* B,
                            const float* sB, float* D, int64_t ldd, int32_t accumulate,
                            fp8bw_scale_mode mode, fp8bw_stream_t stream) {
  if (kind != FP8BW_FPROP && kind != FP8BW_DGRAD && kind != FP8BW_WGRAD) return FP8BW_ERR_INVALID_ARG;
  if (mode != FP8BW_SCALE_FP32 && mode != FP8BW_SCALE_POW2) return FP8BW_ERR_INVALID_ARG;
  if (accumulate != 0 && accumulate != 1) return FP8BW_ERR_INVALID_ARG;
  if (!A || !sA || !B || !sB || !D) return FP8BW_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || K < 0 || ldd < N) return FP8BW_ERR_INVALID_ARG;
  if (M > kMaxDim || N > kMaxDim || K > kMaxDim) return FP8BW_ERR_TOO_LARGE;
  if (!mult128(M) || !mult128(N) || !mult128(K) || (ldd & 3) != 0) return FP8BW_ERR_ALIGNMENT;
  if (!aligned16(A) || !aligned16(B) || !aligned16(D) || !aligned16(sA) || !aligned16(sB))
    return FP8BW_ERR_ALIGNMENT;
  int sms = 0;
  fp8bw_status st = current(&sms);
  if (st != FP8BW_OK) return st;
  if (M == 0 || N == 0) return FP8BW_OK;
  const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0) return accumulate ? FP8BW_OK : from_cuda(cudaMemset2DAsync(D, ldd * 4, 0, N * 4, M, cs));
  return from_cuda(fp8bw::launch_gemm_fp8(kind, false, 0, nullptr, M, N, K, A, sA, B, sB, D, ldd,
                                          mode, sms, cs, accumulate ? 2 : 1));
}

FP8BW_API fp8bw_status fp8bw_grouped_gemm(fp8bw_gemm_kind kind, int32_t G, const int32_t* d_offsets,
                                int64_t M_total_pad, int64_t N, int64_t K, const uint8_t* A,
                                const float* sA, const uint8_t* B, const float* sB, void* D,
                                fp8bw_scale_mode mode, fp8bw_stream_t stream) {
  if (kind != FP8BW_FPROP && kind != FP8BW_DGRAD && kind != FP8BW_WGRAD) return FP8BW_ERR_INVALID_ARG;
  if (mode != FP8BW_SCALE_FP32 && mode != FP8BW_SCALE_POW2) return FP8BW_ERR_INVALID_ARG;
  if (!d_offsets || !A || !sA || !B || !sB || !D) return FP8BW_ERR_INVALID_ARG;
  if (G < 1 || M_total_pad < 0 || N < 0 || K < 0) return FP8BW_ERR_INVALID_ARG;
  if (G > FP8BW_MAX_EXPERTS) return FP8BW_ERR_TOO_LARGE;
  if (M_total_pad > kMaxDim || N > kMaxDim || K > kMaxDim) return FP8BW_ERR_TOO_LARGE;
  if (!mult128(M_total_pad) || !mult128(N) || !mult128(K)) return FP8BW_ERR_ALIGNMENT;
  if (!aligned16(A) || !aligned16(B) || !aligned16(D) || !aligned16(sA) || !aligned16(sB) ||
      (reinterpret_cast<uintptr_t>(d_offsets) & 3u))
    return FP8BW_ERR_ALIGNMENT;
  if ((int64_t)G * N * K > (int64_t(1) << 40)) return FP8BW_ERR_TOO_LARGE;
  int sms = 0;
  fp8bw_status st = current(&sms);
  if (st != FP8BW_OK) return st;
  const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (kind == FP8BW_WGRAD) {
    // GEMM sizes: rows = N (out), cols = K (in), contraction = tokens.
    if (N == 0 || K == 0) return FP8BW_OK;
    return from_cuda(fp8bw::launch_gemm_fp8(kind, true, G, d_offsets, N, K, M_total_pad, A, sA, B,
                                            sB, D, K, mode, sms, cs, 0));
  }
  if (M_total_pad == 0 || N == 0) return FP8BW_OK;
  if (K == 0) return FP8BW_ERR_INVALID_ARG;
  return from_cuda(fp8bw::launch_gemm_fp8(kind, true, G, d_offsets, M_total_pad, N, K, A, sA, B,
                                          sB, D, N, mode, sms, cs, 0));
}

FP8BW_API fp8bw_status fp8bw_grouped_wgrad_f32(int32_t G, const int32_t* d_offsets,
                                     int64_t M_total_pad, int64_t N, int64_t K,
                                     const uint8_t* A, const float* sA, const uint8_t* B,
                                     const float* sB, float* D, int32_t accumulate,
                                     fp8bw_scale_mode mode, fp8bw_stream_t stream) {
  if (mode != FP8BW_SCALE_FP32 && mode != FP8BW_SCALE_POW2) return FP8BW_ERR_INVALID_ARG;
  if (accumulate != 0 && accumulate != 1) return FP8BW_ERR_INVALID_ARG;
  if (!d_offsets || !A || !sA || !B || !sB || !D) return FP8BW_ERR_INVALID_ARG;
  if (G < 1 || M_total_pad < 0 || N < 0 || K < 0) return FP8BW_ERR_INVALID_ARG;
  if (G > FP8BW_MAX_EXPERTS) return FP8BW_ERR_TOO_LARGE;
  if (M_total_pad > kMaxDim || N > kMaxDim || K > kMaxDim) return FP8BW_ERR_TOO_LARGE;
  if (!mult128(M_total_pad) || !mult128(N) || !mult128(K)) return FP8BW_ERR_ALIGNMENT;
  if (!aligned16(A) || !aligned16(B) || !aligned16(D) || !aligned16(sA) || !aligned16(sB) ||
      (reinterpret_cast<uintptr_t>(d_offsets) & 3u))
    return FP8BW_ERR_ALIGNMENT;
  if ((int64_t)G * N * K > (int64_t(1) << 40)) return FP8BW_ERR_TOO_LARGE;
  int sms = 0;
  fp8bw_status st = current(&sms);
  if (st != FP8BW_OK) return st;
  if (N == 0 || K == 0) return FP8BW_OK;
  // GEMM sizes: rows = N (out), cols = K (in), contraction = tokens.
  return from_cuda(fp8bw::launch_gemm_fp8(FP8BW_WGRAD, true, G, d_offsets, N, K, M_total_pad, A, sA,
                                          B, sB, D, K, mode, sms, reinterpret_cast<cudaStream_t>(stream),
                                          accumulate ? 2 : 1));
}

FP8BW_API fp8bw_status fp8bw_gemm_bf16(int64_t M, int64_t N, int64_t K, const void* A, const void* B, void* D,
                             int64_t ldd, fp8bw_stream_t stream) {
  if (!A || !B || !D) return FP8BW_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || K < 0 || ldd < N) return FP8BW_ERR_INVALID_ARG;
  if (M > kMaxDim || N > kMaxDim || K > kMaxDim) return FP8BW_ERR_TOO_LARGE;
  if (!mult128(M) || !mult128(N) || !mult128(K) || (ldd & 7) != 0) return FP8BW_ERR_ALIGNMENT;
  if (!aligned16(A) || !aligned16(B) || !aligned16(D)) return FP8BW_ERR_ALIGNMENT;
  int sms = 0;
  fp8bw_status st = current(&sms);
  if (st != FP8BW_OK) return st;
  if (M == 0 || N == 0) return FP8BW_OK;
  if (K == 0) return from_cuda(cudaMemset2DAsync(D, ldd * 2, 0, N * 2, M, reinterpret_cast<cudaStream_t>(stream)));
  return from_cuda(fp8bw::launch_gemm_bf16(M, N, K, A, B, D, ldd, sms,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

FP8BW_API fp8bw_status fp8bw_quant_tensor_delayed(const void* x, int64_t M, int64_t K, int64_t ldx,
                                        fp8bw_format fmt, fp8bw_scale_mode mode, float* hist,
                                        int32_t H, uint8_t* q, uint8_t* qT, float* scale,
                                        float* amax, float* s_grid, int64_t s_grid_len,
                                        fp8bw_stream_t stream) {
  if (fmt != FP8BW_FMT_E4M3 && fmt != FP8BW_FMT_E5M2) return FP8BW_ERR_INVALID_ARG;
  if (mode != FP8BW_SCALE_FP32 && mode != FP8BW_SCALE_POW2) return FP8BW_ERR_INVALID_ARG;
  if (!hist || !scale || !amax) return FP8BW_ERR_INVALID_ARG;
  if (M != 0 && K != 0 && (!x || !q)) return FP8BW_ERR_INVALID_ARG;  // empty: nothing to touch
  if (H < 1 || H > FP8BW_MAX_HISTORY) return FP8BW_ERR_INVALID_ARG;
  if (s_grid_len < 0 || (s_grid_len > 0 && !s_grid)) return FP8BW_ERR_INVALID_ARG;
  if (M < 0 || K < 0 || ldx < K) return FP8BW_ERR_INVALID_ARG;
  if (M > kMaxDim || K > kMaxDim) return FP8BW_ERR_TOO_LARGE;
  if (!mult128(M) || !mult128(K) || (ldx & 15) != 0) return FP8BW_ERR_ALIGNMENT;
  if (!aligned32(x) || !aligned32(q) || (qT && !aligned32(qT)) || !aligned4(hist) ||
      !aligned4(scale) || !aligned4(amax) || (s_grid && !aligned4(s_grid)))
    return FP8BW_ERR_ALIGNMENT;
  int sms = 0;
  fp8bw_status st = current(&sms);
  if (st != FP8BW_OK) return st;
  return from_cuda(fp8bw::launch_quant_tensor(x, M, K, ldx, mode, fmt, hist, H, q, qT, scale, amax,
                                              s_grid_len > 0 ? s_grid : nullptr, s_grid_len, sms,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

FP8BW_API fp8bw_status fp8bw_gemm_quant(fp8bw_gemm_kind kind, int64_t M, int64_t N, int64_t K,
                                        const uint8_t* A, const float* sA, const uint8_t* B,
                                        const float* sB, fp8bw_scale_mode out_mode, void* D, int64_t ldd,
                                        uint8_t* q_row, float* s_row, uint8_t* q_col, float* s_col,
                                        fp8bw_stream_t stream) {
  if (kind != FP8BW_FPROP && kind != FP8BW_DGRAD && kind != FP8BW_WGRAD) return FP8BW_ERR_INVALID_ARG;
  if (out_mode != FP8BW_SCALE_FP32 && out_mode != FP8BW_SCALE_POW2) return FP8BW_ERR_INVALID_ARG;
  if (!A || !sA || !B || !sB || !q_row || !s_row) return FP8BW_ERR_INVALID_ARG;
  if ((q_col == nullptr) != (s_col == nullptr)) return FP8BW_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || K < 0 || (D && ldd < N)) return FP8BW_ERR_INVALID_ARG;
  if (M > kMaxDim || N > kMaxDim || K > kMaxDim) return FP8BW_ERR_TOO_LARGE;
  if (!mult128(M) || !mult128(N) || !mult128(K) || (D && (ldd & 7) != 0)) return FP8BW_ERR_ALIGNMENT;
  if (!aligned16(A) || !aligned16(B) || !aligned16(sA) || !aligned16(sB) || (D && !aligned16(D)) ||
      !aligned32(q_row) || !aligned16(s_row) || (q_col && !aligned32(q_col)) || (s_col && !aligned16(s_col)))
    return FP8BW_ERR_ALIGNMENT;
  int sms = 0;
  fp8bw_status st = current(&sms);
  if (st != FP8BW_OK) return st;
  if (M == 0 || N == 0) return FP8BW_OK;
  if (K == 0) return FP8BW_ERR_INVALID_ARG;
  return from_cuda(fp8bw::launch_gemm_quant(kind, M, N, K, A, sA, B, sB, out_mode, D, ldd, q_row, s_row,
                                            q_col, s_col, sms, reinterpret_cast<cudaStream_t>(stream)));
}

FP8BW_API fp8bw_status fp8bw_attention_fwd(int64_t T, int32_t Hq, int32_t Hkv, int32_t nseg,
                                           const int32_t* d_seg_off, const int32_t* d_seg_len,
                                           int32_t causal, fp8bw_scale_mode mode,
                                           const uint8_t* q, const float* sq,
                                           const uint8_t* k, const float* sk, const uint8_t* vT,
                                           const float* sv, void* o, fp8bw_stream_t stream) {
  if (!d_seg_off || !d_seg_len || !q || !sq || !k || !sk || !vT || !sv || !o) return FP8BW_ERR_INVALID_ARG;
  if (T < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || nseg < 1 || (causal != 0 && causal != 1))
    return FP8BW_ERR_INVALID_ARG;
  if (mode != FP8BW_SCALE_FP32 && mode != FP8BW_SCALE_POW2) return FP8BW_ERR_INVALID_ARG;
  if (nseg > FP8BW_ATTN_MAX_SEGMENTS || Hq > FP8BW_ATTN_MAX_HEADS) return FP8BW_ERR_TOO_LARGE;
  if (T > kMaxDim || T * Hq * 128 > (int64_t(1) << 40)) return FP8BW_ERR_TOO_LARGE;
  if (!mult128(T)) return FP8BW_ERR_ALIGNMENT;
  if (!aligned16(q) || !aligned16(k) || !aligned16(vT) || !aligned16(sq) || !aligned16(sk) ||
      !aligned16(sv) || !aligned32(o) || !aligned4(d_seg_off) || !aligned4(d_seg_len))
    return FP8BW_ERR_ALIGNMENT;
  int sms = 0;
  fp8bw_status st = current(&sms);
  if (st != FP8BW_OK) return st;
  if (T == 0) return FP8BW_OK;
  return from_cuda(fp8bw::launch_attention_fwd(T, Hq, Hkv, nseg, d_seg_off, d_seg_len, causal, (int)mode, q, sq, k,
                                               sk, vT, sv, o, reinterpret_cast<cudaStream_t>(stream)));
}

FP8BW_API fp8bw_status fp8bw_attention_decode(int32_t B, int32_t Hq, int32_t Hkv, int64_t Lmax,
                                              const int32_t* d_len, const void* q,
                                              const uint8_t* k, const float* sk,
                                              const uint8_t* v, const float* sv, void* o,
                                              fp8bw_stream_t stream) {
  if (!d_len || !q || !k || !sk || !v || !sv || !o) return FP8BW_ERR_INVALID_ARG;
  if (B < 0 || Hkv < 1 || Hq < 1 || Hq % Hkv != 0 || Lmax < 1) return FP8BW_ERR_INVALID_ARG;
  const int32_t G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return FP8BW_ERR_INVALID_ARG;
  if (Hq > FP8BW_ATTN_MAX_HEADS || Lmax > kMaxDim || (int64_t)B * Lmax > kMaxDim ||
      (int64_t)B * Hkv * 8 > (int64_t(1) << 31) - 1)
    return FP8BW_ERR_TOO_LARGE;
  if (!mult128(Lmax)) return FP8BW_ERR_ALIGNMENT;
  if (!aligned16(k) || !aligned16(v) || !aligned16(q) || !aligned16(sk) || !aligned16(sv) ||
      !aligned4(d_len) || (reinterpret_cast<uintptr_t>(o) & 1u) != 0)
    return FP8BW_ERR_ALIGNMENT;
  int sms = 0;
  fp8bw_status st = current(&sms);
  if (st != FP8BW_OK) return st;
  if (B == 0) return FP8BW_OK;
  return from_cuda(fp8bw::launch_attention_decode(B, Hq, Hkv, Lmax, d_len, q, k, sk, v, sv, o,
                                                  reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"

// Per-tensor delayed scaling, the comparison recipe of "FP8
// Trainingsinfrastructuur: Numerieke Precisie van de Volgende Generatie"
// (sections "Transformer Engine: de softwarebasis" and "Scaling-strategieën
// en stabiliteit"): one scale for the whole tensor, taken from the largest
// amax recorded over the previous H calls rather than from the tensor itself.
// The tensor's own amax is reduced while it is quantized and then pushed into
// the history.
//
// A call is three stream-ordered steps: a 4-byte memset of the amax output,
// k_quant_tensor, and k_push_history.
//
// k_quant_tensor (256 threads, 4 CTAs per SM; a grid-stride loop over
// 128x128 tiles of x):
//  * every CTA derives the scale itself from the H history entries, so no
//    launch has to wait for another;
//  * phase 1: a thread reads 32 consecutive bf16 of rows r and r+64 with two
//    32-byte loads each, converts them with the one scale, writes their 32
//    codes as one 32-byte store per row, and parks them in a shared tile;
//  * phase 2 (transposed copy): a thread gathers two columns over 32 rows from
//    the shared tile, 16 bits per row, regroups the bytes with byte permutes
//    and writes each column's 32 codes as one 32-byte store.  With a single
//    scale the column-wise copy is the byte transpose of the codes;
//  * two shared tiles alternate, so each tile needs one barrier;
//  * |x| maxima meet in one atomicMax per warp at the end: non-negative
//    floats order like their bit patterns, so the result is exact and does
//    not depend on the order.  fmaxf drops NaN, so a NaN never becomes the
//    amax.
// k_push_history (one thread): hist[i] = hist[i-1] for i = H-1 .. 1, then
// hist[0] = amax.

#include <cstdint>
#include <cuda_runtime.h>

#include "common.cuh"

namespace fp8bw {
namespace {

constexpr int kTile = 128;
constexpr int kPitch = 144;  // shared-tile row pitch in bytes: 16-byte writes of
                             // 8 rows x 4 segments spread over all banks

__device__ __forceinline__ void ld_nc_v8(const void* p, uint32_t (&r)[8]) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "l"(p));
}

// 16 bf16 (one 32-byte load) -> 16 codes in 4 words; updates the |x| maximum.
template <int MODE, int FMT>
__device__ __forceinline__ void convert16(const uint32_t (&w)[8], float s, float inv,
                                          float& amax, uint32_t* out) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = bf16lo(w[2 * i]), b = bf16hi(w[2 * i]);
    const float c = bf16lo(w[2 * i + 1]), d = bf16hi(w[2 * i + 1]);
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(a), fabsf(b)), fmaxf(fabsf(c), fabsf(d))));
    const uint32_t lo = cvt_fp8x2<FMT>(scale_div<MODE>(a, s, inv), scale_div<MODE>(b, s, inv));
    const uint32_t hi = cvt_fp8x2<FMT>(scale_div<MODE>(c, s, inv), scale_div<MODE>(d, s, inv));
    out[i] = lo | (hi << 16);
  }
}

template <int MODE, int FMT, bool COL>
__global__ void __launch_bounds__(256) k_quant_tensor(
    const uint16_t* __restrict__ x, int64_t M, int64_t K, int64_t ldx,
    const float* __restrict__ hist, int H, uint8_t* __restrict__ q, uint8_t* __restrict__ qT,
    float* __restrict__ scale_out, uint32_t* __restrict__ amax_bits, float* __restrict__ s_grid,
    int64_t s_grid_len) {
  __shared__ __align__(16) uint8_t tile[2][kTile * kPitch];
  const int tid = threadIdx.x;

  float h = 0.0f;
  for (int i = 0; i < H; ++i) h = fmaxf(h, __ldg(hist + i));
  const float s = block_scale<MODE, FMT>(h);
  const float inv = scale_inv<MODE>(s);
  if (blockIdx.x == 0 && tid == 0) *scale_out = s;
  for (int64_t i = (int64_t)blockIdx.x * 256 + tid; i < s_grid_len; i += (int64_t)gridDim.x * 256)
    s_grid[i] = s;

  const int64_t nKt = K / kTile, tiles = (M / kTile) * nKt;
  const int r = tid >> 2, seg = tid & 3;                           // phase 1
  const int warp = tid >> 5, lane = tid & 31;
  const int cp = 32 * (warp & 1) + lane, g = warp >> 1;            // phase 2
  float amax = 0.0f;
  int buf = 0;
  for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, buf ^= 1) {
    const int64_t m0 = (t / nKt) * kTile, k0 = (t % nKt) * kTile;
    uint32_t v[4][8];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const uint16_t* src = x + (m0 + r + 64 * hh) * ldx + k0 + 32 * seg;
      ld_nc_v8(src, v[2 * hh]);
      ld_nc_v8(src + 16, v[2 * hh + 1]);
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      uint32_t c[8];
      convert16<MODE, FMT>(v[2 * hh], s, inv, amax, c);
      convert16<MODE, FMT>(v[2 * hh + 1], s, inv, amax, c + 4);
      const int row = r + 64 * hh;
      st_global_v8(q + (m0 + row) * K + k0 + 32 * seg, make_uint4(c[0], c[1], c[2], c[3]),
                   make_uint4(c[4], c[5], c[6], c[7]));
      if (COL) {
        uint4* d = reinterpret_cast<uint4*>(tile[buf] + row * kPitch + 32 * seg);
        d[0] = make_uint4(c[0], c[1], c[2], c[3]);
        d[1] = make_uint4(c[4], c[5], c[6], c[7]);
      }
    }
    if (COL) {
      __syncthreads();
      const uint8_t* base = tile[buf] + (32 * g) * kPitch + 2 * cp;
      uint32_t c0[8], c1[8];  // columns 2cp and 2cp+1, rows 32g .. 32g+31
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t a = *reinterpret_cast<const uint16_t*>(base + (4 * i + 0) * kPitch);
        const uint32_t b = *reinterpret_cast<const uint16_t*>(base + (4 * i + 1) * kPitch);
        const uint32_t cc = *reinterpret_cast<const uint16_t*>(base + (4 * i + 2) * kPitch);
        const uint32_t d = *reinterpret_cast<const uint16_t*>(base + (4 * i + 3) * kPitch);
        const uint32_t ab = __byte_perm(a, b, 0x5140);   // a0 b0 a1 b1
        const uint32_t cd = __byte_perm(cc, d, 0x5140);  // c0 d0 c1 d1
        c0[i] = __byte_perm(ab, cd, 0x5410);             // a0 b0 c0 d0
        c1[i] = __byte_perm(ab, cd, 0x7632);             // a1 b1 c1 d1
      }
      uint8_t* dst = qT + (k0 + 2 * cp) * M + m0 + 32 * g;
      st_global_v8(dst, make_uint4(c0[0], c0[1], c0[2], c0[3]), make_uint4(c0[4], c0[5], c0[6], c0[7]));
      st_global_v8(dst + M, make_uint4(c1[0], c1[1], c1[2], c1[3]),
                   make_uint4(c1[4], c1[5], c1[6], c1[7]));
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0 && amax > 0.0f) atomicMax(amax_bits, __float_as_uint(amax));
}

__global__ void k_push_history(float* __restrict__ hist, int H, const uint32_t* __restrict__ amax_bits) {
  if (threadIdx.x != 0) return;
  for (int i = H - 1; i > 0; --i) hist[i] = hist[i - 1];
  hist[0] = __uint_as_float(*amax_bits);
}

template <int MODE, int FMT, bool COL>
cudaError_t launch_t(const void* x, int64_t M, int64_t K, int64_t ldx, float* hist, int H,
                     uint8_t* q, uint8_t* qT, float* scale, float* amax, float* s_grid,
                     int64_t s_grid_len, int num_sms, cudaStream_t st) {
  auto kern = k_quant_tensor<MODE, FMT, COL>;
  int occ = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, 256, 0);
  if (e != cudaSuccess) return e;
  // Four resident CTAs per SM stream best on B200 (measured over 1-6 on the
  // [8192, 28672] tensor: five or six CTAs per SM were 15-30 % slower, and
  // prefetching the next tile into registers did not help either).
  if (occ > 4) occ = 4;
  if (occ < 1) occ = 1;
  const int64_t tiles = (M / kTile) * (K / kTile);
  int64_t grid = (int64_t)num_sms * occ;
  if (tiles < grid) grid = tiles;
  if (grid < 1) grid = 1;
  uint32_t* abits = reinterpret_cast<uint32_t*>(amax);
  kern<<<(unsigned)grid, 256, 0, st>>>(static_cast<const uint16_t*>(x), M, K, ldx, hist, H, q,
                                       qT, scale, abits, s_grid, s_grid_len);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k_push_history<<<1, 32, 0, st>>>(hist, H, abits);
  return cudaGetLastError();
}

template <int MODE, int FMT>
cudaError_t launch_col(bool col, const void* x, int64_t M, int64_t K, int64_t ldx, float* hist,
                       int H, uint8_t* q, uint8_t* qT, float* scale, float* amax, float* s_grid,
                       int64_t s_grid_len, int num_sms, cudaStream_t st) {
  return col ? launch_t<MODE, FMT, true>(x, M, K, ldx, hist, H, q, qT, scale, amax, s_grid,
                                         s_grid_len, num_sms, st)
             : launch_t<MODE, FMT, false>(x, M, K, ldx, hist, H, q, qT, scale, amax, s_grid,
                                          s_grid_len, num_sms, st);
}

}  // namespace

cudaError_t launch_quant_tensor(const void* x, int64_t M, int64_t K, int64_t ldx, int mode,
                                int fmt, float* hist, int H, uint8_t* q, uint8_t* qT,
                                float* scale, float* amax, float* s_grid, int64_t s_grid_len,
                                int num_sms, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float), st);
  if (e != cudaSuccess) return e;
  const bool col = qT != nullptr;
  if (mode == FP8BW_SCALE_POW2)
    return fmt == FP8BW_FMT_E5M2
               ? launch_col<FP8BW_SCALE_POW2, FP8BW_FMT_E5M2>(col, x, M, K, ldx, hist, H, q, qT,
                                                              scale, amax, s_grid, s_grid_len,
                                                              num_sms, st)
               : launch_col<FP8BW_SCALE_POW2, FP8BW_FMT_E4M3>(col, x, M, K, ldx, hist, H, q, qT,
                                                              scale, amax, s_grid, s_grid_len,
                                                              num_sms, st);
  return fmt == FP8BW_FMT_E5M2
             ? launch_col<FP8BW_SCALE_FP32, FP8BW_FMT_E5M2>(col, x, M, K, ldx, hist, H, q, qT,
                                                            scale, amax, s_grid, s_grid_len,
                                                            num_sms, st)
             : launch_col<FP8BW_SCALE_FP32, FP8BW_FMT_E4M3>(col, x, M, K, ldx, hist, H, q, qT,
                                                            scale, amax, s_grid, s_grid_len,
                                                            num_sms, st);
}

}  // namespace fp8bw

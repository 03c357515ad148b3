// Blockwise E4M3 quantizers (HBM-bound): activations with 1x128 blocks plus
// the fused column-wise copy, weights with 128x128 blocks plus the byte
// transpose, and the batched per-step requantization of many weights.
//
// Method: "NVIDIA NeMo RL erreicht 48% ..." section "Der technische
// Durchbruch" (E4M3, 128x128 weight blocks, 1x128 activation blocks) and
// "Leistungsgewinne in der Praxis" (scales recalibrated after every step).
//
// Design: one CTA of 256 threads per 128x128 bf16 tile (32 KB).  Each thread
// loads eight 16-byte vectors (coalesced: a half-warp covers one 256-byte
// row segment), keeps them in registers for the row-wise pass and writes
// them to shared memory for the column-wise pass.  Row-wise: a 16-lane
// shuffle reduction gives each 1x128 block's amax; codes leave as 8-byte
// stores (a half-warp writes one 128-byte row).  Column-wise: each thread
// owns two columns x 32 rows of the shared tile (conflict-free 32-bit
// reads), four partial maxima meet in shared memory, and the 2x32 codes
// leave as four 16-byte stores into the transposed output.

#include "common.cuh"

namespace fp8bw {
namespace {

constexpr int QT = 256;  // threads per tile CTA

struct TileSmem {
  uint32_t tile[128][64];  // bf16 pairs, row-major (256 B per row)
  float colmax[4][128];
  float red[8];
};

// Quantizes the 8 bf16 values of one 16-byte vector with scale s.
template <int MODE>
__device__ __forceinline__ uint2 quant8(uint4 v, float s, float inv) {
  uint2 o;
  o.x = cvt_e4m3x2(scale_div<MODE>(bf16lo(v.x), s, inv), scale_div<MODE>(bf16hi(v.x), s, inv)) |
        (cvt_e4m3x2(scale_div<MODE>(bf16lo(v.y), s, inv), scale_div<MODE>(bf16hi(v.y), s, inv))
         << 16);
  o.y = cvt_e4m3x2(scale_div<MODE>(bf16lo(v.z), s, inv), scale_div<MODE>(bf16hi(v.z), s, inv)) |
        (cvt_e4m3x2(scale_div<MODE>(bf16lo(v.w), s, inv), scale_div<MODE>(bf16hi(v.w), s, inv))
         << 16);
  return o;
}

__device__ __forceinline__ float amax8(uint4 v) {
  float a = fmaxf(fabsf(bf16lo(v.x)), fabsf(bf16hi(v.x)));
  a = fmaxf(a, fmaxf(fabsf(bf16lo(v.y)), fabsf(bf16hi(v.y))));
  a = fmaxf(a, fmaxf(fabsf(bf16lo(v.z)), fabsf(bf16hi(v.z))));
  a = fmaxf(a, fmaxf(fabsf(bf16lo(v.w)), fabsf(bf16hi(v.w))));
  return a;
}

// Column pass over a tile already in shared memory: thread (wc, rg) handles
// columns 2wc, 2wc+1 and rows 32rg .. 32rg+31.  If `cs0`/`cs1` are given
// (the weight case) they are the scales; otherwise the column amaxes are
// reduced here and the scales written to s_col[0..127].
template <int MODE, bool BLOCK_SCALE>
__device__ __forceinline__ void column_pass(TileSmem& sm, float blk_s, uint8_t* qc, int64_t ldqc,
                                            float* s_col) {
  const int tid = threadIdx.x;
  const int wc = tid & 63, rg = tid >> 6;
  float s0, s1;
  if (BLOCK_SCALE) {
    s0 = s1 = blk_s;
  } else {
    float a0 = 0.f, a1 = 0.f;
#pragma unroll 8
    for (int i = 0; i < 32; ++i) {
      const uint32_t w = sm.tile[rg * 32 + i][wc];
      a0 = fmaxf(a0, fabsf(bf16lo(w)));
      a1 = fmaxf(a1, fabsf(bf16hi(w)));
    }
    sm.colmax[rg][2 * wc] = a0;
    sm.colmax[rg][2 * wc + 1] = a1;
    __syncthreads();
    a0 = fmaxf(fmaxf(sm.colmax[0][2 * wc], sm.colmax[1][2 * wc]),
               fmaxf(sm.colmax[2][2 * wc], sm.colmax[3][2 * wc]));
    a1 = fmaxf(fmaxf(sm.colmax[0][2 * wc + 1], sm.colmax[1][2 * wc + 1]),
               fmaxf(sm.colmax[2][2 * wc + 1], sm.colmax[3][2 * wc + 1]));
    s0 = block_scale<MODE>(a0);
    s1 = block_scale<MODE>(a1);
    if (rg == 0) *reinterpret_cast<float2*>(s_col + 2 * wc) = make_float2(s0, s1);
  }
  const float i0 = scale_inv<MODE>(s0), i1 = scale_inv<MODE>(s1);
  uint32_t c0[8], c1[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t w0 = sm.tile[rg * 32 + 4 * i + 0][wc];
    const uint32_t w1 = sm.tile[rg * 32 + 4 * i + 1][wc];
    const uint32_t w2 = sm.tile[rg * 32 + 4 * i + 2][wc];
    const uint32_t w3 = sm.tile[rg * 32 + 4 * i + 3][wc];
    c0[i] = cvt_e4m3x2(scale_div<MODE>(bf16lo(w0), s0, i0), scale_div<MODE>(bf16lo(w1), s0, i0)) |
            (cvt_e4m3x2(scale_div<MODE>(bf16lo(w2), s0, i0), scale_div<MODE>(bf16lo(w3), s0, i0))
             << 16);
    c1[i] = cvt_e4m3x2(scale_div<MODE>(bf16hi(w0), s1, i1), scale_div<MODE>(bf16hi(w1), s1, i1)) |
            (cvt_e4m3x2(scale_div<MODE>(bf16hi(w2), s1, i1), scale_div<MODE>(bf16hi(w3), s1, i1))
             << 16);
  }
  uint8_t* d0 = qc + (int64_t)(2 * wc) * ldqc + rg * 32;
  uint8_t* d1 = d0 + ldqc;
  reinterpret_cast<uint4*>(d0)[0] = make_uint4(c0[0], c0[1], c0[2], c0[3]);
  reinterpret_cast<uint4*>(d0)[1] = make_uint4(c0[4], c0[5], c0[6], c0[7]);
  reinterpret_cast<uint4*>(d1)[0] = make_uint4(c1[0], c1[1], c1[2], c1[3]);
  reinterpret_cast<uint4*>(d1)[1] = make_uint4(c1[4], c1[5], c1[6], c1[7]);
}

// ---------------------------------------------------------- activations ---
template <int MODE, bool COL>
__global__ void __launch_bounds__(QT) k_quant_act(const uint16_t* __restrict__ x, int64_t M,
                                                  int64_t K, int64_t ldx, uint8_t* __restrict__ q_row,
                                                  float* __restrict__ s_row,
                                                  uint8_t* __restrict__ q_col,
                                                  float* __restrict__ s_col) {
  __shared__ __align__(16) TileSmem sm;
  const int64_t k0 = (int64_t)blockIdx.x * 128, m0 = (int64_t)blockIdx.y * 128;
  const int tid = threadIdx.x;
  const int r16 = tid >> 4, vec = tid & 15;
  uint4 v[8];
#pragma unroll
  for (int p = 0; p < 8; ++p) v[p] = ld_nc_v4(x + (m0 + p * 16 + r16) * ldx + k0 + vec * 8);
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const int row = p * 16 + r16;
    float a = amax8(v[p]);
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 8));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 4));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
    const float s = block_scale<MODE>(a);
    const float inv = scale_inv<MODE>(s);
    *reinterpret_cast<uint2*>(q_row + (m0 + row) * K + k0 + vec * 8) = quant8<MODE>(v[p], s, inv);
    if (vec == 0) s_row[(k0 / 128) * M + m0 + row] = s;
    if (COL) *reinterpret_cast<uint4*>(&sm.tile[row][vec * 4]) = v[p];
  }
  if (!COL) return;
  __syncthreads();
  column_pass<MODE, false>(sm, 0.f, q_col + k0 * M + m0, M, s_col + (m0 / 128) * K + k0);
}

// --------------------------------------------------------------- weights --
// One 128x128 block: block amax -> one scale -> row-major codes and, if qT is
// given, the transposed codes (the same arithmetic on the same inputs, so the
// exact byte transpose).
template <int MODE>
__device__ __forceinline__ void weight_block(TileSmem& sm, const uint16_t* __restrict__ w,
                                             int64_t ldw, int64_t K, int64_t N, int64_t n0,
                                             int64_t k0, uint8_t* __restrict__ q,
                                             float* __restrict__ s, uint8_t* __restrict__ qT) {
  const int tid = threadIdx.x;
  const int r16 = tid >> 4, vec = tid & 15;
  uint4 v[8];
#pragma unroll
  for (int p = 0; p < 8; ++p) v[p] = ld_nc_v4(w + (n0 + p * 16 + r16) * ldw + k0 + vec * 8);
  float a = 0.f;
#pragma unroll
  for (int p = 0; p < 8; ++p) a = fmaxf(a, amax8(v[p]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((tid & 31) == 0) sm.red[tid >> 5] = a;
  if (qT) {
#pragma unroll
    for (int p = 0; p < 8; ++p)
      *reinterpret_cast<uint4*>(&sm.tile[p * 16 + r16][vec * 4]) = v[p];
  }
  __syncthreads();
  a = sm.red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) a = fmaxf(a, sm.red[i]);
  const float sc = block_scale<MODE>(a);
  const float inv = scale_inv<MODE>(sc);
  if (tid == 0) s[(n0 / 128) * (K / 128) + k0 / 128] = sc;
#pragma unroll
  for (int p = 0; p < 8; ++p)
    *reinterpret_cast<uint2*>(q + (n0 + p * 16 + r16) * K + k0 + vec * 8) =
        quant8<MODE>(v[p], sc, inv);
  if (qT) column_pass<MODE, true>(sm, sc, qT + k0 * N + n0, N, nullptr);
}

template <int MODE>
__global__ void __launch_bounds__(QT) k_quant_weight(const uint16_t* __restrict__ w, int64_t N,
                                                     int64_t K, int64_t ldw, uint8_t* __restrict__ q,
                                                     float* __restrict__ s,
                                                     uint8_t* __restrict__ qT) {
  __shared__ __align__(16) TileSmem sm;
  weight_block<MODE>(sm, w, ldw, K, N, (int64_t)blockIdx.y * 128, (int64_t)blockIdx.x * 128, q, s,
                     qT);
}

// ------------------------------------------------------ batched requant ---
constexpr int kMaxPerLaunch = FP8BW_REQUANT_MAX_PER_LAUNCH;

struct RequantTable {
  int n;
  int64_t first_block[kMaxPerLaunch + 1];  // prefix sums of 128x128 block counts
  const uint16_t* w[kMaxPerLaunch];
  uint8_t* q[kMaxPerLaunch];
  float* s[kMaxPerLaunch];
  uint8_t* qT[kMaxPerLaunch];
  int32_t N[kMaxPerLaunch], K[kMaxPerLaunch];
  int64_t ldw[kMaxPerLaunch];
};

template <int MODE>
__global__ void __launch_bounds__(QT) k_requant(const __grid_constant__ RequantTable t) {
  __shared__ __align__(16) TileSmem sm;
  const int64_t b = blockIdx.x;
  int lo = 0, hi = t.n - 1;  // last i with first_block[i] <= b
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (t.first_block[mid] <= b) lo = mid; else hi = mid - 1;
  }
  const int i = lo;
  const int64_t local = b - t.first_block[i];
  const int64_t nK = t.K[i] / 128;
  const int64_t nb = local / nK, kb = local - nb * nK;
  weight_block<MODE>(sm, t.w[i], t.ldw[i], t.K[i], t.N[i], nb * 128, kb * 128, t.q[i], t.s[i],
                     t.qT[i]);
}

}  // namespace

// ------------------------------------------------------------ launchers ---
cudaError_t launch_quant_act(const void* x, int64_t M, int64_t K, int64_t ldx, int mode,
                             uint8_t* q_row, float* s_row, uint8_t* q_col, float* s_col,
                             cudaStream_t st) {
  const dim3 grid((unsigned)(K / 128), (unsigned)(M / 128));
  const auto* xp = static_cast<const uint16_t*>(x);
  const bool col = q_col != nullptr;
  if (mode == FP8BW_SCALE_FP32) {
    if (col) k_quant_act<0, true><<<grid, QT, 0, st>>>(xp, M, K, ldx, q_row, s_row, q_col, s_col);
    else k_quant_act<0, false><<<grid, QT, 0, st>>>(xp, M, K, ldx, q_row, s_row, q_col, s_col);
  } else {
    if (col) k_quant_act<1, true><<<grid, QT, 0, st>>>(xp, M, K, ldx, q_row, s_row, q_col, s_col);
    else k_quant_act<1, false><<<grid, QT, 0, st>>>(xp, M, K, ldx, q_row, s_row, q_col, s_col);
  }
  return cudaGetLastError();
}

cudaError_t launch_quant_weight(const void* w, int64_t N, int64_t K, int64_t ldw, int mode,
                                uint8_t* q, float* s, uint8_t* qT, cudaStream_t st) {
  const dim3 grid((unsigned)(K / 128), (unsigned)(N / 128));
  const auto* wp = static_cast<const uint16_t*>(w);
  if (mode == FP8BW_SCALE_FP32) k_quant_weight<0><<<grid, QT, 0, st>>>(wp, N, K, ldw, q, s, qT);
  else k_quant_weight<1><<<grid, QT, 0, st>>>(wp, N, K, ldw, q, s, qT);
  return cudaGetLastError();
}

cudaError_t launch_requant(const fp8bw_weight_desc* d, int32_t n, int mode, cudaStream_t st) {
  RequantTable t;
  for (int32_t base = 0; base < n; base += kMaxPerLaunch) {
    const int cnt = (n - base) < kMaxPerLaunch ? (n - base) : kMaxPerLaunch;
    t.n = cnt;
    t.first_block[0] = 0;
    for (int i = 0; i < cnt; ++i) {
      const fp8bw_weight_desc& e = d[base + i];
      t.w[i] = static_cast<const uint16_t*>(e.w);
      t.q[i] = e.q;
      t.s[i] = e.s;
      t.qT[i] = e.qT;
      t.N[i] = (int32_t)e.N;
      t.K[i] = (int32_t)e.K;
      t.ldw[i] = e.ldw;
      t.first_block[i + 1] = t.first_block[i] + (e.N / 128) * (e.K / 128);
    }
    const int64_t blocks = t.first_block[cnt];
    if (blocks == 0) continue;
    if (mode == FP8BW_SCALE_FP32) k_requant<0><<<(unsigned)blocks, QT, 0, st>>>(t);
    else k_requant<1><<<(unsigned)blocks, QT, 0, st>>>(t);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace fp8bw

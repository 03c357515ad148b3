// Blockwise E4M3 quantizers (HBM-bound): activations with 1x128 blocks plus
// the fused column-wise copy, weights with 128x128 blocks plus the byte
// transpose, and the batched per-step requantization of many weights.
//
// Method: "NVIDIA NeMo RL erreicht 48% ..." section "Der technische
// Durchbruch" (E4M3, 128x128 weight blocks, 1x128 activation blocks) and
// "Leistungsgewinne in der Praxis" (scales recalibrated after every step).
//
// Design: activations go through persistent CTAs of 256 threads that walk
// 128x128 bf16 tiles, TMA-loaded (two 64-column boxes, 128-byte swizzle) two
// tiles ahead into a double buffer; weights take one CTA per 128x128 block.
//  * amax: bf16 magnitudes compared as packed unsigned 16-bit integers
//    (sign bit cleared; the bit order of non-negative bf16 values is their
//    numeric order), two elements per instruction.
//  * x / s: the block's divisor is fixed, so its IEEE reciprocal y = RN(1/s)
//    is taken once per block and every element uses one Markstein correction
//    step (P. Markstein, "Computation of elementary functions on the IBM
//    RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990), in the
//    sign-symmetric form
//        q0 = RN(x*y);  r = fma(q0, s, -x) (exact);  q = fma(r, -y, q0)
//    on packed f32x2 lanes.  An exhaustive check over every bf16 block amax
//    >= 2^-80 and every bf16 |x| <= amax shows q equals RN(x/s) wherever
//    |x/s| >= 2^-12 and that the signs always agree, signed zeros included
//    (tests/test_division_scheme.py).  Blocks with a smaller amax use IEEE
//    division.  In power-of-2 mode 1/s is exact and x*(1/s) is the
//    correctly rounded x/s.
//  * activation codes leave as 32-byte stores (whole sectors) straight from
//    registers: a thread holds 64 consecutive row codes of one row, or 32
//    consecutive tokens of two columns for the column-wise copy.

#include "blockquant.cuh"
#include "common.cuh"
#include "tmap.cuh"

namespace fp8bw {

// Device error word of the quantizers (a bounded wait that ran out), read
// and cleared by fp8bw_last_device_error() through quant_read_clear_error().
__device__ uint32_t g_quant_error;

namespace {

constexpr int QT = 256;  // threads per tile CTA

struct WeightSmem {
  uint32_t codes[128][32];   // row-major codes, swizzled words
  uint32_t red[8];
};
// ---------------------------------------------------------- activations ---
// A 128x128 bf16 tile sits in shared memory as two boxes of 64 columns
// (128 rows x 128 bytes each) with the TMA's 128-byte swizzle: 16-byte chunk
// j of row r is stored at chunk j ^ (r & 7).
struct ActSmem {
  uint8_t buf[2][2][128 * 128];  // [buffer][box][row * 128 + byte], 1024-aligned
  uint32_t colmax[2][4][64];     // partial column maxima, by tile parity
  uint64_t full[2];
};


__device__ __forceinline__ void issue_tile(ActSmem& sm, const CUtensorMap* tm, int t, int nK, int b) {
  const uint32_t bar = smem_u32(&sm.full[b]);
  const int k0 = (t % nK) * 128, m0 = (t / nK) * 128;
  mbar_arrive_expect_tx(bar, 128 * 256);
  tma_load_2d(smem_u32(&sm.buf[b][0][0]), tm, bar, k0, m0);
  tma_load_2d(smem_u32(&sm.buf[b][1][0]), tm, bar, k0 + 64, m0);
}

// Persistent activation quantizer: CTA c walks tiles t = c + i*gridDim.x
// (column tile fastest), with tiles i+1 and i+2 in flight while tile i is
// processed.  Per tile and thread:
//   row pass     thread (row rr, half hh) reads its 64 columns (8 conflict-
//                free 16-byte loads), takes the row amax with its partner
//                lane (lane ^ 8 holds the other half), and writes 64 codes
//                and, for hh = 0, the row scale;
//   column pass  thread (column pair wc, row group rg) reads 32 rows of its
//                two columns, posts the partial maxima; after the tile's one
//                barrier it combines the four row groups, quantizes and
//                writes 2 x 32 codes and, for rg = 0, the column scales.
template <int MODE, bool COL, int FMT>
__global__ void __launch_bounds__(QT, 3) k_quant_act(const __grid_constant__ CUtensorMap tmX,
                                                     int64_t M, int64_t K,
                                                     uint8_t* __restrict__ q_row,
                                                     float* __restrict__ s_row,
                                                     uint8_t* __restrict__ q_col,
                                                     float* __restrict__ s_col) {
  extern __shared__ uint8_t smem_raw[];
  ActSmem& sm = *reinterpret_cast<ActSmem*>(smem_align1024(smem_raw));
  const int tid = threadIdx.x;
  const int rr = (tid & 7) + 8 * (tid >> 4), hh = (tid >> 3) & 1;  // row pass
  const int wc = tid & 63, rg = tid >> 6;                            // column pass
  const int cbox = wc >> 5, cchunk = (wc & 31) >> 2, cword = wc & 3;
  const int nK = (int)(K / 128);
  const int tiles = nK * (int)(M / 128);
  if (tid == 0) {
    mbar_init(smem_u32(&sm.full[0]), 1);
    mbar_init(smem_u32(&sm.full[1]), 1);
    fence_barrier_init();
    prefetch_tmap(&tmX);
  }
  __syncthreads();
  if (tid == 0) {
    if ((int)blockIdx.x < tiles) issue_tile(sm, &tmX, blockIdx.x, nK, 0);
    if ((int)(blockIdx.x + gridDim.x) < tiles) issue_tile(sm, &tmX, blockIdx.x + gridDim.x, nK, 1);
  }
  int i = 0;
  for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
    const int cur = i & 1;
    const int64_t k0 = (int64_t)(t % nK) * 128, m0 = (int64_t)(t / nK) * 128;
    if (!mbar_wait(smem_u32(&sm.full[cur]), (i >> 1) & 1)) {
      // A tile load that never lands (not expected): latch the timeout and
      // give the other buffer's load, if one was issued, a bounded chance to
      // land before this CTA's shared memory goes away.
      if (tid == 0) {
        atomicOr(&g_quant_error, DEV_ERR_TIMEOUT);
        if (t + (int)gridDim.x < tiles) (void)mbar_wait(smem_u32(&sm.full[cur ^ 1]), ((i + 1) >> 1) & 1);
      }
      return;
    }
    const uint8_t* tb = &sm.buf[cur][0][0];

    // ---- row pass
    {
      uint4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = *reinterpret_cast<const uint4*>(tb + act_off(hh, rr, j));
      uint32_t m0w = magmax2(v[0].x, v[0].y), m1w = magmax2(v[0].z, v[0].w);
#pragma unroll
      for (int j = 1; j < 8; ++j) {
        m0w = magmax2(m0w, magmax2(v[j].x, v[j].y));
        m1w = magmax2(m1w, magmax2(v[j].z, v[j].w));
      }
      uint32_t m = magmax2(m0w, m1w) & kAbsMask;
      m = umax2(m, __shfl_xor_sync(0xffffffffu, m, 8));
      const Divisor d = make_divisor<MODE, FMT>(halves_max(m));
      if (hh == 0) s_row[(k0 / 128) * M + m0 + rr] = d.s;
      uint8_t* qr = q_row + (m0 + rr) * K + k0 + hh * 64;
#pragma unroll
      for (int j = 0; j < 8; j += 4) {
        const uint2 c0 = quant8<MODE, FMT>(v[j], d), c1 = quant8<MODE, FMT>(v[j + 1], d);
        const uint2 c2 = quant8<MODE, FMT>(v[j + 2], d), c3 = quant8<MODE, FMT>(v[j + 3], d);
        st_global_v8(qr + 8 * j, make_uint4(c0.x, c0.y, c1.x, c1.y), make_uint4(c2.x, c2.y, c3.x, c3.y));
      }
    }

    // ---- column pass, part 1: the words and the partial maxima
    ColWords cw;
    if (COL) {
#pragma unroll
      for (int r = 0; r < 32; ++r)
        cw.w[r] = *reinterpret_cast<const uint32_t*>(tb + act_off(cbox, rg * 32 + r, cchunk) + 4 * cword);
      uint32_t mw[4] = {cw.w[0], cw.w[1], cw.w[2], cw.w[3]};
#pragma unroll
      for (int r = 4; r < 32; ++r) mw[r & 3] = magmax2(mw[r & 3], cw.w[r]);
      sm.colmax[cur][rg][wc] = magmax2(magmax2(mw[0], mw[1]), magmax2(mw[2], mw[3])) & kAbsMask;
    }
    // Partial maxima complete; every thread is done reading this buffer, so
    // it may take the tile after next.
    __syncthreads();
    if (tid == 0 && t + 2 * (int)gridDim.x < tiles) issue_tile(sm, &tmX, t + 2 * gridDim.x, nK, cur);

    // ---- column pass, part 2
    if (COL) {
      const uint32_t m = umax2(umax2(sm.colmax[cur][0][wc], sm.colmax[cur][1][wc]),
                               umax2(sm.colmax[cur][2][wc], sm.colmax[cur][3][wc]));
      const Divisor d0 = make_divisor<MODE, FMT>(__uint_as_float((m & 0xFFFFu) << 16));
      const Divisor d1 = make_divisor<MODE, FMT>(__uint_as_float(m & 0xFFFF0000u));
      if (rg == 0)
        *reinterpret_cast<float2*>(s_col + (m0 / 128) * K + k0 + 2 * wc) = make_float2(d0.s, d1.s);
      uint32_t c0[8], c1[8];
      if (MODE == FP8BW_SCALE_FP32 && __any_sync(0xffffffffu, d0.exact || d1.exact)) {
        const ColCodes c = column_codes_exact<FMT>(cw, d0, d1);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          c0[j] = c.c0[j];
          c1[j] = c.c1[j];
        }
      } else {
        const float2 s2 = make_float2(d0.s, d1.s), y2 = make_float2(d0.y, d1.y);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float2 q[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint32_t w = cw.w[4 * j + u];
            q[u] = div2<MODE>(make_float2(bf16lo(w), bf16hi(w)), s2, y2);
          }
          c0[j] = cvt_fp8x2<FMT>(q[0].x, q[1].x) | (cvt_fp8x2<FMT>(q[2].x, q[3].x) << 16);
          c1[j] = cvt_fp8x2<FMT>(q[0].y, q[1].y) | (cvt_fp8x2<FMT>(q[2].y, q[3].y) << 16);
        }
      }
      uint8_t* qc = q_col + (k0 + 2 * wc) * M + m0 + rg * 32;
      st_global_v8(qc, make_uint4(c0[0], c0[1], c0[2], c0[3]), make_uint4(c0[4], c0[5], c0[6], c0[7]));
      st_global_v8(qc + M, make_uint4(c1[0], c1[1], c1[2], c1[3]), make_uint4(c1[4], c1[5], c1[6], c1[7]));
    }
  }
}

// --------------------------------------------------------------- weights --
// One 128x128 block: block amax -> one scale -> row-major codes and, if qT is
// given, their exact byte transpose (through the swizzled shared tile).
template <int MODE>
__device__ __forceinline__ void weight_block(WeightSmem& sm, const uint16_t* __restrict__ w,
                                             int64_t ldw, int64_t K, int64_t N, int64_t n0,
                                             int64_t k0, uint8_t* __restrict__ q,
                                             float* __restrict__ s, uint8_t* __restrict__ qT) {
  const int tid = threadIdx.x;
  const int r16 = tid >> 4, vec = tid & 15;
  uint4 v[8];
#pragma unroll
  for (int p = 0; p < 8; ++p) v[p] = ld_nc_v4(w + (n0 + p * 16 + r16) * ldw + k0 + vec * 8);
  uint32_t m = 0;
#pragma unroll
  for (int p = 0; p < 8; ++p) m = umax2(m, absmax8(v[p]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = umax2(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((tid & 31) == 0) sm.red[tid >> 5] = m;
  __syncthreads();
  m = sm.red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) m = umax2(m, sm.red[i]);
  const Divisor d = make_divisor<MODE>(halves_max(m));
  if (tid == 0) s[(n0 / 128) * (K / 128) + k0 / 128] = d.s;
  // Row-major codes go to q and, swizzled, to the shared code tile: row n,
  // 32 words; logical word w of row n lives at w ^ (((n >> 4) & 7) << 2).
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const uint2 c = quant8<MODE>(v[p], d);
    const int n = p * 16 + r16;
    *reinterpret_cast<uint2*>(q + (n0 + n) * K + k0 + vec * 8) = c;
    if (qT) *reinterpret_cast<uint2*>(&sm.codes[n][(2 * vec) ^ (p << 2)]) = c;
  }
  if (!qT) return;
  __syncthreads();
  // Byte transpose: lane (g = lane & 7, kq = 4 * warp + lane / 8) reads the
  // words of column group kq (k = 4kq .. 4kq+3) for rows n = 16g .. 16g+15
  // (conflict-free thanks to the swizzle), transposes 4x4 byte blocks with
  // byte permutes and writes 16 bytes of n to each of the 4 rows k of qT
  // (eight lanes fill one 128-byte row).
  const int lane = tid & 31, g = lane & 7, kq = 4 * (tid >> 5) + (lane >> 3);
  uint32_t wv[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) wv[i] = sm.codes[16 * g + i][kq ^ (g << 2)];
  uint32_t col[4][4];  // [k offset][group of 4 rows]
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const uint32_t t0 = __byte_perm(wv[4 * b + 0], wv[4 * b + 1], 0x5140);
    const uint32_t t1 = __byte_perm(wv[4 * b + 0], wv[4 * b + 1], 0x7362);
    const uint32_t t2 = __byte_perm(wv[4 * b + 2], wv[4 * b + 3], 0x5140);
    const uint32_t t3 = __byte_perm(wv[4 * b + 2], wv[4 * b + 3], 0x7362);
    col[0][b] = __byte_perm(t0, t2, 0x5410);
    col[1][b] = __byte_perm(t0, t2, 0x7632);
    col[2][b] = __byte_perm(t1, t3, 0x5410);
    col[3][b] = __byte_perm(t1, t3, 0x7632);
  }
#pragma unroll
  for (int c = 0; c < 4; ++c)
    *reinterpret_cast<uint4*>(qT + (k0 + 4 * kq + c) * N + n0 + 16 * g) =
        make_uint4(col[c][0], col[c][1], col[c][2], col[c][3]);
}

template <int MODE>
__global__ void __launch_bounds__(QT) k_quant_weight(const uint16_t* __restrict__ w, int64_t N,
                                                     int64_t K, int64_t ldw, uint8_t* __restrict__ q,
                                                     float* __restrict__ s,
                                                     uint8_t* __restrict__ qT) {
  __shared__ __align__(16) WeightSmem sm;
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
  __shared__ __align__(16) WeightSmem sm;
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
                             int num_sms, cudaStream_t st, int fmt) {
  CUtensorMap tm;
  if (!make_map(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, (uint64_t)K, (uint64_t)M,
                (uint64_t)ldx, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const int64_t tiles = (K / 128) * (M / 128);
  const int per_sm = 3;
  const unsigned grid = (unsigned)(tiles < (int64_t)num_sms * per_sm ? tiles : (int64_t)num_sms * per_sm);
  const size_t smem = sizeof(ActSmem) + 1024;
  const bool col = q_col != nullptr;
  cudaError_t e = cudaSuccess;
#define FP8BW_QA(MD, CL, FM)                                                                      \
  do {                                                                                            \
    e = cudaFuncSetAttribute(k_quant_act<MD, CL, FM>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             (int)smem);                                                          \
    if (e == cudaSuccess)                                                                         \
      k_quant_act<MD, CL, FM><<<grid, QT, smem, st>>>(tm, M, K, q_row, s_row, q_col, s_col);      \
  } while (0)
  if (fmt == FP8BW_FMT_E5M2) {
    if (mode == FP8BW_SCALE_FP32) {
      if (col) FP8BW_QA(0, true, 1); else FP8BW_QA(0, false, 1);
    } else {
      if (col) FP8BW_QA(1, true, 1); else FP8BW_QA(1, false, 1);
    }
  } else if (mode == FP8BW_SCALE_FP32) {
    if (col) FP8BW_QA(0, true, 0); else FP8BW_QA(0, false, 0);
  } else {
    if (col) FP8BW_QA(1, true, 0); else FP8BW_QA(1, false, 0);
  }
#undef FP8BW_QA
  if (e != cudaSuccess) return e;
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

cudaError_t quant_read_clear_error(uint32_t* out, cudaStream_t st) {
  uint32_t v = 0, z = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_quant_error, sizeof v, 0, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess && v) e = cudaMemcpyToSymbolAsync(g_quant_error, &z, sizeof z, 0, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  *out = v;
  return e;
}

}  // namespace fp8bw

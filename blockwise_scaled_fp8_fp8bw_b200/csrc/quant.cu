// Blockwise E4M3 quantizers (HBM-bound): activations with 1x128 blocks plus
// the fused column-wise copy, weights with 128x128 blocks plus the byte
// transpose, and the batched per-step requantization of many weights.
//
// Method: "NVIDIA NeMo RL erreicht 48% ..." section "Der technische
// Durchbruch" (E4M3, 128x128 weight blocks, 1x128 activation blocks) and
// "Leistungsgewinne in der Praxis" (scales recalibrated after every step).
//
// Design: one CTA of 256 threads per 128x128 bf16 tile (32 KB).  Each thread
// loads eight 16-byte vectors (a half-warp covers one 256-byte row segment),
// keeps them in registers for the row-wise pass and parks them in shared
// memory for the column-wise pass.
//  * amax: bf16 magnitudes compared as packed unsigned 16-bit integers
//    (sign bit cleared; the bit order of non-negative bf16 values is their
//    numeric order), two elements per instruction.
//  * x / s: the block's divisor is fixed, so its IEEE reciprocal y = RN(1/s)
//    is taken once per block and every element uses one Markstein correction
//    step (P. Markstein, "Computation of elementary functions on the IBM
//    RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990):
//        q0 = RN(x*y);  r = fma(-q0, s, x) (exact);  q = fma(r, y, q0)
//    on packed f32x2 lanes, and the sign of x is copied onto q.  An
//    exhaustive check over every bf16 block amax >= 2^-80 and every bf16
//    |x| <= amax shows q equals RN(x/s) wherever |x/s| >= 2^-12; below that
//    both give a signed-zero code (tests/test_division_scheme.py).  Blocks
//    with a smaller amax use IEEE division.  In power-of-2 mode 1/s is exact
//    and x*(1/s) is the correctly rounded x/s.
//  * codes leave as coalesced stores: row-wise codes as 8-byte stores (a
//    half-warp writes a 128-byte row); column-wise codes are staged in a
//    swizzled 16 KB shared tile and written as full 128-byte rows.

#include "common.cuh"
#include "tmap.cuh"

namespace fp8bw {
namespace {

constexpr int QT = 256;  // threads per tile CTA
constexpr uint32_t kAbsMask = 0x7FFF7FFFu;

struct WeightSmem {
  uint32_t codes[128][32];   // row-major codes, swizzled words
  uint32_t red[8];
};

__device__ __forceinline__ uint32_t umax2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// max |x| over a packed word's two halves, as a float (bf16 widened)
__device__ __forceinline__ float halves_max(uint32_t m) {
  const uint32_t lo = m & 0xFFFFu, hi = m >> 16;
  return __uint_as_float((lo > hi ? lo : hi) << 16);
}

__device__ __forceinline__ uint32_t absmax8(uint4 v) {
  return umax2(umax2(v.x & kAbsMask, v.y & kAbsMask), umax2(v.z & kAbsMask, v.w & kAbsMask));
}

__device__ __forceinline__ float rcp_rn(float s) {
  float y;
  asm("rcp.rn.f32 %0, %1;" : "=f"(y) : "f"(s));
  return y;
}

// Per-block divisor: scale s, reciprocal y, and whether the block must use
// IEEE division (FP32 mode with amax < 2^-80).
struct Divisor {
  float s, y;
  bool exact;
};

template <int MODE>
__device__ __forceinline__ Divisor make_divisor(float amax) {
  Divisor d;
  d.s = block_scale<MODE>(amax);
  if (MODE == FP8BW_SCALE_POW2) {
    d.y = rcp_rn(d.s);  // exact: s is a power of two in [2^-127, 2^127]
    d.exact = false;
  } else {
    d.exact = !(amax >= 0x1p-80f);
    d.y = d.exact ? 0.0f : rcp_rn(d.s);
  }
  return d;
}

__device__ __forceinline__ float copysign_bits(float q, float x) {
  return __uint_as_float((__float_as_uint(q) & 0x7FFFFFFFu) | (__float_as_uint(x) & 0x80000000u));
}

// RN(x / s) for a pair of values with per-lane divisors (s0,y0), (s1,y1):
// power-of-2 mode multiplies by the exact reciprocal, FP32 mode takes one
// Markstein step.  Blocks that need IEEE division take the slow path below.
template <int MODE>
__device__ __forceinline__ float2 div2(float2 x, float2 s, float2 y) {
  if (MODE == FP8BW_SCALE_POW2) return fmul2(x, y);
  const float2 q0 = fmul2(x, y);
  const float2 r = ffma2(q0, make_float2(-s.x, -s.y), x);
  const float2 q = ffma2(r, y, q0);
  return make_float2(copysign_bits(q.x, x.x), copysign_bits(q.y, x.y));
}

// Scalar RN(x / s) in FP32 mode, IEEE division for a block that needs it.
__device__ __forceinline__ float div1(float x, const Divisor& d) {
  if (d.exact) return __fdiv_rn(x, d.s);
  const float q0 = __fmul_rn(x, d.y);
  const float r = __fmaf_rn(-q0, d.s, x);
  return copysign_bits(__fmaf_rn(r, d.y, q0), x);
}

template <int MODE>
__device__ __forceinline__ uint2 quant8_fast(uint4 v, float s, float y) {
  const float2 s2 = make_float2(s, s), y2 = make_float2(y, y);
  const float2 a = div2<MODE>(make_float2(bf16lo(v.x), bf16hi(v.x)), s2, y2);
  const float2 b = div2<MODE>(make_float2(bf16lo(v.y), bf16hi(v.y)), s2, y2);
  const float2 c = div2<MODE>(make_float2(bf16lo(v.z), bf16hi(v.z)), s2, y2);
  const float2 e = div2<MODE>(make_float2(bf16lo(v.w), bf16hi(v.w)), s2, y2);
  return make_uint2(cvt_e4m3x2(a.x, a.y) | (cvt_e4m3x2(b.x, b.y) << 16),
                    cvt_e4m3x2(c.x, c.y) | (cvt_e4m3x2(e.x, e.y) << 16));
}

// Slow path (kept out of line so the fast path carries no division code).
__device__ __noinline__ uint2 quant8_exact(uint4 v, Divisor d) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[2];
  for (int i = 0; i < 2; ++i)
    o[i] = cvt_e4m3x2(div1(bf16lo(w[2 * i]), d), div1(bf16hi(w[2 * i]), d)) |
           (cvt_e4m3x2(div1(bf16lo(w[2 * i + 1]), d), div1(bf16hi(w[2 * i + 1]), d)) << 16);
  return make_uint2(o[0], o[1]);
}

// 8 codes of one 16-byte vector with one divisor (uniform branch per warp).
template <int MODE>
__device__ __forceinline__ uint2 quant8(uint4 v, const Divisor& d) {
  if (MODE == FP8BW_SCALE_FP32 && __any_sync(0xffffffffu, d.exact)) return quant8_exact(v, d);
  return quant8_fast<MODE>(v, d.s, d.y);
}

struct ColCodes {
  uint32_t c0[8], c1[8];
};

// Slow path of the column pass: re-reads the thread's 32 words.
__device__ __noinline__ ColCodes column_codes_exact(const uint32_t (*tile)[64], int wc, int rg,
                                                   Divisor d0, Divisor d1) {
  ColCodes c;
  for (int i = 0; i < 8; ++i) {
    float a[4], b[4];
    for (int u = 0; u < 4; ++u) {
      const uint32_t w = tile[rg * 32 + 4 * i + u][wc];
      a[u] = div1(bf16lo(w), d0);
      b[u] = div1(bf16hi(w), d1);
    }
    c.c0[i] = cvt_e4m3x2(a[0], a[1]) | (cvt_e4m3x2(a[2], a[3]) << 16);
    c.c1[i] = cvt_e4m3x2(b[0], b[1]) | (cvt_e4m3x2(b[2], b[3]) << 16);
  }
  return c;
}

// Swizzled byte tile: row r (128 bytes = 8 chunks of 16 B); logical chunk j
// lives at physical chunk j ^ ((r >> 1) & 7).
__device__ __forceinline__ uint4* code_chunk(uint32_t* codes, int r, int j) {
  return reinterpret_cast<uint4*>(codes + r * 32 + 4 * (j ^ ((r >> 1) & 7)));
}

// Writes the 128x128 transposed code tile to dst (row stride ld bytes) as
// full 128-byte rows: thread t copies chunk t%8 of rows t/8 + 32i.
__device__ __forceinline__ void store_code_tile(uint32_t (*tile)[64], uint8_t* dst, int64_t ld) {
  uint32_t* codes = &tile[0][0];
  const int t = threadIdx.x, j = t & 7;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = (t >> 3) + 32 * i;
    *reinterpret_cast<uint4*>(dst + (int64_t)r * ld + 16 * j) = *code_chunk(codes, r, j);
  }
}

// ---------------------------------------------------------- activations ---
// Column pass: thread (wc, rg) owns columns 2wc, 2wc+1 and rows 32rg..+31 of
// the shared bf16 tile; quantizes them with the column blocks' scales into
// the swizzled code tile (row = column index, bytes = token index).
template <int MODE, typename S>
__device__ __forceinline__ void act_column_pass(S& sm, uint32_t (*tile)[64], float* s_col) {
  const int tid = threadIdx.x;
  const int wc = tid & 63, rg = tid >> 6;
  uint32_t wv[32];
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    wv[i] = tile[rg * 32 + i][wc];
    m = umax2(m, wv[i] & kAbsMask);
  }
  sm.colmax[rg][wc] = m;
  __syncthreads();
  m = umax2(umax2(sm.colmax[0][wc], sm.colmax[1][wc]), umax2(sm.colmax[2][wc], sm.colmax[3][wc]));
  const Divisor d0 = make_divisor<MODE>(__uint_as_float((m & 0xFFFFu) << 16));
  const Divisor d1 = make_divisor<MODE>(__uint_as_float(m & 0xFFFF0000u));
  if (rg == 0) *reinterpret_cast<float2*>(s_col + 2 * wc) = make_float2(d0.s, d1.s);
  const float2 s2 = make_float2(d0.s, d1.s), y2 = make_float2(d0.y, d1.y);
  uint32_t c0[8], c1[8];
  if (MODE == FP8BW_SCALE_FP32 && __any_sync(0xffffffffu, d0.exact || d1.exact)) {
    const ColCodes c = column_codes_exact(tile, wc, rg, d0, d1);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      c0[i] = c.c0[i];
      c1[i] = c.c1[i];
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float2 q[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t w = wv[4 * i + u];
        q[u] = div2<MODE>(make_float2(bf16lo(w), bf16hi(w)), s2, y2);
      }
      c0[i] = cvt_e4m3x2(q[0].x, q[1].x) | (cvt_e4m3x2(q[2].x, q[3].x) << 16);
      c1[i] = cvt_e4m3x2(q[0].y, q[1].y) | (cvt_e4m3x2(q[2].y, q[3].y) << 16);
    }
  }
  __syncthreads();  // every thread is done with the bf16 tile; reuse it for codes
  uint32_t* codes = &tile[0][0];
  *code_chunk(codes, 2 * wc, 2 * rg) = make_uint4(c0[0], c0[1], c0[2], c0[3]);
  *code_chunk(codes, 2 * wc, 2 * rg + 1) = make_uint4(c0[4], c0[5], c0[6], c0[7]);
  *code_chunk(codes, 2 * wc + 1, 2 * rg) = make_uint4(c1[0], c1[1], c1[2], c1[3]);
  *code_chunk(codes, 2 * wc + 1, 2 * rg + 1) = make_uint4(c1[4], c1[5], c1[6], c1[7]);
}

// Persistent activation quantizer: each CTA walks tiles t = blockIdx.x +
// i*gridDim.x (column tile fastest).  One thread TMA-loads tile i+1 into the
// other half of a double buffer while all threads work on tile i, so every
// SM keeps about 32 KB of loads in flight per resident CTA.
struct ActSmem {
  uint32_t buf[2][128][64];  // bf16 tiles (256-byte rows); a finished tile's
                             // buffer then holds its transposed codes
  uint32_t colmax[4][64];
  float srow[128];
  uint64_t full[2];
};

__device__ __forceinline__ void issue_tile(ActSmem& sm, const CUtensorMap* tm, int t, int nK, int b) {
  const uint32_t bar = smem_u32(&sm.full[b]);
  mbar_arrive_expect_tx(bar, 128 * 256);
  tma_load_2d(smem_u32(&sm.buf[b][0][0]), tm, bar, (t % nK) * 128, (t / nK) * 128);
}

template <int MODE, bool COL>
__global__ void __launch_bounds__(QT, 3) k_quant_act(const __grid_constant__ CUtensorMap tmX,
                                                     int64_t M, int64_t K,
                                                     uint8_t* __restrict__ q_row,
                                                     float* __restrict__ s_row,
                                                     uint8_t* __restrict__ q_col,
                                                     float* __restrict__ s_col) {
  extern __shared__ uint8_t smem_raw[];
  ActSmem& sm = *reinterpret_cast<ActSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                            ~uintptr_t(127));
  const int tid = threadIdx.x;
  const int r16 = tid >> 4, vec = tid & 15;
  const int lane = tid & 31, half_base = lane & 16;
  const int nK = (int)(K / 128);
  const int tiles = nK * (int)(M / 128);
  if (tid == 0) {
    mbar_init(smem_u32(&sm.full[0]), 1);
    mbar_init(smem_u32(&sm.full[1]), 1);
    fence_barrier_init();
    prefetch_tmap(&tmX);
  }
  __syncthreads();
  if (tid == 0 && (int)blockIdx.x < tiles) issue_tile(sm, &tmX, blockIdx.x, nK, 0);
  int i = 0;
  for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
    const int cur = i & 1;
    const int64_t k0 = (int64_t)(t % nK) * 128, m0 = (int64_t)(t / nK) * 128;
    if (tid == 0 && t + (int)gridDim.x < tiles) {
      fence_proxy_async_smem();  // generic accesses to the other buffer are done
      issue_tile(sm, &tmX, t + gridDim.x, nK, cur ^ 1);
    }
    if (!mbar_wait(smem_u32(&sm.full[cur]), (i >> 1) & 1)) return;  // bounded: never expected
    uint32_t (*tile)[64] = sm.buf[cur];
    uint4 v[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) v[p] = *reinterpret_cast<const uint4*>(&tile[p * 16 + r16][vec * 4]);
    // Row amaxes of the 8 rows this half-warp touches (reduced over 16 lanes).
    uint32_t m[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      m[p] = absmax8(v[p]);
      m[p] = umax2(m[p], __shfl_xor_sync(0xffffffffu, m[p], 8));
      m[p] = umax2(m[p], __shfl_xor_sync(0xffffffffu, m[p], 4));
      m[p] = umax2(m[p], __shfl_xor_sync(0xffffffffu, m[p], 2));
      m[p] = umax2(m[p], __shfl_xor_sync(0xffffffffu, m[p], 1));
    }
    // One divisor per lane instead of one per row per lane: lane L of each
    // half-warp prepares the divisor of pass L & 7; the others fetch it by
    // shuffle.
    uint32_t mine = m[0];
#pragma unroll
    for (int p = 1; p < 8; ++p) mine = ((lane & 7) == p) ? m[p] : mine;
    const Divisor dl = make_divisor<MODE>(halves_max(mine));
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const int row = p * 16 + r16;
      Divisor d;
      d.s = __shfl_sync(0xffffffffu, dl.s, half_base + p);
      d.y = __shfl_sync(0xffffffffu, dl.y, half_base + p);
      d.exact = MODE == FP8BW_SCALE_FP32 && !(halves_max(m[p]) >= 0x1p-80f);
      *reinterpret_cast<uint2*>(q_row + (m0 + row) * K + k0 + vec * 8) = quant8<MODE>(v[p], d);
      if (vec == 0) sm.srow[row] = d.s;
    }
    if (COL) {
      // the row pass only read the tile: no barrier needed before the column pass
      act_column_pass<MODE>(sm, tile, s_col + (m0 / 128) * K + k0);
    }
    __syncthreads();
    if (tid < 32)
      *reinterpret_cast<float4*>(s_row + (k0 / 128) * M + m0 + 4 * tid) =
          *reinterpret_cast<const float4*>(&sm.srow[4 * tid]);
    if (COL) store_code_tile(tile, q_col + k0 * M + m0, M);
    fence_proxy_async_smem();
    __syncthreads();  // this buffer may now be refilled by the next TMA load
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
                             int num_sms, cudaStream_t st) {
  CUtensorMap tm;
  if (!make_map(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, (uint64_t)K, (uint64_t)M,
                (uint64_t)ldx, 128, 128, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  const int64_t tiles = (K / 128) * (M / 128);
  const int per_sm = 3;
  const unsigned grid = (unsigned)(tiles < (int64_t)num_sms * per_sm ? tiles : (int64_t)num_sms * per_sm);
  const size_t smem = sizeof(ActSmem) + 128;
  const bool col = q_col != nullptr;
  cudaError_t e = cudaSuccess;
#define FP8BW_QA(MD, CL)                                                                      \
  do {                                                                                        \
    e = cudaFuncSetAttribute(k_quant_act<MD, CL>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             (int)smem);                                                      \
    if (e == cudaSuccess) k_quant_act<MD, CL><<<grid, QT, smem, st>>>(tm, M, K, q_row, s_row, q_col, s_col); \
  } while (0)
  if (mode == FP8BW_SCALE_FP32) {
    if (col) FP8BW_QA(0, true); else FP8BW_QA(0, false);
  } else {
    if (col) FP8BW_QA(1, true); else FP8BW_QA(1, false);
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

}  // namespace fp8bw

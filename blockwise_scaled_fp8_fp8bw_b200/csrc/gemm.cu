// Tensor-core GEMMs for sm_100a: the blockwise-scaled FP8 GEMM (dense and
// grouped, fprop / dgrad / wgrad) and the BF16 comparison GEMM.
//
// Method: "NVIDIA NeMo RL erreicht 48% ..." section "Der technische
// Durchbruch": linear layers run FP8 math on E4M3 operands with one scale per
// 1x128 activation block and per 128x128 weight block; FP8 has twice the
// BF16 peak.  Section "Leistungsgewinne in der Praxis": the Qwen3-30B MoE
// model trains with the same recipe (grouped expert GEMMs).
//
// FP8 kernel (persistent, 384 threads per CTA, one CTA per SM).  Output tile
// 256x256 per CTA pair (PAIR: a 2-CTA cluster, tcgen05 cta_group::2, M=256
// split over the two SMs, each SM holding its own 128 A rows and half of the
// 256 B rows); grouped fprop/dgrad pair tiles stay inside one expert (see
// decode_tile).  Roles per CTA:
//   warp 0      TMA producer: per 128-wide K chunk, the CTA's 128x128 A tile
//               and its B tile (128 or 256 rows) into a shared-memory ring
//               (E4M3, 128-byte swizzle).  In a pair both CTAs count their
//               bytes on the first CTA's barrier.
//   warp 1      MMA issuer (first CTA of a pair only): four tcgen05.mma
//               kind::f8f6f4 (K = 32) per chunk into one of two TMEM chunk
//               accumulators (2 x 256 columns = all of TMEM), then commits
//               to the stage-empty and chunk-full barriers of both CTAs.
//   warp 2      scale loader: the chunk's 128 A-row scales and the B scales
//               (2 block scales, or 256 column scales for wgrad) into an
//               8-slot shared ring with cp.async.
//   warps 4-11  promotion: each warp owns a 32-row quarter of TMEM lanes and
//               128 columns (fprop/dgrad: a thread per row, 32x32b loads in
//               two rounds of 64 columns; wgrad: 4 rows x 32 columns per
//               thread, 16x256b loads, so the per-column scales need few
//               shared loads — with the quantizing epilogue a thread per row
//               and the column scales as warp-wide 16-byte shared
//               broadcasts); per chunk it reads the chunk product from TMEM,
//               multiplies by sA*sB in fp32 and adds it to its registers
//               (packed f32x2 FMAs), releasing the TMEM buffer as soon as
//               the last round is in registers so the MMA of the next
//               chunk overlaps.  At the end of a tile the results are
//               rounded to bf16 (or kept fp32), staged in shared memory
//               (64-byte swizzle, three pieces per warp) and written by TMA
//               stores (or TMA reduce-adds).
// Registers: warpgroup 0 drops to 56 per thread, the promotion warpgroups
// rise to 224 (128 accumulators + 64 staging); 56*128 + 224*256 = 64512 =
// 384 * 168, the launch allocation (checked on the host before launch).
// Every wait is bounded; on a timeout the kernel latches an error bit and
// leaves its loops.

#include <cstring>

#include "blockquant.cuh"
#include "common.cuh"
#include "tmap.cuh"

namespace fp8bw {

__device__ uint32_t g_gemm_error;

namespace {

constexpr int BM = 128, BN = 256, BK = 128;
constexpr int kThreads = 384;
constexpr int kScaleStages = 8;
constexpr uint32_t kATile = BM * BK;  // 16 KB: one CTA's A rows
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxGroups = FP8BW_MAX_EXPERTS;
constexpr uint32_t kEpiPiece = 2048;  // 32 rows x 32 bf16 (or 16 fp32): one TMA store

// Output of the FP8 GEMMs: bf16 (the default), fp32, or fp32 added to D.
enum OutMode : int { OUT_BF16 = 0, OUT_F32 = 1, OUT_F32_ADD = 2 };

// Epilogue kind of the promotion kernel (a template parameter): bf16 tiles,
// fp32 tiles (stored or added, per OutMode), or the bf16 result quantized
// into 1x128 row blocks and the column-wise copy (FP32 or POW2 scale rule).
enum OutKind : int { OK_BF16 = 0, OK_F32 = 1, OK_QUANT_FP32 = 2, OK_QUANT_POW2 = 3 };

// Quantizing epilogue: per column half of the tile (4 warps, 128 rows x 128
// columns) a swizzled bf16 tile, the partial column maxima and a barrier.
constexpr uint32_t kQHalfBytes = 40960;
constexpr uint32_t kQColmaxOff = 32768, kQBarOff = 33280;

template <bool PAIR, bool QOUT = false>
struct Cfg {
  static constexpr uint32_t kBTile = PAIR ? (BN / 2) * BK : BN * BK;  // this CTA's B rows
  static constexpr uint32_t kStageBytes = kATile + kBTile;
  static constexpr int kStages = QOUT ? 4 : (PAIR ? 5 : 4);
  static constexpr int kEpiBufs = PAIR ? 3 : 1;  // staging pieces per promotion warp
  static constexpr uint32_t kEpiBytes = QOUT ? kQHalfBytes / 4 : kEpiBufs * kEpiPiece;
  static constexpr uint32_t kIdesc = idesc_make(0, 0, PAIR ? 2 * BM : BM, BN);  // E4M3 -> F32
  static constexpr uint32_t kTemptyCount = PAIR ? 16 : 8;
};


constexpr int kRegsLow = 56, kRegsHigh = 224, kRegsLaunch = 168;


static_assert(kRegsLow * 128 + kRegsHigh * 256 <= kRegsLaunch * kThreads, "register split");

struct ScaleSlot {
  float sa[128];
  float sb[256];
};

constexpr int kMaxStages = 6;
struct Bars {
  uint64_t full[kMaxStages], empty[kMaxStages];
  uint64_t sfull[kScaleStages], sempty[kScaleStages];
  uint64_t tfull[2], tempty[2];
  uint32_t tmem_base;
  int32_t abort;
  int32_t bad_offsets;
};

struct GemmArgs {
  int M, N, K;         // GEMM sizes (grouped wgrad: M = out, N = in, K = tokens)
  int m_tiles, n_tiles, tiles, band;
  const float* sA;     // [K/128][M]
  const float* sB;     // per kind
  const int32_t* offsets;  // grouped: device [G+1]
  int G;
  uint16_t* D;         // quantizing epilogue: optional bf16 copy of the result
  int64_t ldd;
  uint8_t* q_row;      // quantizing epilogue: [M][N] codes, s_row [N/128][M]
  float* s_row;
  uint8_t* q_col;      // column-wise copy [N][M], s_col [M/128][N]
  float* s_col;
  int out_mode;        // OutMode of the FP8 kernels' epilogue
  uint32_t fmt_bits;   // operand formats in the MMA instruction descriptor (0: both E4M3)
  int stall_chunk;     // testing: CTA 0's producer never fills this chunk (-1: off)
};

template <bool PAIR, bool QOUT = false>
constexpr size_t smem_fp8() {
  return 1024 + size_t(Cfg<PAIR, QOUT>::kStages) * Cfg<PAIR, QOUT>::kStageBytes +
         size_t(kScaleStages) * sizeof(ScaleSlot) + 8 * Cfg<PAIR, QOUT>::kEpiBytes + sizeof(Bars) +
         2 * sizeof(int32_t) * (kMaxGroups + 1);
}
static_assert(smem_fp8<true>() <= 232448 && smem_fp8<false>() <= 232448 && smem_fp8<true, true>() <= 232448,
              "shared memory budget");

// The four warps of one column half meet (bounded); `uses` counts the
// half's earlier meetings.  False if a warp did not arrive in time.
__device__ __forceinline__ bool half_meet(uint32_t bar, int lane, uint32_t uses) {
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
  return __all_sync(0xffffffffu, mbar_wait(bar, uses & 1));
}

// Quantizing epilogue of one column half: this thread holds row `rr` (of the
// CTA's 128) of the bf16-rounded result, 128 columns as 64 packed words.
// Writes D (if requested), the row codes and scale of its 1x128 block, and,
// with the other 127 threads of the half, the column-wise copy of the
// 128x128 tile: exactly what fp8bw_quant_act_1x128 makes of D.
template <int QM>
__device__ __forceinline__ bool quant_epilogue(const GemmArgs& a, uint8_t* hb, int tid, int lane,
                                               uint32_t& uses, int row0, int col0, const uint32_t (&w)[64]) {
  const int rr = tid;                      // the thread's row within the tile
  const int64_t grow = row0 + rr;
  const int64_t M = a.M, N = a.N;
  if (a.D) {
    uint4* drow = reinterpret_cast<uint4*>(a.D + grow * a.ldd + col0);
#pragma unroll
    for (int k = 0; k < 16; ++k) drow[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
  }
  // row pass: the thread's 128 values are one 1x128 block
  {
    uint32_t m = 0;
#pragma unroll
    for (int k = 0; k < 64; ++k) m = umax2(m, w[k] & kAbsMask);
    const Divisor d = make_divisor<QM>(halves_max(m));
    a.s_row[(col0 / 128) * M + grow] = d.s;
    uint8_t* qr = a.q_row + grow * N + col0;
#pragma unroll
    for (int k = 0; k < 16; k += 4) {
      const uint2 c0 = quant8<QM>(make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]), d);
      const uint2 c1 = quant8<QM>(make_uint4(w[4 * k + 4], w[4 * k + 5], w[4 * k + 6], w[4 * k + 7]), d);
      const uint2 c2 = quant8<QM>(make_uint4(w[4 * k + 8], w[4 * k + 9], w[4 * k + 10], w[4 * k + 11]), d);
      const uint2 c3 = quant8<QM>(make_uint4(w[4 * k + 12], w[4 * k + 13], w[4 * k + 14], w[4 * k + 15]), d);
      st_global_v8(qr + 8 * k, make_uint4(c0.x, c0.y, c1.x, c1.y), make_uint4(c2.x, c2.y, c3.x, c3.y));
    }
  }
  if (!a.q_col) return true;
  // column-wise copy: the tile goes through shared memory (two boxes of 64
  // columns, 128-byte swizzle), a thread takes two columns x 64 rows
  const uint32_t bar = smem_u32(hb + kQBarOff);
  uint32_t* colmax = reinterpret_cast<uint32_t*>(hb + kQColmaxOff);
#pragma unroll
  for (int k = 0; k < 16; ++k)
    *reinterpret_cast<uint4*>(hb + act_off(k >> 3, rr, k & 7)) = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
  if (!half_meet(bar, lane, uses++)) return false;
  const int wc = tid & 63, rg = tid >> 6;
  const int cbox = wc >> 5, cchunk = (wc & 31) >> 2, cword = wc & 3;
  ColWords cw[2];
  uint32_t m = 0;
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      cw[h].w[r] = *reinterpret_cast<const uint32_t*>(hb + act_off(cbox, rg * 64 + h * 32 + r, cchunk) + 4 * cword);
      m = umax2(m, cw[h].w[r] & kAbsMask);
    }
  colmax[rg * 64 + wc] = m;
  if (!half_meet(bar, lane, uses++)) return false;
  m = umax2(colmax[wc], colmax[64 + wc]);
  const Divisor d0 = make_divisor<QM>(__uint_as_float((m & 0xFFFFu) << 16));
  const Divisor d1 = make_divisor<QM>(__uint_as_float(m & 0xFFFF0000u));
  if (rg == 0) *reinterpret_cast<float2*>(a.s_col + (int64_t)(row0 / 128) * N + col0 + 2 * wc) = make_float2(d0.s, d1.s);
  const bool slow = QM == FP8BW_SCALE_FP32 && __any_sync(0xffffffffu, d0.exact || d1.exact);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t c0[8], c1[8];
    if (slow) {
      const ColCodes c = column_codes_exact<FP8BW_FMT_E4M3>(cw[h], d0, d1);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c0[j] = c.c0[j];
        c1[j] = c.c1[j];
      }
    } else {
      const float2 s2 = make_float2(d0.s, d1.s), y2 = make_float2(d0.y, d1.y);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float2 qv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t x = cw[h].w[4 * j + u];
          qv[u] = div2<QM>(make_float2(bf16lo(x), bf16hi(x)), s2, y2);
        }
        c0[j] = cvt_e4m3x2(qv[0].x, qv[1].x) | (cvt_e4m3x2(qv[2].x, qv[3].x) << 16);
        c1[j] = cvt_e4m3x2(qv[0].y, qv[1].y) | (cvt_e4m3x2(qv[2].y, qv[3].y) << 16);
      }
    }
    uint8_t* qc = a.q_col + (int64_t)(col0 + 2 * wc) * M + row0 + rg * 64 + h * 32;
    st_global_v8(qc, make_uint4(c0[0], c0[1], c0[2], c0[3]), make_uint4(c0[4], c0[5], c0[6], c0[7]));
    st_global_v8(qc + M, make_uint4(c1[0], c1[1], c1[2], c1[3]), make_uint4(c1[4], c1[5], c1[6], c1[7]));
  }
  return true;
}

struct TileInfo {
  int mt, nt, g, kb0, kb1;
  int m0;    // first row of the tile (of the pair's 256 rows for a pair)
  int mend;  // rows at or past mend are not part of the result
  bool skip;
};

// Tile t -> (rows, n tile, expert, K-chunk range).  M tiles are 256 rows
// for a pair, 128 otherwise; dense tiles go in bands of `band` M tiles so
// that the CTAs running at once share A and B panels in L2.  Grouped
// fprop/dgrad tiles are pair tiles inside one expert: expert g's rows
// [off[g], off[g+1]) form ceil(rows/256) of them (pp[g] = those of the
// experts before g); in the last one the second CTA's 128 rows may lie past
// the segment, and that CTA then writes nothing.
template <int KIND, bool GROUPED, bool PAIR, bool WARP = false>
__device__ __forceinline__ TileInfo decode_tile(const GemmArgs& a, int t, const int32_t* off,
                                                const int32_t* pp, int& hint) {
  TileInfo ti;
  ti.g = 0;
  ti.skip = false;
  ti.mend = a.M;
  if (GROUPED && KIND == FP8BW_WGRAD) {
    const int per = a.m_tiles * a.n_tiles;
    ti.g = t / per;
    const int r = t - ti.g * per;
    ti.mt = r % a.m_tiles;
    ti.nt = r / a.m_tiles;
    ti.m0 = ti.mt * (PAIR ? 2 * BM : BM);
    ti.kb0 = off[ti.g] >> 7;
    ti.kb1 = off[ti.g + 1] >> 7;
    return ti;
  }
  ti.kb0 = 0;
  ti.kb1 = a.K / BK;
  if (GROUPED && PAIR) {
    const int pt = t / a.n_tiles;
    ti.nt = t - pt * a.n_tiles;
    ti.mt = pt;
    if (pt >= pp[a.G]) {
      ti.skip = true;
      ti.m0 = 0;
      return ti;
    }
    // The expert that owns pt: the last g with pp[g] <= pt.  A role visits
    // its tiles in increasing order, so the search moves forward from the
    // expert of its previous tile (`hint`).  A role steps over one tile per
    // CTA pair, so with short experts it passes many of them per tile: a
    // whole warp (WARP) tests the next 32 experts at once (pp is
    // non-decreasing, so the passing lanes are a prefix and their count is
    // the step); a single thread walks one expert per shared load.
    int g = hint;
    if (WARP) {
      const int lane = (int)(threadIdx.x & 31);
      for (;;) {
        const int cand = g + 1 + lane;
        const int adv = __popc(__ballot_sync(0xffffffffu, cand < a.G && pp[cand] <= pt));
        g += adv;
        if (adv < 32) break;
      }
    } else {
      while (g + 1 < a.G && pp[g + 1] <= pt) ++g;
    }
    hint = g;
    ti.g = g;
    ti.m0 = off[g] + (pt - pp[g]) * (2 * BM);
    ti.mend = off[g + 1];
    return ti;
  }
  const int band_tiles = a.band * a.n_tiles;
  const int band = t / band_tiles;
  const int r = t - band * band_tiles;
  const int rows = min(a.band, a.m_tiles - band * a.band);
  ti.mt = band * a.band + r % rows;
  ti.nt = r / rows;
  ti.m0 = ti.mt * (PAIR ? 2 * BM : BM);
  if (GROUPED) {
    const int row0 = ti.mt * BM;
    if (row0 >= off[a.G]) {
      ti.skip = true;
    } else {
      int lo = 0, hi = a.G - 1;  // last g with off[g] <= row0
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= row0) lo = mid; else hi = mid - 1;
      }
      ti.g = lo;
      ti.mend = off[lo + 1];
    }
  }
  return ti;
}

// Pair tiles per expert for grouped fprop/dgrad: pp[g+1] = pp[g] +
// ceil((off[g+1] - off[g]) / 256), scanned by warp 0 (32 experts a round).
// Every thread of the CTA must call it.
__device__ __forceinline__ void pair_prefix(const int32_t* off, int32_t* pp, int G) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int carry = 0;
    for (int base = 0; base < G; base += 32) {
      const int g = base + lane;
      int v = g < G ? (off[g + 1] - off[g] + 2 * BM - 1) / (2 * BM) : 0;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, d);
        if (lane >= d) v += u;
      }
      if (g < G) pp[g + 1] = carry + v;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) pp[0] = 0;
  }
  __syncthreads();
}

// fp32 output pieces are 32 rows x 16 columns (64-byte rows, 64-byte
// swizzle: 16-byte chunk c of row r at chunk c ^ ((r >> 1) & 3)).
// Row-per-lane accumulators (32x32b TMEM shape): a[j] = columns 2j, 2j+1.
__device__ __forceinline__ void stage_rows_f32(uint8_t* epi, int lane, const float2* a) {
#pragma unroll
  for (int c = 0; c < 4; ++c)
    *reinterpret_cast<float4*>(epi + lane * 64 + 16 * (c ^ ((lane >> 1) & 3))) =
        make_float4(a[2 * c].x, a[2 * c].y, a[2 * c + 1].x, a[2 * c + 1].y);
}

// Accumulators of the 16x256b shape (wgrad promotion): acc[16 i + g] holds
// row 8i + lane/4 and columns 8g + 2(lane%4) + {0, 1}; piece pp covers the
// column groups g = 2pp, 2pp + 1.
__device__ __forceinline__ void stage_quad_f32(uint8_t* epi, int lane, const float2* acc, int pp) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = 8 * i + (lane >> 2);
#pragma unroll
    for (int gg = 0; gg < 2; ++gg) {
      const int chunk = 2 * gg + ((lane & 3) >> 1);
      *reinterpret_cast<float2*>(epi + row * 64 + 16 * (chunk ^ ((row >> 1) & 3)) + 8 * (lane & 1)) =
          acc[16 * i + 2 * pp + gg];
    }
  }
}

// Writes (or adds) one staged fp32 piece.
__device__ __forceinline__ void emit_f32(const CUtensorMap* tmD, uint32_t src, int x, int y, int out_mode) {
  if (out_mode == OUT_F32_ADD) tma_reduce_add_2d(tmD, src, x, y);
  else tma_store_2d(tmD, src, x, y);
}

__device__ __forceinline__ void raise_timeout(Bars* bars) {
  atomicOr(&g_gemm_error, DEV_ERR_TIMEOUT);
  atomicExch(&bars->abort, 1);
}

template <typename B>
__device__ __forceinline__ void raise_timeout_mx(B* bars) {
  atomicOr(&g_gemm_error, DEV_ERR_TIMEOUT);
  atomicExch(&bars->abort, 1);
}

template <int KIND, bool GROUPED, bool PAIR, int OUTK>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm_fp8(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmD, const GemmArgs a) {
  constexpr bool F32OUT = OUTK == OK_F32;
  constexpr bool QOUT = OUTK == OK_QUANT_FP32 || OUTK == OK_QUANT_POW2;
  static_assert(!(QOUT && GROUPED), "quantizing epilogue: dense GEMMs only");
  using C = Cfg<PAIR, QOUT>;
  // wgrad promotion layout: the 16x256b shape (4 rows x 32 columns per
  // thread, PW = 0) in general; the quantizing epilogue needs a thread per
  // row (32x32b, PW = 2)
  constexpr int PW = QOUT ? 2 : 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  uint8_t* stage_base = smem;
  uint8_t* epi_base = smem + C::kStages * C::kStageBytes;  // 1024-aligned
  ScaleSlot* slots = reinterpret_cast<ScaleSlot*>(epi_base + 8 * C::kEpiBytes);
  Bars* bars = reinterpret_cast<Bars*>(slots + kScaleStages);
  int32_t* s_off = reinterpret_cast<int32_t*>(bars + 1);
  int32_t* s_pp = s_off + (kMaxGroups + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0;
  const bool leader = rank == 0;
  const int cta_slot = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;   // tile-loop index
  const int cta_step = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  int ghint = 0;  // expert of this thread's previous tile (grouped fprop/dgrad)

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(smem_u32(&bars->full[i]), 1);
      mbar_init(smem_u32(&bars->empty[i]), 1);
    }
    for (int i = 0; i < kScaleStages; ++i) {
      mbar_init(smem_u32(&bars->sfull[i]), 32);
      mbar_init(smem_u32(&bars->sempty[i]), 8);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars->tfull[i]), 1);
      mbar_init(smem_u32(&bars->tempty[i]), C::kTemptyCount);
    }
    if (QOUT)
      for (int h = 0; h < 2; ++h) mbar_init(smem_u32(epi_base + h * kQHalfBytes + kQBarOff), 4);
    bars->abort = 0;
    bars->bad_offsets = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    if (PAIR) {
      tmem_alloc_pair(smem_u32(&bars->tmem_base), kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
      tmem_relinquish();
    }
  }
  if (GROUPED) {
    for (int i = threadIdx.x; i <= a.G; i += kThreads) s_off[i] = a.offsets[i];
  }
  tc_fence_before();
  if (PAIR) cluster_sync(); else __syncthreads();
  tc_fence_after();
  if (GROUPED) {
    // Offsets must start at 0, be non-decreasing multiples of 128 and end
    // within the token matrix; otherwise nothing is computed or written.
    int bad = 0;
    for (int i = threadIdx.x; i < a.G; i += kThreads) {
      const int o0 = s_off[i], o1 = s_off[i + 1];
      if (o1 < o0 || (o1 & 127) || (i == 0 && o0 != 0)) bad = 1;
    }
    if (threadIdx.x == 0) {
      const int mtot = (KIND == FP8BW_WGRAD) ? a.K : a.M;
      if (s_off[a.G] > mtot || s_off[a.G] < 0) bad = 1;
    }
    if (__syncthreads_or(bad)) {
      if (threadIdx.x == 0) atomicOr(&g_gemm_error, DEV_ERR_CHECK);
      tc_fence_before();
      if (PAIR) cluster_sync();
      if (warp == 1) {
        if (PAIR) tmem_dealloc_pair(bars->tmem_base, kTmemCols);
        else tmem_dealloc(bars->tmem_base, kTmemCols);
      }
      return;
    }
    if (KIND != FP8BW_WGRAD && PAIR) pair_prefix(s_off, s_pp, a.G);
  }
  const uint32_t tmem = bars->tmem_base;
  // Barriers the MMA waits on live in the first CTA of a pair.
  const uint32_t full0 = PAIR ? mapa_shared(smem_u32(&bars->full[0]), 0) : smem_u32(&bars->full[0]);
  const uint32_t tempty0 = PAIR ? mapa_shared(smem_u32(&bars->tempty[0]), 0) : smem_u32(&bars->tempty[0]);

  if (warp < 4) {
    regs_dec<kRegsLow>();
    if (warp == 0) {
      // ------------------------------------------------ TMA producer ----
      if (lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
      }
      int stage = 0, chunk = 0;
      uint32_t phase = 0;
      for (int t = cta_slot; t < a.tiles; t += cta_step) {
        const TileInfo ti = decode_tile<KIND, GROUPED, PAIR, KIND != FP8BW_WGRAD>(a, t, s_off, s_pp, ghint);
        if (ti.skip) continue;
        const int arow = ti.m0 + (PAIR ? (int)rank * BM : 0);
        const int brow = PAIR ? ti.nt * BN + (int)rank * (BN / 2) : ti.nt * BN;
        for (int kb = ti.kb0; kb < ti.kb1; ++kb, ++chunk) {
          if (!mbar_wait(smem_u32(&bars->empty[stage]), phase ^ 1)) {
            raise_timeout(bars);
            goto done;
          }
          if (lane == 0 && !(blockIdx.x == 0 && chunk == a.stall_chunk)) {
            const uint32_t full = full0 + stage * 8;
            const uint32_t sa = smem_u32(stage_base + stage * C::kStageBytes);
            if (PAIR) {
              if (leader) mbar_arrive_expect_tx(smem_u32(&bars->full[stage]), 2 * C::kStageBytes);
              tma_load_2d_pair(sa, &tmA, full, kb * BK, arow);
              if (GROUPED && KIND != FP8BW_WGRAD)
                tma_load_3d_pair(sa + kATile, &tmB, full, kb * BK, brow, ti.g);
              else
                tma_load_2d_pair(sa + kATile, &tmB, full, kb * BK, brow);
            } else {
              mbar_arrive_expect_tx(full, C::kStageBytes);
              tma_load_2d(sa, &tmA, full, kb * BK, arow);
              if (GROUPED && KIND != FP8BW_WGRAD)
                tma_load_3d(sa + kATile, &tmB, full, kb * BK, brow, ti.g);
              else
                tma_load_2d(sa + kATile, &tmB, full, kb * BK, brow);
            }
          }
          __syncwarp();
          if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        }
        if (bars->abort) break;
      }
    } else if (warp == 1) {
      // ------------------------------------------------- MMA issuer -----
      if (leader && lane == 0) {
        int stage = 0, buf = 0;
        uint32_t phase = 0, bphase = 0;
        for (int t = cta_slot; t < a.tiles; t += cta_step) {
          const TileInfo ti = decode_tile<KIND, GROUPED, PAIR>(a, t, s_off, s_pp, ghint);
          if (ti.skip) continue;
          for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
            if (!mbar_wait(smem_u32(&bars->tempty[buf]), bphase ^ 1) ||
                !mbar_wait(smem_u32(&bars->full[stage]), phase)) {
              raise_timeout(bars);
              goto done;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(stage_base + stage * C::kStageBytes);
            const uint64_t da = sdesc_k_sw128(sa), db = sdesc_k_sw128(sa + kATile);
            const uint32_t d = tmem + buf * BN;
#pragma unroll
            for (int kk = 0; kk < BK / 32; ++kk) {  // +32 bytes = +2 in the >>4 address field
              if (PAIR) umma_f8f6f4_pair(d, da + 2 * kk, db + 2 * kk, C::kIdesc | a.fmt_bits, kk > 0 ? 1u : 0u);
              else umma_f8f6f4(d, da + 2 * kk, db + 2 * kk, C::kIdesc | a.fmt_bits, kk > 0 ? 1u : 0u);
            }
            if (PAIR) {
              umma_commit_pair(smem_u32(&bars->empty[stage]), 0x3);
              umma_commit_pair(smem_u32(&bars->tfull[buf]), 0x3);
            } else {
              umma_commit(smem_u32(&bars->empty[stage]));
              umma_commit(smem_u32(&bars->tfull[buf]));
            }
            if (++stage == C::kStages) { stage = 0; phase ^= 1; }
            if (++buf == 2) { buf = 0; bphase ^= 1; }
          }
          if (bars->abort) break;
        }
      }
    } else if (warp == 2) {
      // ------------------------------------------------ scale loader ----
      int ss = 0;
      uint32_t sphase = 0;
      const int nKb = a.K / BK, nNb = a.N / 128;
      for (int t = cta_slot; t < a.tiles; t += cta_step) {
        const TileInfo ti = decode_tile<KIND, GROUPED, PAIR, KIND != FP8BW_WGRAD>(a, t, s_off, s_pp, ghint);
        if (ti.skip) continue;
        const int row0 = ti.m0 + (PAIR ? (int)rank * BM : 0);
        const bool rows_ok = row0 < a.M;
        const float* sBg = a.sB;
        if (GROUPED && KIND != FP8BW_WGRAD) sBg += (size_t)ti.g * nNb * nKb;
        for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
          if (!mbar_wait(smem_u32(&bars->sempty[ss]), sphase ^ 1)) {
            raise_timeout(bars);
            goto done;
          }
          ScaleSlot* sl = &slots[ss];
          if (rows_ok)
            cp_async_16(smem_u32(&sl->sa[lane * 4]), a.sA + (size_t)kb * a.M + row0 + lane * 4);
          if (KIND == FP8BW_WGRAD) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int n = ti.nt * BN + h * 128 + lane * 4;
              if (n < a.N) cp_async_16(smem_u32(&sl->sb[h * 128 + lane * 4]), sBg + (size_t)kb * a.N + n);
            }
          } else if (lane < 2) {
            const int nb = ti.nt * 2 + lane;
            if (nb < nNb) {
              const float* src = (KIND == FP8BW_FPROP) ? sBg + (size_t)nb * nKb + kb
                                                       : sBg + (size_t)kb * nNb + nb;
              cp_async_4(smem_u32(&sl->sb[lane]), src);
            }
          }
          cp_async_mbar_arrive_noinc(smem_u32(&bars->sfull[ss]));
          if (++ss == kScaleStages) { ss = 0; sphase ^= 1; }
        }
        if (bars->abort) break;
      }
      asm volatile("cp.async.wait_all;" ::: "memory");
    }
  } else {
    regs_inc<kRegsHigh>();
    // -------------------------------------------------------- promotion --
    const int q = warp & 3;            // TMEM lane quarter of this warp
    const int half = (warp - 4) >> 2;  // column half of the 256-wide tile
    uint8_t* epi0 = epi_base + (warp - 4) * C::kEpiBytes;
    uint32_t qmeets = 0;  // quantizing epilogue: meetings of this column half
    int ss = 0;
    uint32_t sphase = 0;
    int buf = 0;
    uint32_t bphase = 0;
    for (int t = cta_slot; t < a.tiles; t += cta_step) {
      const TileInfo ti = decode_tile<KIND, GROUPED, PAIR, KIND != FP8BW_WGRAD>(a, t, s_off, s_pp, ghint);
      if (ti.skip) continue;
      const int row0 = ti.m0 + (PAIR ? (int)rank * BM : 0);
      const int col0 = ti.nt * BN + half * 128;
      float2 acc[64];
#pragma unroll
      for (int j = 0; j < 64; ++j) acc[j] = make_float2(0.f, 0.f);
      for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
        if (!mbar_wait(smem_u32(&bars->sfull[ss]), sphase) ||
            !mbar_wait(smem_u32(&bars->tfull[buf]), bphase)) {
          raise_timeout(bars);
          goto done;
        }
        tc_fence_after();
        const ScaleSlot* sl = &slots[ss];
        const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + buf * BN + half * 128;
        if (KIND == FP8BW_WGRAD && PW == 0) {
          // 16x256b shape: a thread holds 4 rows x 32 columns, so a chunk
          // costs 4 row-scale and 16 column-pair loads from shared memory.
          // acc[16 * i + g] holds row 8i + lane/4 of the quarter and columns
          // 8g + 2(lane%4) + {0, 1} of the warp's 128.
          float sa4[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) sa4[i] = sl->sa[q * 32 + 8 * i + (lane >> 2)];
          const float* sbw = &sl->sb[half * 128 + 2 * (lane & 3)];
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {  // 64-column halves of the warp's 128 columns
            uint32_t r[2][32];
            tmem_ld16x64(taddr + h2 * 64, r[0]);                      // quarter lanes 0-15
            tmem_ld16x64(taddr + (16u << 16) + h2 * 64, r[1]);        // quarter lanes 16-31
            tmem_wait_ld();
            tmem_fence_regs(r[0]);
            tmem_fence_regs(r[1]);
            if (h2 == 1) {
              // chunk fully read: hand the TMEM buffer back to the MMA warp
              tc_fence_before();
              __syncwarp();
              if (lane == 0) {
                if (PAIR && !leader) mbar_arrive_cluster(tempty0 + buf * 8);
                else mbar_arrive(smem_u32(&bars->tempty[buf]));
              }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int g = h2 * 8 + j;
              const float2 b2 = *reinterpret_cast<const float2*>(sbw + 8 * g);
#pragma unroll
              for (int u = 0; u < 2; ++u) {
#pragma unroll
                for (int v = 0; v < 2; ++v) {
                  const int i = 2 * u + v;
                  const float2 sc = fmul2(make_float2(sa4[i], sa4[i]), b2);
                  acc[16 * i + g] = ffma2(make_float2(__uint_as_float(r[u][4 * j + 2 * v]),
                                                      __uint_as_float(r[u][4 * j + 2 * v + 1])),
                                          sc, acc[16 * i + g]);
                }
              }
            }
          }
        } else {
          // The thread owns row q*32 + lane of the CTA's 128 and the 128
          // columns of its half (32x32b TMEM loads); wgrad's per-column
          // scales arrive as warp-wide 16-byte shared-memory broadcasts.
          const float sa = sl->sa[q * 32 + lane];
          float2 s2 = make_float2(sa, sa);
          if (KIND != FP8BW_WGRAD) {
            const float sc = sa * sl->sb[half];   // one scale for the row's 128 columns
            s2 = make_float2(sc, sc);
          }
          const float4* sb4 = reinterpret_cast<const float4*>(&sl->sb[half * 128]);
          // 32 columns (group g, registers rg) into the accumulators
          auto promote_group = [&](int g, const uint32_t* rg) {
            if (KIND == FP8BW_WGRAD) {
#pragma unroll
              for (int j4 = 0; j4 < 8; ++j4) {
                const float4 b = sb4[8 * g + j4];
                const float2 c0 = fmul2(s2, make_float2(b.x, b.y));
                const float2 c1 = fmul2(s2, make_float2(b.z, b.w));
                acc[16 * g + 2 * j4] = ffma2(make_float2(__uint_as_float(rg[4 * j4]), __uint_as_float(rg[4 * j4 + 1])),
                                             c0, acc[16 * g + 2 * j4]);
                acc[16 * g + 2 * j4 + 1] = ffma2(make_float2(__uint_as_float(rg[4 * j4 + 2]), __uint_as_float(rg[4 * j4 + 3])),
                                                 c1, acc[16 * g + 2 * j4 + 1]);
              }
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j)
                acc[16 * g + j] = ffma2(make_float2(__uint_as_float(rg[2 * j]), __uint_as_float(rg[2 * j + 1])),
                                        s2, acc[16 * g + j]);
            }
          };
          auto release = [&]() {
            // chunk fully read: hand the TMEM buffer back to the MMA warp
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              if (PAIR && !leader) mbar_arrive_cluster(tempty0 + buf * 8);
              else mbar_arrive(smem_u32(&bars->tempty[buf]));
            }
          };
          {
            // two rounds of 64 columns: release after the second round lands
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              uint32_t r[2][32];
              tmem_ld64(taddr + h2 * 64, r[0], r[1]);
              tmem_wait_ld();
              tmem_fence_regs(r[0]);
              tmem_fence_regs(r[1]);
              if (h2 == 1) release();
              promote_group(2 * h2, r[0]);
              promote_group(2 * h2 + 1, r[1]);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->sempty[ss]));
        if (++ss == kScaleStages) { ss = 0; sphase ^= 1; }
        if (++buf == 2) { buf = 0; bphase ^= 1; }
      }
      // ---- epilogue: bf16 rows through shared memory, TMA stores of 32x32
      // pieces (rows / columns outside the output are clipped by the TMA).
      const int drow = (GROUPED && KIND == FP8BW_WGRAD ? ti.g * a.M : 0) + row0 + q * 32;
      // (a pair's second CTA past the last row of M, or of the expert's
      // segment, computed nothing real)
      if (row0 >= ti.mend) {
        // nothing of this CTA's rows is part of the result
      } else if (QOUT) {
        if (col0 < a.N) {
          uint32_t w[64];
#pragma unroll
          for (int j = 0; j < 64; ++j) w[j] = pack_bf16x2(acc[j].x, acc[j].y);
          if (!quant_epilogue<OUTK == OK_QUANT_POW2 ? FP8BW_SCALE_POW2 : FP8BW_SCALE_FP32>(
                  a, epi_base + half * kQHalfBytes, q * 32 + lane, lane, qmeets, row0, col0, w)) {
            raise_timeout(bars);
            goto done;
          }
        }
      } else if (F32OUT) {
        // fp32 output: eight 32x16 pieces per warp, stored or added to D
#pragma unroll
        for (int pp = 0; pp < 8; ++pp) {
          uint8_t* epi = epi0 + (pp % C::kEpiBufs) * kEpiPiece;
          if (lane == 0) {
            bulk_wait_read<C::kEpiBufs - 1>();
          }
          __syncwarp();
          if (KIND == FP8BW_WGRAD && PW == 0) stage_quad_f32(epi, lane, acc, pp);
          else stage_rows_f32(epi, lane, &acc[8 * pp]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            emit_f32(&tmD, smem_u32(epi), col0 + 16 * pp, drow, a.out_mode);
            bulk_commit();
          }
        }
      } else {
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        uint8_t* epi = epi0 + (p % C::kEpiBufs) * kEpiPiece;
        // the store that last used this staging piece has read it
        if (lane == 0) {
          bulk_wait_read<C::kEpiBufs - 1>();
        }
        __syncwarp();
        if (KIND == FP8BW_WGRAD && PW == 0) {
          // rows 8i + lane/4, columns 8c + 2(lane%4) + {0, 1} of the piece:
          // one bf16 pair per store; the 64-byte swizzle keeps the 32 lanes
          // of each store on 32 distinct banks
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int row = 8 * i + (lane >> 2);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const float2 v2 = acc[16 * i + 4 * p + c];
              *reinterpret_cast<uint32_t*>(epi + row * 64 + 16 * (c ^ ((row >> 1) & 3)) + 4 * (lane & 3)) =
                  pack_bf16x2(v2.x, v2.y);
            }
          }
        } else {
          // row `lane` of the piece: 64 bytes = 4 chunks, 64-byte swizzle
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint4 o;
            o.x = pack_bf16x2(acc[p * 16 + 4 * c + 0].x, acc[p * 16 + 4 * c + 0].y);
            o.y = pack_bf16x2(acc[p * 16 + 4 * c + 1].x, acc[p * 16 + 4 * c + 1].y);
            o.z = pack_bf16x2(acc[p * 16 + 4 * c + 2].x, acc[p * 16 + 4 * c + 2].y);
            o.w = pack_bf16x2(acc[p * 16 + 4 * c + 3].x, acc[p * 16 + 4 * c + 3].y);
            *reinterpret_cast<uint4*>(epi + lane * 64 + 16 * (c ^ ((lane >> 1) & 3))) = o;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmD, smem_u32(epi), col0 + p * 32, drow);
          bulk_commit();
        }
      }
      }
      if (bars->abort) break;
    }
  }
done:
  if (warp >= 4 && lane == 0) bulk_wait0();  // TMA stores have finished
  tc_fence_before();
  if (PAIR) cluster_sync(); else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if (PAIR) tmem_dealloc_pair(tmem, kTmemCols);
    else tmem_dealloc(tmem, kTmemCols);
  }
}

// ----------------------------------------------- block-scaled (MX) GEMM ---
// Power-of-2 scales (FP8BW_SCALE_POW2, "Warum dies für die KI-Ökonomie
// wichtig ist": power-of-2 scale factors as an optimization) are exactly
// UE8M0 values, so the tensor core applies them itself
// (tcgen05.mma.kind::mxf8f6f4.block_scale): each 128-wide scale block is one
// UE8M0 byte replicated over its four 32-element MMA blocks, and the whole K
// loop accumulates in one TMEM accumulator with no promotion.
// Tiles as in the promotion kernel: 256x256 per CTA pair (cta_group::2).
// 384 threads per CTA:
//   warp 0      TMA producer
//   warp 1      MMA issuer (first CTA of a pair): per chunk, tcgen05.cp of
//               the chunk's scale bytes (A: the CTA's 128 rows, B: all 256
//               rows) from shared memory into a per-stage TMEM slot of each
//               CTA, then four block-scaled MMAs
//   warp 2      scale loader: fp32 scales by cp.async into a raw ring, then
//               converted to UE8M0 bytes in the tcgen05.cp layout (row r of a
//               128-row group at lane r%32, word r/32; the four bytes of a
//               word are the four 32-K blocks); a scale that is not a power
//               of two latches FP8BW_ERR_DEVICE_CHECK
//   warps 4-11  epilogue: drain the accumulator (tcgen05.ld), release it,
//               round to bf16 and TMA-store (as in the promotion kernel)
// Scales of 4 consecutive chunks share one TMEM word per row (byte j = chunk
// j of the group; the MMAs of a chunk select their byte), so one tcgen05.cp
// per matrix serves 4 chunks.
constexpr int kSfGroup = 4;                     // chunks per scale group
constexpr int kSfSlots = 2;                     // scale groups in flight
constexpr int kMxRaw = kSfGroup * kSfSlots;     // raw fp32 chunk slots
constexpr uint32_t kSfCol0 = 256;               // TMEM: accumulator [0,256), scales after
constexpr uint32_t kSfCols = 12;                // per group: A 4 columns + B 8 columns
constexpr int kMxMaxStages = 6;
constexpr int kMxEpiBufs = 2;                   // staging pieces per epilogue warp

template <bool PAIR>
struct MxCfg {
  static constexpr uint32_t kStageBytes = kATile + (PAIR ? (BN / 2) * BK : BN * BK);
  static constexpr int kStages = PAIR ? 5 : 3;  // (single-CTA tiles: not launched)
  static constexpr uint32_t kIdescM = PAIR ? 2 * BM : BM;
};

struct MxBars {
  uint64_t full[kMxMaxStages], empty[kMxMaxStages];
  uint64_t sffull[kSfSlots], sfempty[kSfSlots];
  uint64_t tfull, tempty;
  uint32_t tmem_base;
  int32_t abort;
};

struct SfSlot {
  uint32_t a[32][4];     // A rows: row i + 32b at [i][b]
  uint32_t b[2][32][4];  // B rows 0..127 and 128..255
};

template <bool PAIR>
constexpr size_t smem_mx() {
  return 1024 + size_t(MxCfg<PAIR>::kStages) * MxCfg<PAIR>::kStageBytes + 8 * kMxEpiBufs * kEpiPiece +
         size_t(kMxRaw) * sizeof(ScaleSlot) + size_t(kSfSlots) * sizeof(SfSlot) +
         sizeof(MxBars) + 2 * sizeof(int32_t) * (kMaxGroups + 1);
}
static_assert(smem_mx<true>() <= 232448 && smem_mx<false>() <= 232448, "shared memory budget (MX)");

// UE8M0 byte of a power-of-2 fp32 scale (2^-127 is the subnormal 0x00400000),
// replicated into the four bytes of a word.
__device__ __forceinline__ uint32_t ue8m0_x4(float s, bool& bad) {
  const uint32_t b = __float_as_uint(s);
  if ((b & 0x7FFFFFu) != 0u && b != 0x00400000u) bad = true;
  return ((b >> 23) & 0xFFu) * 0x01010101u;
}

// Builds one scale group: byte j of every word comes from chunk j of the
// group (raw slots r[0..n-1]); bytes of absent chunks hold 127 (1.0).
template <int KIND>
__device__ __forceinline__ void sf_convert(const ScaleSlot* const* r, int n, SfSlot* o, int lane,
                                           bool& bad) {
  uint32_t wa[4] = {0, 0, 0, 0}, wb[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
#pragma unroll
  for (int j = 0; j < kSfGroup; ++j) {
    const uint32_t sh = 8 * j;
    if (j < n) {
#pragma unroll
      for (int b = 0; b < 4; ++b) wa[b] |= (ue8m0_x4(r[j]->sa[lane + 32 * b], bad) & 0xFFu) << sh;
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const float v = (KIND == FP8BW_WGRAD) ? r[j]->sb[h * 128 + lane + 32 * b] : r[j]->sb[h];
          wb[h][b] |= (ue8m0_x4(v, bad) & 0xFFu) << sh;
        }
    } else {
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        wa[b] |= 127u << sh;
        wb[0][b] |= 127u << sh;
        wb[1][b] |= 127u << sh;
      }
    }
  }
  *reinterpret_cast<uint4*>(&o->a[lane][0]) = make_uint4(wa[0], wa[1], wa[2], wa[3]);
  *reinterpret_cast<uint4*>(&o->b[0][lane][0]) = make_uint4(wb[0][0], wb[0][1], wb[0][2], wb[0][3]);
  *reinterpret_cast<uint4*>(&o->b[1][lane][0]) = make_uint4(wb[1][0], wb[1][1], wb[1][2], wb[1][3]);
}

template <int KIND, bool GROUPED, bool PAIR, bool F32OUT>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm_mx(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmD, const GemmArgs a) {
  using C = MxCfg<PAIR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  uint8_t* stage_base = smem;
  uint8_t* epi_base = smem + C::kStages * C::kStageBytes;
  ScaleSlot* raw = reinterpret_cast<ScaleSlot*>(epi_base + 8 * kMxEpiBufs * kEpiPiece);
  SfSlot* sf = reinterpret_cast<SfSlot*>(raw + kMxRaw);
  MxBars* bars = reinterpret_cast<MxBars*>(sf + kSfSlots);
  int32_t* s_off = reinterpret_cast<int32_t*>(bars + 1);
  int32_t* s_pp = s_off + (kMaxGroups + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0;
  const bool leader = rank == 0;
  const int cta_slot = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int cta_step = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  int ghint = 0;  // expert of this thread's previous tile (grouped fprop/dgrad)

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(smem_u32(&bars->full[i]), 1);
      mbar_init(smem_u32(&bars->empty[i]), 1);
    }
    for (int i = 0; i < kSfSlots; ++i) {
      mbar_init(smem_u32(&bars->sffull[i]), PAIR ? 2 : 1);
      mbar_init(smem_u32(&bars->sfempty[i]), 1);
    }
    mbar_init(smem_u32(&bars->tfull), 1);
    mbar_init(smem_u32(&bars->tempty), PAIR ? 16 : 8);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    if (PAIR) {
      tmem_alloc_pair(smem_u32(&bars->tmem_base), kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
      tmem_relinquish();
    }
  }
  if (GROUPED) {
    for (int i = threadIdx.x; i <= a.G; i += kThreads) s_off[i] = a.offsets[i];
  }
  tc_fence_before();
  if (PAIR) cluster_sync(); else __syncthreads();
  tc_fence_after();
  if (GROUPED) {
    int bad = 0;
    for (int i = threadIdx.x; i < a.G; i += kThreads) {
      const int o0 = s_off[i], o1 = s_off[i + 1];
      if (o1 < o0 || (o1 & 127) || (i == 0 && o0 != 0)) bad = 1;
    }
    if (threadIdx.x == 0) {
      const int mtot = (KIND == FP8BW_WGRAD) ? a.K : a.M;
      if (s_off[a.G] > mtot || s_off[a.G] < 0) bad = 1;
    }
    if (__syncthreads_or(bad)) {
      if (threadIdx.x == 0) atomicOr(&g_gemm_error, DEV_ERR_CHECK);
      tc_fence_before();
      if (PAIR) cluster_sync();
      if (warp == 1) {
        if (PAIR) tmem_dealloc_pair(bars->tmem_base, kTmemCols);
        else tmem_dealloc(bars->tmem_base, kTmemCols);
      }
      return;
    }
    if (KIND != FP8BW_WGRAD && PAIR) pair_prefix(s_off, s_pp, a.G);
  }
  const uint32_t tmem = bars->tmem_base;
  // Barriers the MMA waits on live in the first CTA of a pair.
  const uint32_t full0 = PAIR ? mapa_shared(smem_u32(&bars->full[0]), 0) : smem_u32(&bars->full[0]);
  const uint32_t sffull0 = PAIR ? mapa_shared(smem_u32(&bars->sffull[0]), 0) : smem_u32(&bars->sffull[0]);
  const uint32_t tempty0 = PAIR ? mapa_shared(smem_u32(&bars->tempty), 0) : smem_u32(&bars->tempty);

  if (warp < 4) {
    regs_dec<kRegsLow>();
    if (warp == 0) {
      // ------------------------------------------------ TMA producer ----
      if (lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
      }
      int stage = 0, chunk = 0;
      uint32_t phase = 0;
      for (int t = cta_slot; t < a.tiles; t += cta_step) {
        const TileInfo ti = decode_tile<KIND, GROUPED, PAIR, KIND != FP8BW_WGRAD>(a, t, s_off, s_pp, ghint);
        if (ti.skip) continue;
        const int arow = ti.m0 + (PAIR ? (int)rank * BM : 0);
        const int brow = PAIR ? ti.nt * BN + (int)rank * (BN / 2) : ti.nt * BN;
        for (int kb = ti.kb0; kb < ti.kb1; ++kb, ++chunk) {
          if (!mbar_wait(smem_u32(&bars->empty[stage]), phase ^ 1)) {
            raise_timeout_mx(bars);
            goto done;
          }
          if (lane == 0 && !(blockIdx.x == 0 && chunk == a.stall_chunk)) {
            const uint32_t full = full0 + stage * 8;
            const uint32_t sa = smem_u32(stage_base + stage * C::kStageBytes);
            if (PAIR) {
              if (leader) mbar_arrive_expect_tx(smem_u32(&bars->full[stage]), 2 * C::kStageBytes);
              tma_load_2d_pair(sa, &tmA, full, kb * BK, arow);
              if (GROUPED && KIND != FP8BW_WGRAD)
                tma_load_3d_pair(sa + kATile, &tmB, full, kb * BK, brow, ti.g);
              else
                tma_load_2d_pair(sa + kATile, &tmB, full, kb * BK, brow);
            } else {
              mbar_arrive_expect_tx(full, C::kStageBytes);
              tma_load_2d(sa, &tmA, full, kb * BK, arow);
              if (GROUPED && KIND != FP8BW_WGRAD)
                tma_load_3d(sa + kATile, &tmB, full, kb * BK, brow, ti.g);
              else
                tma_load_2d(sa + kATile, &tmB, full, kb * BK, brow);
            }
          }
          __syncwarp();
          if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        }
        if (bars->abort) break;
      }
    } else if (warp == 1) {
      // ------------------------------------------------- MMA issuer -----
      if (leader && lane == 0) {
        int stage = 0, gslot = 0;
        uint32_t phase = 0, tphase = 0, gphase = 0;
        for (int t = cta_slot; t < a.tiles; t += cta_step) {
          const TileInfo ti = decode_tile<KIND, GROUPED, PAIR>(a, t, s_off, s_pp, ghint);
          if (ti.skip || ti.kb0 == ti.kb1) continue;
          if (!mbar_wait(smem_u32(&bars->tempty), tphase ^ 1)) {
            raise_timeout_mx(bars);
            goto done;
          }
          tc_fence_after();
          for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
            const int i = kb - ti.kb0, j = i % kSfGroup;
            const uint32_t tsf = tmem + kSfCol0 + gslot * kSfCols;
            if (j == 0) {
              if (!mbar_wait(smem_u32(&bars->sffull[gslot]), gphase)) {
                raise_timeout_mx(bars);
                goto done;
              }
              tc_fence_after();
              const uint64_t sda = sdesc_k_noswz_16B(smem_u32(&sf[gslot].a[0][0]));
              const uint64_t sdb0 = sdesc_k_noswz_16B(smem_u32(&sf[gslot].b[0][0][0]));
              const uint64_t sdb1 = sdesc_k_noswz_16B(smem_u32(&sf[gslot].b[1][0][0]));
              if (PAIR) {
                tmem_cp_32x128b_x4_pair(tsf, sda);
                tmem_cp_32x128b_x4_pair(tsf + 4, sdb0);
                tmem_cp_32x128b_x4_pair(tsf + 8, sdb1);
              } else {
                tmem_cp_32x128b_x4(tsf, sda);
                tmem_cp_32x128b_x4(tsf + 4, sdb0);
                tmem_cp_32x128b_x4(tsf + 8, sdb1);
              }
            }
            if (!mbar_wait(smem_u32(&bars->full[stage]), phase)) {
              raise_timeout_mx(bars);
              goto done;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(stage_base + stage * C::kStageBytes);
            const uint64_t da = sdesc_k_sw128(sa), db = sdesc_k_sw128(sa + kATile);
#pragma unroll
            for (int kk = 0; kk < BK / 32; ++kk) {
              const uint32_t acc = (kb > ti.kb0 || kk > 0) ? 1u : 0u;
              if (PAIR)
                umma_mx_pair(tmem, da + 2 * kk, db + 2 * kk, idesc_mx(C::kIdescM, BN, j) | a.fmt_bits, tsf, tsf + 4, acc);
              else
                umma_mx(tmem, da + 2 * kk, db + 2 * kk, idesc_mx(C::kIdescM, BN, j) | a.fmt_bits, tsf, tsf + 4, acc);
            }
            if (PAIR) umma_commit_pair(smem_u32(&bars->empty[stage]), 0x3);
            else umma_commit(smem_u32(&bars->empty[stage]));
            if (++stage == C::kStages) { stage = 0; phase ^= 1; }
            if (j == kSfGroup - 1 || kb + 1 == ti.kb1) {
              // the group's scales may be replaced once these MMAs are done
              if (PAIR) umma_commit_pair(smem_u32(&bars->sfempty[gslot]), 0x3);
              else umma_commit(smem_u32(&bars->sfempty[gslot]));
              if (++gslot == kSfSlots) { gslot = 0; gphase ^= 1; }
            }
          }
          if (PAIR) umma_commit_pair(smem_u32(&bars->tfull), 0x3);
          else umma_commit(smem_u32(&bars->tfull));
          tphase ^= 1;
          if (bars->abort) break;
        }
      }
    } else if (warp == 2) {
      // ------------------------------------------------ scale loader ----
      // Per scale group (up to 4 chunks of one tile): the chunks' fp32 scales
      // go to raw slots by cp.async as one copy group; the previous group is
      // converted once its copies have landed and its SF slot is free.
      const int nKb = a.K / BK, nNb = a.N / 128;
      int rbase = 0, gslot = 0, pend_n = 0, pend_base = 0;
      uint32_t gphase = 0;
      bool bad = false, pend = false;
      for (int t = cta_slot;; t += cta_step) {
        const bool have = t < a.tiles;
        TileInfo ti = {};
        if (have) {
          ti = decode_tile<KIND, GROUPED, PAIR, KIND != FP8BW_WGRAD>(a, t, s_off, s_pp, ghint);
          if (ti.skip) continue;
        }
        const int row0 = ti.m0 + (PAIR ? (int)rank * BM : 0);
        const float* sBg = a.sB;
        if (GROUPED && KIND != FP8BW_WGRAD) sBg += (size_t)ti.g * nNb * nKb;
        for (int kg = ti.kb0; have ? kg < ti.kb1 : pend; kg += kSfGroup) {
          int n = 0;
          if (have) {
            n = min(kSfGroup, ti.kb1 - kg);
            for (int j = 0; j < n; ++j) {
              const int kb = kg + j;
              ScaleSlot* sl = &raw[(rbase + j) % kMxRaw];
              if (row0 < a.M)
                cp_async_16(smem_u32(&sl->sa[lane * 4]), a.sA + (size_t)kb * a.M + row0 + lane * 4);
              else
                *reinterpret_cast<float4*>(&sl->sa[lane * 4]) = make_float4(1.f, 1.f, 1.f, 1.f);
              if (KIND == FP8BW_WGRAD) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                  const int nn = ti.nt * BN + h * 128 + lane * 4;
                  if (nn < a.N) cp_async_16(smem_u32(&sl->sb[h * 128 + lane * 4]), sBg + (size_t)kb * a.N + nn);
                  else *reinterpret_cast<float4*>(&sl->sb[h * 128 + lane * 4]) = make_float4(1.f, 1.f, 1.f, 1.f);
                }
              } else if (lane < 2) {
                const int nb = ti.nt * 2 + lane;
                if (nb < nNb)
                  cp_async_4(smem_u32(&sl->sb[lane]), (KIND == FP8BW_FPROP) ? sBg + (size_t)nb * nKb + kb
                                                                            : sBg + (size_t)kb * nNb + nb);
                else
                  sl->sb[lane] = 1.f;
              }
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
            asm volatile("cp.async.wait_group 1;" ::: "memory");  // the previous group has landed
          } else {
            asm volatile("cp.async.wait_all;" ::: "memory");
          }
          __syncwarp();
          if (pend) {
            if (!mbar_wait(smem_u32(&bars->sfempty[gslot]), gphase ^ 1)) {
              raise_timeout_mx(bars);
              goto done;
            }
            const ScaleSlot* r[kSfGroup];
#pragma unroll
            for (int j = 0; j < kSfGroup; ++j) r[j] = &raw[(pend_base + j) % kMxRaw];
            sf_convert<KIND>(r, pend_n, &sf[gslot], lane, bad);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (PAIR && !leader) mbar_arrive_cluster(sffull0 + gslot * 8);
              else mbar_arrive(smem_u32(&bars->sffull[gslot]));
            }
            if (++gslot == kSfSlots) { gslot = 0; gphase ^= 1; }
          }
          pend = have;
          pend_n = n;
          pend_base = rbase;
          rbase = (rbase + kSfGroup) % kMxRaw;
          if (!have) break;
        }
        if (!have || bars->abort) break;
      }
      if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&g_gemm_error, DEV_ERR_CHECK);
    }
  } else {
    regs_inc<kRegsHigh>();
    // -------------------------------------------------------- epilogue ---
    const int q = warp & 3, half = (warp - 4) >> 2;
    uint8_t* epi0 = epi_base + (warp - 4) * kMxEpiBufs * kEpiPiece;
    uint32_t tphase = 0;
    for (int t = cta_slot; t < a.tiles; t += cta_step) {
      const TileInfo ti = decode_tile<KIND, GROUPED, PAIR, KIND != FP8BW_WGRAD>(a, t, s_off, s_pp, ghint);
      if (ti.skip) continue;
      const int row0 = ti.m0 + (PAIR ? (int)rank * BM : 0);
      const int col0 = ti.nt * BN + half * 128;
      float2 acc[64];
      if (ti.kb0 == ti.kb1) {
#pragma unroll
        for (int j = 0; j < 64; ++j) acc[j] = make_float2(0.f, 0.f);
      } else {
        if (!mbar_wait(smem_u32(&bars->tfull), tphase)) {
          raise_timeout_mx(bars);
          goto done;
        }
        tc_fence_after();
        const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + half * 128;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t r[2][32];
          tmem_ld64(taddr + h2 * 64, r[0], r[1]);
          tmem_wait_ld();
#pragma unroll
          for (int p2 = 0; p2 < 2; ++p2)
#pragma unroll
            for (int j = 0; j < 16; ++j)
              acc[(h2 * 2 + p2) * 16 + j] =
                  make_float2(__uint_as_float(r[p2][2 * j]), __uint_as_float(r[p2][2 * j + 1]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (PAIR && !leader) mbar_arrive_cluster(tempty0);
          else mbar_arrive(smem_u32(&bars->tempty));
        }
        tphase ^= 1;
      }
      const int drow = (GROUPED && KIND == FP8BW_WGRAD ? ti.g * a.M : 0) + row0 + q * 32;
      if (F32OUT) {
#pragma unroll
        for (int pp = 0; pp < 8 && row0 < ti.mend; ++pp) {
          uint8_t* epi = epi0 + (pp % kMxEpiBufs) * kEpiPiece;
          if (lane == 0) bulk_wait_read<kMxEpiBufs - 1>();
          __syncwarp();
          stage_rows_f32(epi, lane, &acc[8 * pp]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            emit_f32(&tmD, smem_u32(epi), col0 + 16 * pp, drow, a.out_mode);
            bulk_commit();
          }
        }
        if (bars->abort) break;
        continue;
      }
#pragma unroll
      for (int p = 0; p < 4 && row0 < ti.mend; ++p) {
        uint8_t* epi = epi0 + (p % kMxEpiBufs) * kEpiPiece;
        if (lane == 0) bulk_wait_read<kMxEpiBufs - 1>();
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint4 o;
          o.x = pack_bf16x2(acc[p * 16 + 4 * c + 0].x, acc[p * 16 + 4 * c + 0].y);
          o.y = pack_bf16x2(acc[p * 16 + 4 * c + 1].x, acc[p * 16 + 4 * c + 1].y);
          o.z = pack_bf16x2(acc[p * 16 + 4 * c + 2].x, acc[p * 16 + 4 * c + 2].y);
          o.w = pack_bf16x2(acc[p * 16 + 4 * c + 3].x, acc[p * 16 + 4 * c + 3].y);
          *reinterpret_cast<uint4*>(epi + lane * 64 + 16 * (c ^ ((lane >> 1) & 3))) = o;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmD, smem_u32(epi), col0 + p * 32, drow);
          bulk_commit();
        }
      }
      if (bars->abort) break;
    }
  }
done:
  if (warp >= 4 && lane == 0) bulk_wait0();
  tc_fence_before();
  if (PAIR) cluster_sync(); else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if (PAIR) tmem_dealloc_pair(tmem, kTmemCols);
    else tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------ BF16 GEMM ---
// The BF16 comparison GEMM on the same CTA-pair tiles as the FP8 kernels
// (256x256 per pair, tcgen05.mma.cta_group::2.kind::f16, K = 16 per
// instruction): BK = 64 bf16 (128-byte rows) per stage, four MMAs per stage,
// the accumulator stays in TMEM for the whole K loop, double-buffered across
// tiles (2 x 256 columns), and 8 epilogue warps drain a finished tile (bf16,
// 32x32 pieces through shared memory, TMA stores) while the next one
// accumulates.
constexpr int BK16 = 64;
constexpr int kBf16Stages = 5;
constexpr uint32_t kBf16StageBytes = BM * BK16 * 2 + (BN / 2) * BK16 * 2;  // A 128x64 + B half 128x64 bf16
constexpr int kBf16EpiBufs = 2;
constexpr uint32_t kIdescBF16Pair = idesc_make(1, 1, 2 * BM, BN);         // BF16 x BF16 -> F32, M = 256

struct Bf16Bars {
  uint64_t full[kBf16Stages], empty[kBf16Stages];
  uint64_t tfull[2], tempty[2];
  uint32_t tmem_base;
  int32_t abort;
};

constexpr size_t smem_bf16() {
  return 1024 + size_t(kBf16Stages) * kBf16StageBytes + 8 * kBf16EpiBufs * kEpiPiece + sizeof(Bf16Bars);
}
static_assert(smem_bf16() <= 232448, "shared memory budget (BF16)");

__global__ void __launch_bounds__(kThreads, 1)
    k_gemm_bf16(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmD, const GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  uint8_t* stage_base = smem;
  uint8_t* epi_base = smem + kBf16Stages * kBf16StageBytes;
  Bf16Bars* bars = reinterpret_cast<Bf16Bars*>(epi_base + 8 * kBf16EpiBufs * kEpiPiece);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cta_slot = (int)(blockIdx.x >> 1), cta_step = (int)(gridDim.x >> 1);
  int ghint = 0;  // unused by dense tiles
  const int nkb = a.K / BK16;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kBf16Stages; ++i) {
      mbar_init(smem_u32(&bars->full[i]), 1);
      mbar_init(smem_u32(&bars->empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars->tfull[i]), 1);
      mbar_init(smem_u32(&bars->tempty[i]), 16);
    }
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(&bars->tmem_base), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint32_t full0 = mapa_shared(smem_u32(&bars->full[0]), 0);
  const uint32_t tempty0 = mapa_shared(smem_u32(&bars->tempty[0]), 0);

  if (warp < 4) {
    regs_dec<kRegsLow>();
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------ TMA producer ----
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB);
      int stage = 0;
      uint32_t phase = 0;
      for (int t = cta_slot; t < a.tiles; t += cta_step) {
        const TileInfo ti = decode_tile<FP8BW_FPROP, false, true>(a, t, nullptr, nullptr, ghint);
        const int arow = ti.m0 + (int)rank * BM, brow = ti.nt * BN + (int)rank * (BN / 2);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(smem_u32(&bars->empty[stage]), phase ^ 1)) {
            raise_timeout_mx(bars);
            goto done;
          }
          const uint32_t sa = smem_u32(stage_base + stage * kBf16StageBytes);
          if (leader) mbar_arrive_expect_tx(smem_u32(&bars->full[stage]), 2 * kBf16StageBytes);
          tma_load_2d_pair(sa, &tmA, full0 + stage * 8, kb * BK16, arow);
          tma_load_2d_pair(sa + BM * BK16 * 2, &tmB, full0 + stage * 8, kb * BK16, brow);
          if (++stage == kBf16Stages) { stage = 0; phase ^= 1; }
        }
        if (bars->abort) break;
      }
    } else if (warp == 1 && leader && lane == 0) {
      // ------------------------------------------------- MMA issuer -----
      int stage = 0, buf = 0;
      uint32_t phase = 0, bphase = 0;
      for (int t = cta_slot; t < a.tiles; t += cta_step) {
        if (!mbar_wait(smem_u32(&bars->tempty[buf]), bphase ^ 1)) {
          raise_timeout_mx(bars);
          goto done;
        }
        tc_fence_after();
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(smem_u32(&bars->full[stage]), phase)) {
            raise_timeout_mx(bars);
            goto done;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(stage_base + stage * kBf16StageBytes);
          const uint64_t da = sdesc_k_sw128(sa), db = sdesc_k_sw128(sa + BM * BK16 * 2);
#pragma unroll
          for (int kk = 0; kk < BK16 / 16; ++kk)  // +32 bytes = +2 in the >>4 address field
            umma_f16_pair(tmem + buf * BN, da + 2 * kk, db + 2 * kk, kIdescBF16Pair,
                          (kb > 0 || kk > 0) ? 1u : 0u);
          umma_commit_pair(smem_u32(&bars->empty[stage]), 0x3);
          if (++stage == kBf16Stages) { stage = 0; phase ^= 1; }
        }
        umma_commit_pair(smem_u32(&bars->tfull[buf]), 0x3);
        if (++buf == 2) { buf = 0; bphase ^= 1; }
        if (bars->abort) break;
      }
    }
  } else {
    regs_inc<kRegsHigh>();
    // -------------------------------------------------------- epilogue ---
    const int q = warp & 3, half = (warp - 4) >> 2;
    uint8_t* epi0 = epi_base + (warp - 4) * kBf16EpiBufs * kEpiPiece;
    int buf = 0;
    uint32_t bphase = 0;
    for (int t = cta_slot; t < a.tiles; t += cta_step) {
      const TileInfo ti = decode_tile<FP8BW_FPROP, false, true>(a, t, nullptr, nullptr, ghint);
      if (!mbar_wait(smem_u32(&bars->tfull[buf]), bphase)) {
        raise_timeout_mx(bars);
        goto done;
      }
      tc_fence_after();
      const int row0 = ti.m0 + (int)rank * BM;
      const int col0 = ti.nt * BN + half * 128;
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + buf * BN + half * 128;
      const int drow = row0 + q * 32;
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        uint32_t r[32];
        tmem_ld32(taddr + p * 32, r);
        tmem_wait_ld();
        tmem_fence_regs(r);
        if (p == 3) {
          // the whole accumulator is in registers: the next tile may start
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (!leader) mbar_arrive_cluster(tempty0 + buf * 8);
            else mbar_arrive(smem_u32(&bars->tempty[buf]));
          }
        }
        uint8_t* epi = epi0 + (p % kBf16EpiBufs) * kEpiPiece;
        if (lane == 0) bulk_wait_read<kBf16EpiBufs - 1>();
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint4 o;
          o.x = pack_bf16x2(__uint_as_float(r[8 * c + 0]), __uint_as_float(r[8 * c + 1]));
          o.y = pack_bf16x2(__uint_as_float(r[8 * c + 2]), __uint_as_float(r[8 * c + 3]));
          o.z = pack_bf16x2(__uint_as_float(r[8 * c + 4]), __uint_as_float(r[8 * c + 5]));
          o.w = pack_bf16x2(__uint_as_float(r[8 * c + 6]), __uint_as_float(r[8 * c + 7]));
          *reinterpret_cast<uint4*>(epi + lane * 64 + 16 * (c ^ ((lane >> 1) & 3))) = o;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmD, smem_u32(epi), col0 + p * 32, drow);
          bulk_commit();
        }
      }
      if (++buf == 2) { buf = 0; bphase ^= 1; }
      if (bars->abort) break;
    }
  }
done:
  if (warp >= 4 && lane == 0) bulk_wait0();
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// -------------------------------------------------------------- host ------
template <typename K>
cudaError_t prepare(K kernel, size_t smem, bool check_regs) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (!check_regs) return cudaSuccess;
  cudaFuncAttributes attr;
  e = cudaFuncGetAttributes(&attr, kernel);
  if (e != cudaSuccess) return e;
  // setmaxnreg draws on the launch allocation: refuse to launch if the
  // compiled register count could not cover the split.
  if (attr.numRegs < kRegsLaunch) return cudaErrorInvalidConfiguration;
  return cudaSuccess;
}

template <int KIND, bool GROUPED, bool PAIR, int OUTK = OK_BF16>
cudaError_t launch_one(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& td,
                       const GemmArgs& a, int grid, cudaStream_t st) {
  auto kern = k_gemm_fp8<KIND, GROUPED, PAIR, OUTK>;
  const size_t smem = smem_fp8<PAIR, OUTK == OK_QUANT_FP32 || OUTK == OK_QUANT_POW2>();
  cudaError_t e = prepare(kern, smem, true);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  if (PAIR) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, kern, ta, tb, td, a);
}

template <int KIND, bool GROUPED, bool PAIR, bool F32OUT = false>
cudaError_t launch_mx(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& td,
                      const GemmArgs& a, int grid, cudaStream_t st) {
  auto kern = k_gemm_mx<KIND, GROUPED, PAIR, F32OUT>;
  const size_t smem = smem_mx<PAIR>();
  cudaError_t e = prepare(kern, smem, true);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  if (PAIR) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, kern, ta, tb, td, a);
}

}  // namespace

int gemm_band_rows = 16;
int gemm_stall_chunk = -1;  // testing hook, consumed by the next FP8 GEMM launch

cudaError_t launch_gemm_fp8(int kind, bool grouped, int G, const int32_t* d_off, int64_t M, int64_t N,
                            int64_t K, const uint8_t* A, const float* sA, const uint8_t* B,
                            const float* sB, void* D, int64_t ldd, int mode, int num_sms,
                            cudaStream_t st, int out_mode, int a_fmt, int b_fmt) {
  // CTA pairs everywhere; grouped fprop/dgrad pair tiles stay inside one
  // expert, so their number is only bounded here (sum of ceil(rows_g/256)
  // <= (M/128 + G)/2) and the kernel skips the tiles past the real count.
  const bool pair = true;
  GemmArgs a = {};
  a.M = (int)M;
  a.N = (int)N;
  a.K = (int)K;
  if (grouped && kind != FP8BW_WGRAD) a.m_tiles = (int)((M / BM + G + 1) / 2);
  else a.m_tiles = (int)((M + 2 * BM - 1) / (2 * BM));
  a.n_tiles = (int)((N + BN - 1) / BN);
  a.band = pair ? (gemm_band_rows + 1) / 2 : gemm_band_rows;
  a.sA = sA;
  a.sB = sB;
  a.offsets = d_off;
  a.G = G;
  a.stall_chunk = gemm_stall_chunk;
  a.out_mode = out_mode;
  a.fmt_bits = idesc_fmt_bits((uint32_t)a_fmt, (uint32_t)b_fmt);
  gemm_stall_chunk = -1;
  if (grouped && kind == FP8BW_WGRAD) a.tiles = G * a.m_tiles * a.n_tiles;
  else a.tiles = a.m_tiles * a.n_tiles;
  if (a.tiles == 0) return cudaSuccess;
  CUtensorMap ta, tb, td;
  if (!make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, A, K, M, K, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const bool b3 = grouped && kind != FP8BW_WGRAD;
  if (!make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, B, K, N, K, BK, pair ? BN / 2 : BN,
                CU_TENSOR_MAP_SWIZZLE_128B, b3 ? (uint64_t)G : 0))
    return cudaErrorInvalidValue;
  const uint64_t drows = (grouped && kind == FP8BW_WGRAD) ? (uint64_t)G * M : (uint64_t)M;
  const bool f32 = out_mode != OUT_BF16;
  if (!make_map(&td, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                f32 ? 4 : 2, D, N, drows, ldd, f32 ? 16 : 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  int grid;
  cudaError_t e;
  if (pair) {
    const int clusters = num_sms / 2;
    grid = 2 * (a.tiles < clusters ? a.tiles : clusters);
  } else {
    grid = a.tiles < num_sms ? a.tiles : num_sms;
  }
  if (f32) {  // fp32 output: dense GEMMs and grouped wgrad
    if (grouped && kind != FP8BW_WGRAD) return cudaErrorInvalidValue;
    if (grouped) {
      if (mode == FP8BW_SCALE_POW2) e = launch_mx<FP8BW_WGRAD, true, true, true>(ta, tb, td, a, grid, st);
      else e = launch_one<FP8BW_WGRAD, true, true, OK_F32>(ta, tb, td, a, grid, st);
    } else if (mode == FP8BW_SCALE_POW2) {
      if (kind == FP8BW_FPROP) e = launch_mx<FP8BW_FPROP, false, true, true>(ta, tb, td, a, grid, st);
      else if (kind == FP8BW_DGRAD) e = launch_mx<FP8BW_DGRAD, false, true, true>(ta, tb, td, a, grid, st);
      else e = launch_mx<FP8BW_WGRAD, false, true, true>(ta, tb, td, a, grid, st);
    } else {
      if (kind == FP8BW_FPROP) e = launch_one<FP8BW_FPROP, false, true, OK_F32>(ta, tb, td, a, grid, st);
      else if (kind == FP8BW_DGRAD) e = launch_one<FP8BW_DGRAD, false, true, OK_F32>(ta, tb, td, a, grid, st);
      else e = launch_one<FP8BW_WGRAD, false, true, OK_F32>(ta, tb, td, a, grid, st);
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  if (mode == FP8BW_SCALE_POW2) {
    if (!grouped) {
      if (kind == FP8BW_FPROP) e = launch_mx<FP8BW_FPROP, false, true>(ta, tb, td, a, grid, st);
      else if (kind == FP8BW_DGRAD) e = launch_mx<FP8BW_DGRAD, false, true>(ta, tb, td, a, grid, st);
      else e = launch_mx<FP8BW_WGRAD, false, true>(ta, tb, td, a, grid, st);
    } else {
      if (kind == FP8BW_FPROP) e = launch_mx<FP8BW_FPROP, true, true>(ta, tb, td, a, grid, st);
      else if (kind == FP8BW_DGRAD) e = launch_mx<FP8BW_DGRAD, true, true>(ta, tb, td, a, grid, st);
      else e = launch_mx<FP8BW_WGRAD, true, true>(ta, tb, td, a, grid, st);
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  if (!grouped) {
    if (kind == FP8BW_FPROP) e = launch_one<FP8BW_FPROP, false, true>(ta, tb, td, a, grid, st);
    else if (kind == FP8BW_DGRAD) e = launch_one<FP8BW_DGRAD, false, true>(ta, tb, td, a, grid, st);
    else e = launch_one<FP8BW_WGRAD, false, true>(ta, tb, td, a, grid, st);
  } else {
    if (kind == FP8BW_FPROP) e = launch_one<FP8BW_FPROP, true, true>(ta, tb, td, a, grid, st);
    else if (kind == FP8BW_DGRAD) e = launch_one<FP8BW_DGRAD, true, true>(ta, tb, td, a, grid, st);
    else e = launch_one<FP8BW_WGRAD, true, true>(ta, tb, td, a, grid, st);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// The GEMM with the quantizing epilogue (dense, promotion kernel, any fp32
// operand scales): D = bf16(A B^T) quantized into q_row/s_row and, if q_col
// is given, the column-wise copy q_col/s_col with scale rule `qmode`; D
// itself is written only if non-null.
cudaError_t launch_gemm_quant(int kind, int64_t M, int64_t N, int64_t K, const uint8_t* A, const float* sA,
                              const uint8_t* B, const float* sB, int qmode, void* D, int64_t ldd,
                              uint8_t* q_row, float* s_row, uint8_t* q_col, float* s_col, int num_sms,
                              cudaStream_t st) {
  GemmArgs a = {};
  a.M = (int)M;
  a.N = (int)N;
  a.K = (int)K;
  a.m_tiles = (int)((M + 2 * BM - 1) / (2 * BM));
  a.n_tiles = (int)((N + BN - 1) / BN);
  a.band = (gemm_band_rows + 1) / 2;
  a.tiles = a.m_tiles * a.n_tiles;
  a.sA = sA;
  a.sB = sB;
  a.D = static_cast<uint16_t*>(D);
  a.ldd = ldd;
  a.q_row = q_row;
  a.s_row = s_row;
  a.q_col = q_col;
  a.s_col = s_col;
  a.stall_chunk = gemm_stall_chunk;
  gemm_stall_chunk = -1;
  if (a.tiles == 0) return cudaSuccess;
  CUtensorMap ta, tb, td;
  std::memset(&td, 0, sizeof td);  // no tensor-map store in this epilogue
  if (!make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, A, K, M, K, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, B, K, N, K, BK, BN / 2, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const int clusters = num_sms / 2;
  const int grid = 2 * (a.tiles < clusters ? a.tiles : clusters);
  cudaError_t e;
  if (qmode == FP8BW_SCALE_POW2) {
    if (kind == FP8BW_FPROP) e = launch_one<FP8BW_FPROP, false, true, OK_QUANT_POW2>(ta, tb, td, a, grid, st);
    else if (kind == FP8BW_DGRAD) e = launch_one<FP8BW_DGRAD, false, true, OK_QUANT_POW2>(ta, tb, td, a, grid, st);
    else e = launch_one<FP8BW_WGRAD, false, true, OK_QUANT_POW2>(ta, tb, td, a, grid, st);
  } else {
    if (kind == FP8BW_FPROP) e = launch_one<FP8BW_FPROP, false, true, OK_QUANT_FP32>(ta, tb, td, a, grid, st);
    else if (kind == FP8BW_DGRAD) e = launch_one<FP8BW_DGRAD, false, true, OK_QUANT_FP32>(ta, tb, td, a, grid, st);
    else e = launch_one<FP8BW_WGRAD, false, true, OK_QUANT_FP32>(ta, tb, td, a, grid, st);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_gemm_bf16(int64_t M, int64_t N, int64_t K, const void* A, const void* B, void* D,
                             int64_t ldd, int num_sms, cudaStream_t st) {
  GemmArgs a = {};
  a.M = (int)M;
  a.N = (int)N;
  a.K = (int)K;
  a.m_tiles = (int)((M + 2 * BM - 1) / (2 * BM));
  a.n_tiles = (int)((N + BN - 1) / BN);
  a.band = (gemm_band_rows + 1) / 2;
  a.tiles = a.m_tiles * a.n_tiles;
  if (a.tiles == 0) return cudaSuccess;
  CUtensorMap ta, tb, td;
  if (!make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, A, K, M, K, BK16, BM, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, B, K, N, K, BK16, BN / 2, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!make_map(&td, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, N, M, ldd, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  const int clusters = num_sms / 2;
  const int grid = 2 * (a.tiles < clusters ? a.tiles : clusters);
  const size_t smem = smem_bf16();
  cudaError_t e = prepare(k_gemm_bf16, smem, true);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, k_gemm_bf16, ta, tb, td, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t gemm_read_clear_error(uint32_t* out, cudaStream_t st) {
  uint32_t v = 0, z = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_gemm_error, sizeof v, 0, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess && v) e = cudaMemcpyToSymbolAsync(g_gemm_error, &z, sizeof z, 0, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  *out = v;
  return e;
}

}  // namespace fp8bw

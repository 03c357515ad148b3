// FP8 attention forward for sm_100a: E4M3 Q, K, V with the recipe's 1x128
// blocks, softmax in fp32, P quantized to E4M3 per 128-key block, both
// contractions on tcgen05 tensor cores.
//
// Method: "NVIDIA NeMo RL erreicht 48% ..." section "Leistungsgewinne in der
// Praxis": the recipe extends FP8 from the linear layers to the KV cache and
// the attention operations.  Every FP8 operand carries one scale per 128
// elements along its contraction ("Der technische Durchbruch": 1x128 blocks
// for activations): Q and K one per token and head (head dimension 128), V
// the activation quantizer's column-wise copy (one per 128 tokens of a
// channel, codes channel-major), and the softmax numerator P one per query
// row and 128-key block, by the FP32 rule s = amax / 448.
//
// One CTA computes a 128-query block of one head over its keys (causal or
// not, inside one packed sequence; GQA: query head h reads KV head
// h / (Hq / Hkv)).  128 + 32 * kSoftWarps threads:
//   warp 0      TMA producer: the Q tile once, then per 128-key block the K
//               tile [128 keys][128] and the V tile [128 channels][128 keys]
//               into a 3-stage ring, and the block's 128 key scales and 128
//               channel scales (bulk copies) into a 4-slot ring
//   warp 1      MMA issuer (one thread): S_b = Q K_b^T into one of two TMEM
//               buffers, then O_(b-1) = P_(b-1) V_(b-1)^T into one of two
//               more, so the tensor core computes the next S while the
//               softmax warps work on the current one
//   warps 4..   softmax and correction, kNH warps per TMEM lane quarter
//               (kCols of the 128 columns each; a thread owns one query
//               row): read S_b, scale by the key and query scales, block
//               maximum (exchanged between the kNH parts of the row),
//               running maximum, p = 2^(z - m), partial row sums, P codes
//               into a shared tile in the MMA's layout; then fold O_(b-1)
//               into the fp32 output accumulator, kept in TMEM:
//               O = O * 2^(m_old - m_new) + s_P * s_V[channel] * O_(b-1).
// At the end O / l is rounded to bf16 and stored; padding query rows get 0.
// TMEM: S buffers at columns 0 and 128, the P.V product at 256, the output
// accumulator at 384.  Every wait is bounded; a timeout latches an error bit
// and the CTA leaves.  With power-of-2 scales the tensor core applies every
// scale (k_attn_fwd_mx).  When Hq / Hkv is even a CTA takes two query heads
// of one KV group instead (k_attn_fwd2, k_attn_fwd_mx2), so that one head's
// exponentials overlap the other head's remaining softmax phases.

#include "common.cuh"
#include "tmap.cuh"

namespace fp8bw {

__device__ uint32_t g_attn_error;

namespace {

constexpr int kD = 128;              // head dimension (one 1x128 block)
#ifndef FP8BW_ATTN_WARPS_PER_QUARTER
#define FP8BW_ATTN_WARPS_PER_QUARTER 2
#endif
// Softmax warps per TMEM lane quarter: each owns kCols of a row's 128
// columns.  All warps of a quarter run on one scheduler (TMEM lane quarter =
// warp index mod 4).  Four per quarter (640 threads, 112 registers) is
// correct but slower on B200 (570 against 617 TFLOP/s on the packed 32K
// batch): every block's maximum then waits for the slowest of four warps.
constexpr int kNH = FP8BW_ATTN_WARPS_PER_QUARTER;
static_assert(kNH == 2 || kNH == 4, "2 or 4 softmax warps per lane quarter");
constexpr int kCols = 128 / kNH;                 // columns per softmax thread
constexpr int kSoftWarps = 4 * kNH;
constexpr int kThreads = 128 + 32 * kSoftWarps;  // warps 0-3 + the softmax warps
constexpr int kStages = 3;           // K/V ring
constexpr int kScSlots = 4;          // scale ring
constexpr uint32_t kTile = 128 * 128;  // one 128x128 E4M3 tile
constexpr uint32_t kIdesc = idesc_make(0, 0, 128, 128);  // E4M3 x E4M3 -> F32, M = N = 128
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLog2_448 = 8.807354922057604f;   // log2(448)
// setmaxnreg split of the launch allocation (kThreads x kRegsLaunch, checked
// on the host before the launch): kRegsLow for warps 0-3, kRegsHigh for the
// softmax warps.  2 per quarter: 56*128 + 224*256 = 64512 <= 384*168;
// 4 per quarter: 32*128 + 112*512 = 61440 <= 640*96.
constexpr int kRegsLow = kNH == 2 ? 56 : 32;
constexpr int kRegsHigh = kNH == 2 ? 224 : 112;
constexpr int kRegsLaunch = kNH == 2 ? 168 : 96;
static_assert(kRegsLow * 128 + kRegsHigh * 32 * kSoftWarps <= kRegsLaunch * kThreads, "register split");
static_assert(kRegsLaunch * kThreads <= 65536, "launch allocation");

struct ScSlot {
  float sk[128];   // key scales of the block (one per key)
  float sv[128];   // V scales of the block (one per channel)
};

struct AttnBars {
  uint64_t q_full;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t sc_full[kScSlots], sc_empty[kScSlots];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full[2], p_empty[2];
  uint64_t o_full, o_empty;  // the single P.V product buffer
  uint64_t pair[4];          // the kNH warps of a TMEM lane quarter meet here
  uint32_t tmem_base;
  int32_t abort;
};

struct AttnSmem {
  uint8_t q[kTile];                    // 1024-aligned tiles first
  uint8_t kv[kStages][2][kTile];       // [stage][K, V^T]
  uint8_t p[2][kTile];
  ScSlot sc[kScSlots];
  float red[2][kNH][128];              // [block parity][column part][row]: block maxima
  float lsum[kNH][128];                // [column part][row]: row sums at the end
  AttnBars bars;
};

struct AttnArgs {
  int T, Hq, Hkv, nseg, causal;
  const int32_t* off;   // device [nseg + 1]
  const int32_t* len;   // device [nseg]
  const float* sq;      // [Hq][T]
  const float* sk;      // [Hkv][T]
  const float* sv;      // [T/128][Hkv*128]
  uint16_t* o;          // [T][Hq*128] bf16
};

template <class Bars>
__device__ __forceinline__ void raise_attn_timeout(Bars* b) {
  atomicOr(&g_attn_error, DEV_ERR_TIMEOUT);
  atomicExch(&b->abort, 1);
}

// A bounded wait whose outcome is the same for the whole warp (the warp's
// tcgen05.ld / st that follow must be executed by all 32 lanes together).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}

// 32 lanes x 16 consecutive 32-bit columns (thread i: row lane base + i).
__device__ __forceinline__ void tmem_ld16c(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_st16c(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
// tmem_fence_regs for 16 registers.
__device__ __forceinline__ void fence_regs16(uint32_t (&r)[16]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]),
                 "+r"(r[13]), "+r"(r[14]), "+r"(r[15]));
}

// Folds O_c (block c's P.V product in TMEM) into the output accumulator
// (TMEM columns 384..511, this thread's row and kCols columns):
// acc = acc * alpha + s_P * s_V[channel] * O_c (acc = 0 before block 0),
// then hands the product buffer and the block's scale slot back.  False if
// a wait ran out.
__device__ __forceinline__ bool fold_block(AttnSmem& sm, AttnBars* bars, uint32_t tmem, uint32_t lane_off,
                                          int col0, int lane, int c, float alpha, float sp) {
  if (!warp_wait(smem_u32(&bars->o_full), c & 1)) return false;
  tc_fence_after();
  const uint32_t tp = tmem + lane_off + 256 + col0, to = tmem + lane_off + 384 + col0;
  const float2 sp2 = make_float2(sp, sp), a2 = make_float2(alpha, alpha);
  const float4* sv4 = reinterpret_cast<const float4*>(&sm.sc[c % kScSlots].sv[col0]);
  // rounds of 16 columns
#pragma unroll
  for (int u = 0; u < kCols / 16; ++u) {
    uint32_t r[16], o[16];
    tmem_ld16c(tp + 16 * u, r);
    if (c > 0) tmem_ld16c(to + 16 * u, o);
    tmem_wait_ld();
    fence_regs16(r);
    if (c > 0) fence_regs16(o);
    if (u == kCols / 16 - 1) {
      // the product is in registers: the next P.V may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->o_empty));
    }
#pragma unroll
    for (int j4 = 0; j4 < 4; ++j4) {
      const float4 v = sv4[u * 4 + j4];
      const float2 c0 = fmul2(sp2, make_float2(v.x, v.y));
      const float2 c1 = fmul2(sp2, make_float2(v.z, v.w));
      float2 o0 = make_float2(0.f, 0.f), o1 = make_float2(0.f, 0.f);
      if (c > 0) {
        o0 = fmul2(make_float2(__uint_as_float(o[4 * j4]), __uint_as_float(o[4 * j4 + 1])), a2);
        o1 = fmul2(make_float2(__uint_as_float(o[4 * j4 + 2]), __uint_as_float(o[4 * j4 + 3])), a2);
      }
      o0 = ffma2(make_float2(__uint_as_float(r[4 * j4]), __uint_as_float(r[4 * j4 + 1])), c0, o0);
      o1 = ffma2(make_float2(__uint_as_float(r[4 * j4 + 2]), __uint_as_float(r[4 * j4 + 3])), c1, o1);
      o[4 * j4] = __float_as_uint(o0.x);
      o[4 * j4 + 1] = __float_as_uint(o0.y);
      o[4 * j4 + 2] = __float_as_uint(o1.x);
      o[4 * j4 + 3] = __float_as_uint(o1.y);
    }
    tmem_st16c(to + 16 * u, o);
  }
  tmem_wait_st();
  __syncwarp();
  if (lane == 0) mbar_arrive(smem_u32(&bars->sc_empty[c % kScSlots]));
  return true;
}

// The kNH warps of lane quarter q meet (each after writing its part's value
// to shared memory); `uses` counts this quarter's earlier meetings.  False if
// another warp did not arrive in time.
template <class Bars>
__device__ __forceinline__ bool pair_meet(Bars* bars, int q, int lane, uint32_t uses) {
  __syncwarp();
  if (lane == 0) mbar_arrive(smem_u32(&bars->pair[q]));
  return warp_wait(smem_u32(&bars->pair[q]), uses & 1);
}

// TMA producer (one thread): the NQ Q tiles (heads h .. h+NQ-1, stored one
// after another from sm.q) once, then per 128-key block the K tile [128
// keys][128] and the V tile [128 channels][128 keys] into the kStages ring,
// and the block's 128 key scales and 128 channel scales (bulk copies) into
// the kScSlots ring.
template <int NQ, class Smem, class Bars>
__device__ __forceinline__ void attn_producer(Smem& sm, Bars* bars, const CUtensorMap* tmQ,
                                              const CUtensorMap* tmK, const CUtensorMap* tmV,
                                              const AttnArgs& a, int h, int g, int q0, int kb_first, int nb) {
  prefetch_tmap(tmQ);
  prefetch_tmap(tmK);
  prefetch_tmap(tmV);
  mbar_arrive_expect_tx(smem_u32(&bars->q_full), NQ * kTile);
  uint8_t* qdst = reinterpret_cast<uint8_t*>(&sm.q);
#pragma unroll
  for (int i = 0; i < NQ; ++i)
    tma_load_2d(smem_u32(qdst + i * kTile), tmQ, smem_u32(&bars->q_full), (h + i) * kD, q0);
  for (int b = 0; b < nb; ++b) {
    const int kb = kb_first + b, s = b % kStages, sl = b % kScSlots;
    if (!mbar_wait(smem_u32(&bars->kv_empty[s]), ((b / kStages) & 1) ^ 1)) {
      raise_attn_timeout(bars);
      break;
    }
    mbar_arrive_expect_tx(smem_u32(&bars->kv_full[s]), 2 * kTile);
    tma_load_2d(smem_u32(sm.kv[s][0]), tmK, smem_u32(&bars->kv_full[s]), g * kD, kb * 128);
    tma_load_2d(smem_u32(sm.kv[s][1]), tmV, smem_u32(&bars->kv_full[s]), kb * 128, g * kD);
    if (!mbar_wait(smem_u32(&bars->sc_empty[sl]), ((b / kScSlots) & 1) ^ 1)) {
      raise_attn_timeout(bars);
      break;
    }
    mbar_arrive_expect_tx(smem_u32(&bars->sc_full[sl]), 1024);
    bulk_load(smem_u32(sm.sc[sl].sk), a.sk + (size_t)g * a.T + kb * 128, 512, smem_u32(&bars->sc_full[sl]));
    bulk_load(smem_u32(sm.sc[sl].sv), a.sv + (size_t)kb * a.Hkv * kD + g * kD, 512,
              smem_u32(&bars->sc_full[sl]));
    if (bars->abort) break;
  }
}

// The CTA's work: query block qb (heavy, late blocks launched first) of
// heads h .. h+HPC-1 (HPC query heads of one KV group), its segment and key
// blocks.  Validates the segment table (every CTA; an invalid one latches
// FP8BW_ERR_DEVICE_CHECK and nothing is written) and writes zeros for a
// query block that is all padding; done = true then.  Called by every
// thread (it synchronizes the CTA).
struct AttnBlock {
  int qb, h, g, q0, j0, jreal, kb_first, nb;
  bool done;
};

template <int NT, int HPC = 1>
__device__ __forceinline__ AttnBlock attn_block(const AttnArgs& a, int* s_seg) {
  AttnBlock w;
  const int nqb = a.T / 128, hgroups = a.Hq / HPC;
  w.qb = nqb - 1 - (int)(blockIdx.x / hgroups);
  w.h = (int)(blockIdx.x % hgroups) * HPC;
  w.g = w.h / (a.Hq / a.Hkv);
  w.q0 = w.qb * 128;
  w.done = false;
  if (threadIdx.x == 0) *s_seg = -1;
  __syncthreads();
  int bad = 0;
  for (int i = threadIdx.x; i < a.nseg; i += NT) {
    const int o0 = a.off[i], o1 = a.off[i + 1], ln = a.len[i];
    if (o1 < o0 || (o0 & 127) || (o1 & 127) || ln < 0 || ln > o1 - o0 || (i == 0 && o0 != 0)) bad = 1;
    if (o0 <= w.q0 && w.q0 < o1) *s_seg = i;   // at most one segment holds the block
  }
  if (threadIdx.x == 0 && a.off[a.nseg] > a.T) bad = 1;
  if (__syncthreads_or(bad)) {
    if (threadIdx.x == 0) atomicOr(&g_attn_error, DEV_ERR_CHECK);
    w.done = true;
    return w;
  }
  const int seg = *s_seg;                      // -1: past the last segment
  w.j0 = seg >= 0 ? a.off[seg] : w.q0;
  w.jreal = seg >= 0 ? w.j0 + a.len[seg] : w.q0;   // first padding token of the segment
  if (w.q0 >= w.jreal) {
    // the whole query block is padding: zeros
    uint16_t* orow_base = a.o + (size_t)w.h * kD;
    const size_t ostride = (size_t)a.Hq * kD;
    for (int idx = threadIdx.x; idx < HPC * 128 * 8; idx += NT) {
      const int hh = idx / (128 * 8), r = (idx >> 3) & 127, c = idx & 7;
      st_global_v8(orow_base + (size_t)(w.q0 + r) * ostride + hh * kD + c * 16, make_uint4(0, 0, 0, 0),
                   make_uint4(0, 0, 0, 0));
    }
    w.done = true;
    return w;
  }
  w.kb_first = w.j0 / 128;
  const int kb_last = a.causal ? min(w.qb, (w.jreal - 1) / 128) : (w.jreal - 1) / 128;
  w.nb = kb_last - w.kb_first + 1;
  return w;
}

__global__ void __launch_bounds__(kThreads, 1)
    k_attn_fwd(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>(smem_align1024(smem_raw));
  AttnBars* bars = &sm.bars;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  __shared__ int s_seg;
  const AttnBlock wk = attn_block<kThreads>(a, &s_seg);
  if (wk.done) return;
  const int h = wk.h, g = wk.g, q0 = wk.q0, jreal = wk.jreal;
  const int kb_first = wk.kb_first, nb = wk.nb;
  uint16_t* orow_base = a.o + (size_t)h * kD;
  const size_t ostride = (size_t)a.Hq * kD;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_u32(&bars->kv_full[i]), 1);
      mbar_init(smem_u32(&bars->kv_empty[i]), 1);
    }
    for (int i = 0; i < kScSlots; ++i) {
      mbar_init(smem_u32(&bars->sc_full[i]), 1);
      mbar_init(smem_u32(&bars->sc_empty[i]), kSoftWarps);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars->s_full[i]), 1);
      mbar_init(smem_u32(&bars->s_empty[i]), kSoftWarps);
      mbar_init(smem_u32(&bars->p_full[i]), kSoftWarps);
      mbar_init(smem_u32(&bars->p_empty[i]), 1);
    }
    mbar_init(smem_u32(&bars->o_full), 1);
    mbar_init(smem_u32(&bars->o_empty), kSoftWarps);
    for (int i = 0; i < 4; ++i) mbar_init(smem_u32(&bars->pair[i]), kNH);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp < 4) {
  regs_dec<kRegsLow>();
  if (warp == 0) {
    // ---------------------------------------------------- TMA producer ----
    if (lane == 0) attn_producer<1>(sm, bars, &tmQ, &tmK, &tmV, a, h, g, q0, kb_first, nb);
  } else if (warp == 1) {
    // ----------------------------------------------------- MMA issuer -----
    if (lane == 0) {
      bool ok = mbar_wait(smem_u32(&bars->q_full), 0);
      tc_fence_after();
      const uint64_t dq = sdesc_k_sw128(smem_u32(sm.q));
      for (int b = 0; ok && b <= nb; ++b) {
        if (b < nb) {
          const int s = b % kStages;
          if (!mbar_wait(smem_u32(&bars->kv_full[s]), (b / kStages) & 1) ||
              !mbar_wait(smem_u32(&bars->s_empty[b & 1]), ((b >> 1) & 1) ^ 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t dk = sdesc_k_sw128(smem_u32(sm.kv[s][0]));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f8f6f4(tmem + (b & 1) * 128, dq + 2 * kk, dk + 2 * kk, kIdesc, kk > 0 ? 1u : 0u);
          umma_commit(smem_u32(&bars->s_full[b & 1]));
        }
        if (b >= 1) {
          const int c = b - 1, s = c % kStages;
          if (!mbar_wait(smem_u32(&bars->p_full[c & 1]), (c >> 1) & 1) ||
              !mbar_wait(smem_u32(&bars->o_empty), (c & 1) ^ 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t dp = sdesc_k_sw128(smem_u32(sm.p[c & 1]));
          const uint64_t dv = sdesc_k_sw128(smem_u32(sm.kv[s][1]));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f8f6f4(tmem + 256, dp + 2 * kk, dv + 2 * kk, kIdesc, kk > 0 ? 1u : 0u);
          umma_commit(smem_u32(&bars->p_empty[c & 1]));
          umma_commit(smem_u32(&bars->o_full));
          umma_commit(smem_u32(&bars->kv_empty[s]));
        }
        if (bars->abort) break;
      }
      if (!ok) raise_attn_timeout(bars);
    }
  }
  } else {
    regs_inc<kRegsHigh>();
    // --------------------------------------------- softmax and correction --
    const int q = warp & 3, hf = (warp - 4) >> 2;   // lane quarter, column part
    const int i = q * 32 + lane, t = q0 + i;
    const int col0 = hf * kCols;                    // this thread's kCols columns
    const float cq = a.sq[(size_t)h * a.T + t] * (kLog2e * 0.08838834764831845f);  // sq * log2(e) / sqrt(128)
    // keys of this row: [j0, jend); a block needs a mask where it reaches jend
    const int jend = a.causal ? min(jreal, t + 1) : jreal;
    float m = -INFINITY, lh = 0.0f;
    float a_prev = 0.0f, sp_prev = 0.0f;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    bool ok = true;
    uint32_t meets = 0;
    constexpr int kU = kCols / 32;                  // 32-column TMEM loads per thread

    for (int b = 0; b < nb && ok; ++b) {
      const int kb = kb_first + b;
      if (!warp_wait(smem_u32(&bars->sc_full[b % kScSlots]), (b / kScSlots) & 1) ||
          !warp_wait(smem_u32(&bars->s_full[b & 1]), (b >> 1) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t r[kU][32];
      const uint32_t ta = tmem + lane_off + (b & 1) * 128 + col0;
#pragma unroll
      for (int u = 0; u < kU; ++u) tmem_ld32(ta + 32 * u, r[u]);
      tmem_wait_ld();
#pragma unroll
      for (int u = 0; u < kU; ++u) tmem_fence_regs(r[u]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->s_empty[b & 1]));

      // y = (q . k) * s_k per key; the query scale and 1/sqrt(d) log2(e)
      // (cq > 0) are applied after the maximum
      const int lim = jend - kb * 128 - col0;      // columns >= lim are masked
      const float4* sk4 = reinterpret_cast<const float4*>(&sm.sc[b % kScSlots].sk[col0]);
      // in place: r becomes y = s_k * (q . k), then p (as fp32 bits)
      float mh;
#pragma unroll
      for (int u = 0; u < kU; ++u) {
#pragma unroll
        for (int j4 = 0; j4 < 8; ++j4) {
          const float4 kv4 = sk4[u * 8 + j4];
          const float2 p0 = fmul2(make_float2(__uint_as_float(r[u][4 * j4]), __uint_as_float(r[u][4 * j4 + 1])),
                                  make_float2(kv4.x, kv4.y));
          const float2 p1 = fmul2(make_float2(__uint_as_float(r[u][4 * j4 + 2]), __uint_as_float(r[u][4 * j4 + 3])),
                                  make_float2(kv4.z, kv4.w));
          r[u][4 * j4] = __float_as_uint(p0.x);
          r[u][4 * j4 + 1] = __float_as_uint(p0.y);
          r[u][4 * j4 + 2] = __float_as_uint(p1.x);
          r[u][4 * j4 + 3] = __float_as_uint(p1.y);
        }
      }
      if (lim < kCols) {
#pragma unroll
        for (int j = 0; j < kCols; ++j)
          if (j >= lim) r[j >> 5][j & 31] = __float_as_uint(-INFINITY);
      }
      {
        // block maximum of the thread's kCols values: three-input maxima over
        // groups of 8, then over the groups
        float mg[kCols / 8];
#pragma unroll
        for (int g = 0; g < kCols / 8; ++g) {
          const uint32_t* v = &r[(8 * g) >> 5][(8 * g) & 31];
          mg[g] = fmax3(fmax3(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2])),
                        fmax3(__uint_as_float(v[3]), __uint_as_float(v[4]), __uint_as_float(v[5])),
                        fmaxf(__uint_as_float(v[6]), __uint_as_float(v[7])));
        }
        mh = mg[0];
#pragma unroll
        for (int g = 1; g + 1 < kCols / 8; g += 2) mh = fmax3(mh, mg[g], mg[g + 1]);
        if ((kCols / 8) % 2 == 0) mh = fmaxf(mh, mg[kCols / 8 - 1]);
      }
      // block maximum of the row: combine the kNH parts
      sm.red[b & 1][hf][i] = mh;
      if (!pair_meet(bars, q, lane, meets++)) {
        ok = false;
        break;
      }
      float mrow = sm.red[b & 1][0][i];
#pragma unroll
      for (int k = 1; k < kNH; ++k) mrow = fmaxf(mrow, sm.red[b & 1][k][i]);
      const float mb = mrow * cq;
      // The warps of a quarter share one scheduler and meet here every
      // block; the odd parts fold the previous block's product first and the
      // even parts exponentiate first, so exponentials overlap folds instead
      // of all of them waiting on the same unit.
      const bool fold_first = (hf & 1) != 0;
      if (fold_first && b >= 1 &&
          !fold_block(sm, bars, tmem, lane_off, col0, lane, b - 1, a_prev, sp_prev)) {
        ok = false;
        break;
      }
      const float m_new = fmaxf(m, mb);
      const float alpha = ex2(m - m_new);       // 0 on the first block
      m = m_new;
      // P's block scale s_P = amax / 448, amax = 2^(mb - m) the block's
      // largest p.  The code input p / s_P = 2^(y * cq - mb + log2 448) is
      // exponentiated directly (it does not depend on m), and the row sum
      // gains s_P * sum(p / s_P).  If amax underflows, s_P = 0 and the block
      // adds nothing, as its p do.
      const float amax = ex2(mb - m_new);
      const float sp = amax * (1.0f / 448.0f);
      const float2 cq2 = make_float2(cq, cq), nm2 = make_float2(kLog2_448 - mb, kLog2_448 - mb);
      float2 ps2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int j = 0; j < kCols; j += 2) {
        const int u = j >> 5, k = j & 31;
        const float2 z = ffma2(make_float2(__uint_as_float(r[u][k]), __uint_as_float(r[u][k + 1])), cq2, nm2);
        const float2 pj = make_float2(ex2(z.x), ex2(z.y));
        r[u][k] = __float_as_uint(pj.x);
        r[u][k + 1] = __float_as_uint(pj.y);
        ps2[(j >> 1) & 3] = fadd2(ps2[(j >> 1) & 3], pj);
      }
      const float2 psum = fadd2(fadd2(ps2[0], ps2[1]), fadd2(ps2[2], ps2[3]));
      lh = lh * alpha + sp * (psum.x + psum.y);
      uint32_t w[kCols / 4];
#pragma unroll
      for (int j = 0; j < kCols / 4; ++j) {
        const int u = j >> 3, k = 4 * (j & 7);
        w[j] = cvt_e4m3x2(__uint_as_float(r[u][k]), __uint_as_float(r[u][k + 1])) |
               (cvt_e4m3x2(__uint_as_float(r[u][k + 2]), __uint_as_float(r[u][k + 3])) << 16);
      }
      if (!warp_wait(smem_u32(&bars->p_empty[b & 1]), ((b >> 1) & 1) ^ 1)) {
        ok = false;
        break;
      }
      // row i of the P tile: 16-byte chunk c at c ^ (i & 7) (128-byte swizzle)
      uint8_t* prow = sm.p[b & 1] + i * 128;
#pragma unroll
      for (int c = 0; c < kCols / 16; ++c)
        *reinterpret_cast<uint4*>(prow + (((hf * (kCols / 16) + c) ^ (i & 7)) << 4)) =
            make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->p_full[b & 1]));
      if (!fold_first && b >= 1 &&
          !fold_block(sm, bars, tmem, lane_off, col0, lane, b - 1, a_prev, sp_prev))
        ok = false;
      a_prev = alpha;
      sp_prev = sp;
      if (bars->abort) ok = false;
    }
    if (ok && !fold_block(sm, bars, tmem, lane_off, col0, lane, nb - 1, a_prev, sp_prev)) ok = false;
    if (!ok) raise_attn_timeout(bars);
    // row sum of the kNH parts, then O / l in bf16 (padding rows: 0)
    sm.lsum[hf][i] = lh;
    if (!pair_meet(bars, q, lane, meets++)) ok = false;
    float l = sm.lsum[0][i];
#pragma unroll
    for (int k = 1; k < kNH; ++k) l += sm.lsum[k][i];
    const bool real = t < jreal && ok;
    const float il = real ? __fdiv_rn(1.0f, l) : 0.0f;
    uint16_t* orow = orow_base + (size_t)t * ostride + col0;
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      uint32_t o[32];
      tmem_ld32(tmem + lane_off + 384 + col0 + 32 * u, o);
      tmem_wait_ld();
      tmem_fence_regs(o);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t o8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          o8[j] = real ? pack_bf16x2(__uint_as_float(o[16 * c + 2 * j]) * il, __uint_as_float(o[16 * c + 2 * j + 1]) * il)
                       : 0u;
        st_global_v8(orow + 32 * u + 16 * c, make_uint4(o8[0], o8[1], o8[2], o8[3]),
                     make_uint4(o8[4], o8[5], o8[6], o8[7]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------
// FP32 scales, two query heads per CTA (the arrangement of k_attn_fwd_mx2
// for k_attn_fwd's numerics).  A CTA takes one 128-query block of query
// heads h, h+1 of one KV group; each head has four softmax warps (one per
// lane quarter, a thread owning a whole row), so one head's exponentials
// overlap the other's key scaling, P codes and folds.  TMEM: one S buffer
// at 0 and one P.V product buffer at 128, each taken by the two heads in
// turn; the output accumulators at 256 (head A) and 384 (head B).  Per key
// block the MMA warp computes S_A, S_B, then P_A V^T and P_B V^T of the
// previous block (P_B V^T once head A has read its product).  Launched
// when Hq / Hkv is even.
constexpr uint32_t kF2S = 0, kF2P = 128, kF2O = 256;   // O of head tl at kF2O + 128 tl

struct AttnBars2 {
  uint64_t q_full;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t sc_full[kScSlots], sc_empty[kScSlots];
  uint64_t s_full[2];              // [head]: its S is in the buffer
  uint64_t s_empty;                // the buffer's last S has been read (four warps)
  uint64_t p_full[2][2], p_empty[2][2];   // [head][slot]
  uint64_t o_full[2];              // [head]: its P.V product is in the product buffer
  uint64_t o_empty;                // the product buffer's last product has been read
  uint32_t tmem_base;
  int32_t abort;
};

struct AttnSmem2 {
  uint8_t q[2][kTile];                 // 1024-aligned tiles first
  uint8_t kv[kStages][2][kTile];
  uint8_t p[2][2][kTile];              // [head][slot]
  ScSlot sc[kScSlots];
  AttnBars2 bars;
};
static_assert(sizeof(AttnSmem2) + 1024 <= 232448, "shared memory budget (two heads, FP32 scales)");

// Folds block c's P.V product of head tl into its accumulator (this
// thread's row, all 128 columns): acc = acc * alpha + s_P * s_V[channel] *
// O_c (acc = 0 before block 0).  The product is read whole first, so the
// buffer goes back to the MMA before the arithmetic; then the block's scale
// slot is released.  `rescale` (warp-uniform) is false when every row of
// the warp has alpha = 1 (its running maximum did not move), and the
// multiply by alpha is skipped: the same result.  False if a wait ran out.
__device__ __forceinline__ bool fold_block2(AttnSmem2& sm, AttnBars2* bars, uint32_t tmem, uint32_t lane_off,
                                           int tl, int lane, int c, float alpha, float sp, bool rescale) {
  if (!warp_wait(smem_u32(&bars->o_full[tl]), c & 1)) return false;
  tc_fence_after();
  const uint32_t tp = tmem + lane_off + kF2P, to = tmem + lane_off + kF2O + 128 * tl;
  uint32_t pr[4][32];
  tmem_ld64(tp, pr[0], pr[1]);
  tmem_ld64(tp + 64, pr[2], pr[3]);
  tmem_wait_ld();
#pragma unroll
  for (int u = 0; u < 4; ++u) tmem_fence_regs(pr[u]);
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(smem_u32(&bars->o_empty));
  const float2 sp2 = make_float2(sp, sp), a2 = make_float2(alpha, alpha);
  const float4* sv4 = reinterpret_cast<const float4*>(sm.sc[c % kScSlots].sv);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    uint32_t o[32];
    if (c > 0) {
      tmem_ld32(to + 32 * u, o);
      tmem_wait_ld();
      tmem_fence_regs(o);
    }
#pragma unroll
    for (int j4 = 0; j4 < 8; ++j4) {
      const float4 v = sv4[u * 8 + j4];
      const float2 c0 = fmul2(sp2, make_float2(v.x, v.y));
      const float2 c1 = fmul2(sp2, make_float2(v.z, v.w));
      float2 o0 = make_float2(0.f, 0.f), o1 = make_float2(0.f, 0.f);
      if (c > 0) {
        o0 = make_float2(__uint_as_float(o[4 * j4]), __uint_as_float(o[4 * j4 + 1]));
        o1 = make_float2(__uint_as_float(o[4 * j4 + 2]), __uint_as_float(o[4 * j4 + 3]));
        if (rescale) {
          o0 = fmul2(o0, a2);
          o1 = fmul2(o1, a2);
        }
      }
      o0 = ffma2(make_float2(__uint_as_float(pr[u][4 * j4]), __uint_as_float(pr[u][4 * j4 + 1])), c0, o0);
      o1 = ffma2(make_float2(__uint_as_float(pr[u][4 * j4 + 2]), __uint_as_float(pr[u][4 * j4 + 3])), c1, o1);
      o[4 * j4] = __float_as_uint(o0.x);
      o[4 * j4 + 1] = __float_as_uint(o0.y);
      o[4 * j4 + 2] = __float_as_uint(o1.x);
      o[4 * j4 + 3] = __float_as_uint(o1.y);
    }
    tmem_st32(to + 32 * u, o);
  }
  tmem_wait_st();
  __syncwarp();
  if (lane == 0) mbar_arrive(smem_u32(&bars->sc_empty[c % kScSlots]));
  return true;
}

__global__ void __launch_bounds__(kThreads, 1)
    k_attn_fwd2(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const AttnArgs a) {
  static_assert(kSoftWarps == 8, "four softmax warps per head of the pair");
  extern __shared__ uint8_t smem_raw[];
  AttnSmem2& sm = *reinterpret_cast<AttnSmem2*>(smem_align1024(smem_raw));
  AttnBars2* bars = &sm.bars;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ int s_seg;
  const AttnBlock wk = attn_block<kThreads, 2>(a, &s_seg);
  if (wk.done) return;
  const int h0 = wk.h, g = wk.g, q0 = wk.q0, jreal = wk.jreal;
  const int kb_first = wk.kb_first, nb = wk.nb;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_u32(&bars->kv_full[i]), 1);
      mbar_init(smem_u32(&bars->kv_empty[i]), 1);
    }
    for (int i = 0; i < kScSlots; ++i) {
      mbar_init(smem_u32(&bars->sc_full[i]), 1);
      mbar_init(smem_u32(&bars->sc_empty[i]), kSoftWarps);   // both heads' warps
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars->s_full[i]), 1);
      mbar_init(smem_u32(&bars->o_full[i]), 1);
      for (int j = 0; j < 2; ++j) {
        mbar_init(smem_u32(&bars->p_full[i][j]), 4);
        mbar_init(smem_u32(&bars->p_empty[i][j]), 1);
      }
    }
    mbar_init(smem_u32(&bars->s_empty), 4);
    mbar_init(smem_u32(&bars->o_empty), 4);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp < 4) {
  regs_dec<kRegsLow>();
  if (warp == 0) {
    // ---------------------------------------------------- TMA producer ----
    if (lane == 0) attn_producer<2>(sm, bars, &tmQ, &tmK, &tmV, a, h0, g, q0, kb_first, nb);
  } else if (warp == 1) {
    // ----------------------------------------------------- MMA issuer -----
    if (lane == 0) {
      bool ok = mbar_wait(smem_u32(&bars->q_full), 0);
      tc_fence_after();
      const uint64_t dq0 = sdesc_k_sw128(smem_u32(sm.q[0])), dq1 = sdesc_k_sw128(smem_u32(sm.q[1]));
      uint32_t suse = 0, ouse = 0;   // S and product computations so far (each buffer alternates)
      for (int b = 0; ok && b <= nb; ++b) {
        if (b < nb) {
          const int s = b % kStages;
          if (!mbar_wait(smem_u32(&bars->kv_full[s]), (b / kStages) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t dk = sdesc_k_sw128(smem_u32(sm.kv[s][0]));
          for (int tl = 0; tl < 2 && ok; ++tl) {
            if (!mbar_wait(smem_u32(&bars->s_empty), (suse & 1) ^ 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_f8f6f4(tmem + kF2S, (tl ? dq1 : dq0) + 2 * kk, dk + 2 * kk, kIdesc, kk > 0 ? 1u : 0u);
            umma_commit(smem_u32(&bars->s_full[tl]));
            ++suse;
          }
          if (!ok) break;
        }
        if (b >= 1) {
          const int c = b - 1, s = c % kStages;
          const uint64_t dv = sdesc_k_sw128(smem_u32(sm.kv[s][1]));
          for (int tl = 0; tl < 2 && ok; ++tl) {
            if (!mbar_wait(smem_u32(&bars->p_full[tl][c & 1]), (c >> 1) & 1) ||
                !mbar_wait(smem_u32(&bars->o_empty), (ouse & 1) ^ 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t dp = sdesc_k_sw128(smem_u32(sm.p[tl][c & 1]));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_f8f6f4(tmem + kF2P, dp + 2 * kk, dv + 2 * kk, kIdesc, kk > 0 ? 1u : 0u);
            umma_commit(smem_u32(&bars->p_empty[tl][c & 1]));
            umma_commit(smem_u32(&bars->o_full[tl]));
            ++ouse;
          }
          if (!ok) break;
          umma_commit(smem_u32(&bars->kv_empty[s]));
        }
        if (bars->abort) break;
      }
      if (!ok) raise_attn_timeout(bars);
    }
  }
  } else {
    regs_inc<kRegsHigh>();
    // --------------------------------------------- softmax and correction --
    const int q = warp & 3, tl = (warp - 4) >> 2;   // lane quarter, head of the pair
    const int h = h0 + tl;
    const int i = q * 32 + lane, t = q0 + i;
    const float cq = a.sq[(size_t)h * a.T + t] * (kLog2e * 0.08838834764831845f);  // sq * log2(e) / sqrt(128)
    const int jend = a.causal ? min(jreal, t + 1) : jreal;
    float m = -INFINITY, lh = 0.0f;
    float a_prev = 0.0f, sp_prev = 0.0f;
    bool rs_prev = true;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    bool ok = true;

    for (int b = 0; b < nb && ok; ++b) {
      const int kb = kb_first + b;
      if (!warp_wait(smem_u32(&bars->sc_full[b % kScSlots]), (b / kScSlots) & 1) ||
          !warp_wait(smem_u32(&bars->s_full[tl]), b & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t r[4][32];
      tmem_ld64(tmem + lane_off + kF2S, r[0], r[1]);
      tmem_ld64(tmem + lane_off + kF2S + 64, r[2], r[3]);
      tmem_wait_ld();
#pragma unroll
      for (int u = 0; u < 4; ++u) tmem_fence_regs(r[u]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->s_empty));

      // y = (q . k) * s_k per key; the query scale and 1/sqrt(d) log2(e)
      // (cq > 0) are applied after the maximum
      const int lim = jend - kb * 128;             // columns >= lim are masked
      const float4* sk4 = reinterpret_cast<const float4*>(sm.sc[b % kScSlots].sk);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
#pragma unroll
        for (int j4 = 0; j4 < 8; ++j4) {
          const float4 kv4 = sk4[u * 8 + j4];
          const float2 p0 = fmul2(make_float2(__uint_as_float(r[u][4 * j4]), __uint_as_float(r[u][4 * j4 + 1])),
                                  make_float2(kv4.x, kv4.y));
          const float2 p1 = fmul2(make_float2(__uint_as_float(r[u][4 * j4 + 2]), __uint_as_float(r[u][4 * j4 + 3])),
                                  make_float2(kv4.z, kv4.w));
          r[u][4 * j4] = __float_as_uint(p0.x);
          r[u][4 * j4 + 1] = __float_as_uint(p0.y);
          r[u][4 * j4 + 2] = __float_as_uint(p1.x);
          r[u][4 * j4 + 3] = __float_as_uint(p1.y);
        }
      }
      if (lim < 128) {
#pragma unroll
        for (int j = 0; j < 128; ++j)
          if (j >= lim) r[j >> 5][j & 31] = __float_as_uint(-INFINITY);
      }
      float mrow;
      {
        float mg[16];
#pragma unroll
        for (int gi = 0; gi < 16; ++gi) {
          const uint32_t* v = &r[gi >> 2][(8 * gi) & 31];
          mg[gi] = fmax3(fmax3(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2])),
                         fmax3(__uint_as_float(v[3]), __uint_as_float(v[4]), __uint_as_float(v[5])),
                         fmaxf(__uint_as_float(v[6]), __uint_as_float(v[7])));
        }
#pragma unroll
        for (int gi = 0; gi < 8; ++gi) mg[gi] = fmaxf(mg[gi], mg[gi + 8]);
        mrow = fmax3(fmax3(mg[0], mg[1], mg[2]), fmax3(mg[3], mg[4], mg[5]), fmaxf(mg[6], mg[7]));
      }
      const float mb = mrow * cq;
      const float m_new = fmaxf(m, mb);
      const float alpha = ex2(m - m_new);       // 0 on the first block
      m = m_new;
      // P's block scale s_P = amax / 448, amax = 2^(mb - m) the block's
      // largest p; the code input p / s_P = 2^(y * cq - mb + log2 448)
      const float amax = ex2(mb - m_new);
      const float sp = amax * (1.0f / 448.0f);
      const float2 cq2 = make_float2(cq, cq), nm2 = make_float2(kLog2_448 - mb, kLog2_448 - mb);
      float2 ps2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int j = 0; j < 128; j += 2) {
        const int u = j >> 5, k = j & 31;
        const float2 z = ffma2(make_float2(__uint_as_float(r[u][k]), __uint_as_float(r[u][k + 1])), cq2, nm2);
        const float2 pj = make_float2(ex2(z.x), ex2(z.y));
        r[u][k] = __float_as_uint(pj.x);
        r[u][k + 1] = __float_as_uint(pj.y);
        ps2[(j >> 1) & 3] = fadd2(ps2[(j >> 1) & 3], pj);
      }
      const float2 psum = fadd2(fadd2(ps2[0], ps2[1]), fadd2(ps2[2], ps2[3]));
      lh = lh * alpha + sp * (psum.x + psum.y);
      uint32_t w[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int u = j >> 3, k = 4 * (j & 7);
        w[j] = cvt_e4m3x2(__uint_as_float(r[u][k]), __uint_as_float(r[u][k + 1])) |
               (cvt_e4m3x2(__uint_as_float(r[u][k + 2]), __uint_as_float(r[u][k + 3])) << 16);
      }
      if (!warp_wait(smem_u32(&bars->p_empty[tl][b & 1]), ((b >> 1) & 1) ^ 1)) {
        ok = false;
        break;
      }
      // row i of the P tile: 16-byte chunk cc at cc ^ (i & 7) (128-byte swizzle)
      uint8_t* prow = sm.p[tl][b & 1] + i * 128;
#pragma unroll
      for (int cc = 0; cc < 8; ++cc)
        *reinterpret_cast<uint4*>(prow + ((cc ^ (i & 7)) << 4)) =
            make_uint4(w[4 * cc], w[4 * cc + 1], w[4 * cc + 2], w[4 * cc + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->p_full[tl][b & 1]));
      if (b >= 1 && !fold_block2(sm, bars, tmem, lane_off, tl, lane, b - 1, a_prev, sp_prev, rs_prev)) ok = false;
      a_prev = alpha;
      sp_prev = sp;
      rs_prev = __any_sync(0xffffffffu, alpha != 1.0f);
      if (bars->abort) ok = false;
    }
    if (ok && !fold_block2(sm, bars, tmem, lane_off, tl, lane, nb - 1, a_prev, sp_prev, rs_prev)) ok = false;
    if (!ok) raise_attn_timeout(bars);
    const bool real = t < jreal && ok;
    const float il = real ? __fdiv_rn(1.0f, lh) : 0.0f;
    uint16_t* orow = a.o + (size_t)h * kD + (size_t)t * ((size_t)a.Hq * kD);
    const uint32_t to = tmem + lane_off + kF2O + 128 * tl;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      uint32_t o[32];
      tmem_ld32(to + 32 * u, o);
      tmem_wait_ld();
      tmem_fence_regs(o);
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t o8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          o8[j] = real ? pack_bf16x2(__uint_as_float(o[16 * cc + 2 * j]) * il,
                                     __uint_as_float(o[16 * cc + 2 * j + 1]) * il)
                       : 0u;
        st_global_v8(orow + 32 * u + 16 * cc, make_uint4(o8[0], o8[1], o8[2], o8[3]),
                     make_uint4(o8[4], o8[5], o8[6], o8[7]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------
// Power-of-2 scales ("Warum dies für die KI-Ökonomie wichtig ist": the
// recipe's optional power-of-2 scale factors).  Every scale is then a UE8M0
// value, so the tensor core applies them itself
// (tcgen05.mma.kind::mxf8f6f4.block_scale, one scale per row per 32-element
// block, here replicated over the four 32-blocks of a 128-wide one): Q's
// and K's scales inside S = Q K^T, which comes out fully scaled, and P's and
// V's inside O += P V^T, which accumulates across key blocks in one TMEM
// accumulator.  There is no per-block fold: the softmax warps rescale O in
// TMEM only when a row's running maximum moves, and they keep that maximum
// an integer (log2 units) that moves only when a block's maximum exceeds it
// by more than kLazy.  P is taken against it, p / s_P = 2^(y c - m - e), e
// the power-of-2 exponent of the block's amax = 2^(m_b - m); any integer
// reference gives the same codes.  Roles as in k_attn_fwd, plus warp 2,
// which turns each block's fp32 scales into UE8M0 tiles in shared memory
// (row i + 32b of 128 at word [i][b], the byte replicated), and latches
// FP8BW_ERR_DEVICE_CHECK for a scale that is not a power of two.
// TMEM: S at 0 and 128, O at 256, scale tiles (4 columns each) from 384.
constexpr uint32_t kMxO = 256;
constexpr uint32_t kMxSfq = 384, kMxSfk = 388, kMxSfp = 396, kMxSfv = 404;   // K, P, V: two slots each
constexpr float kLazy = 8.0f;

struct SfTile {
  uint32_t w[32][4];
};

struct AttnBarsMx {
  uint64_t q_full;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t sc_full[kScSlots], sc_empty[kScSlots];
  uint64_t sfq_full, sfkv_full[2], sfkv_empty[2];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full[2], p_empty[2];
  uint64_t o_full;           // one P.V into O complete
  uint64_t pair[4];
  uint32_t tmem_base;
  int32_t abort;
};

struct AttnSmemMx {
  uint8_t q[kTile];                    // 1024-aligned tiles first
  uint8_t kv[kStages][2][kTile];
  uint8_t p[2][kTile];
  SfTile sfq, sfk[2], sfv[2], sfp[2];  // UE8M0 tiles for tcgen05.cp (16-byte rows)
  ScSlot sc[kScSlots];
  float red[2][kNH][128];
  float lsum[kNH][128];
  AttnBarsMx bars;
};

// The UE8M0 byte of a positive power-of-two fp32 scale, replicated into the
// four bytes of a word (2^-127 is the subnormal 0x00400000: code 0).
__device__ __forceinline__ uint32_t ue8m0_word(float s, bool& bad) {
  const uint32_t b = __float_as_uint(s);
  if (((b & 0x7FFFFFu) != 0u && b != 0x00400000u) || (b >> 23) == 0xFFu || (b >> 31) != 0u || b == 0u) bad = true;
  return ((b >> 23) & 0xFFu) * 0x01010101u;
}

// One warp: the 128 scales src[0..127] as a UE8M0 tile.
__device__ __forceinline__ bool sf_tile(const float* src, SfTile* dst, int lane) {
  bool bad = false;
  uint4 v;
  v.x = ue8m0_word(src[lane], bad);
  v.y = ue8m0_word(src[lane + 32], bad);
  v.z = ue8m0_word(src[lane + 64], bad);
  v.w = ue8m0_word(src[lane + 96], bad);
  *reinterpret_cast<uint4*>(&dst->w[lane][0]) = v;
  return bad;
}

// 2^e for an integer e in [-126, 127] (exact).
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((e + 127) << 23); }

// Softmax and correction warps of k_attn_fwd_mx (one query row per thread,
// kCols of its 128 columns): per key block, S_b (fully scaled by the MMA)
// from TMEM, mask and block maximum (combined across the row's kNH parts),
// the integer running maximum, the P codes 2^(y c - m - e) and the row's
// scale byte e + 127 into shared memory, the rescale of O in TMEM when the
// row's maximum moved (after the previous P.V is complete), then the signal
// for the next P.V.  At the end O / l in bf16.
__device__ __forceinline__ void attn_softmax_mx(AttnSmemMx& sm, AttnBarsMx* bars, uint32_t tmem,
                                                const AttnArgs& a, int warp, int lane, int h, int q0,
                                                int jreal, int kb_first, int nb) {
  const int q = warp & 3, hf = (warp - 4) >> 2;   // lane quarter, column part
  const int i = q * 32 + lane, t = q0 + i;
  const int col0 = hf * kCols;
  constexpr float c = kLog2e * 0.08838834764831845f;   // log2(e) / sqrt(128)
  const int jend = a.causal ? min(jreal, t + 1) : jreal;
  const uint32_t lane_off = (uint32_t)(q * 32) << 16;
  constexpr int kU = kCols / 32;
  float m = -INFINITY, lh = 0.0f;
  bool ok = true;
  uint32_t meets = 0;

  for (int b = 0; b < nb && ok; ++b) {
    const int kb = kb_first + b;
    if (!warp_wait(smem_u32(&bars->s_full[b & 1]), (b >> 1) & 1)) {
      ok = false;
      break;
    }
    tc_fence_after();
    uint32_t r[kU][32];
    const uint32_t ta = tmem + lane_off + (b & 1) * 128 + col0;
#pragma unroll
    for (int u = 0; u < kU; ++u) tmem_ld32(ta + 32 * u, r[u]);
    tmem_wait_ld();
#pragma unroll
    for (int u = 0; u < kU; ++u) tmem_fence_regs(r[u]);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars->s_empty[b & 1]));

    const int lim = jend - kb * 128 - col0;      // columns >= lim are masked
    if (lim < kCols) {
#pragma unroll
      for (int j = 0; j < kCols; ++j)
        if (j >= lim) r[j >> 5][j & 31] = __float_as_uint(-INFINITY);
    }
    float mh;
    {
      float mg[kCols / 8];
#pragma unroll
      for (int gi = 0; gi < kCols / 8; ++gi) {
        const uint32_t* v = &r[(8 * gi) >> 5][(8 * gi) & 31];
        mg[gi] = fmax3(fmax3(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2])),
                       fmax3(__uint_as_float(v[3]), __uint_as_float(v[4]), __uint_as_float(v[5])),
                       fmaxf(__uint_as_float(v[6]), __uint_as_float(v[7])));
      }
      mh = mg[0];
#pragma unroll
      for (int gi = 1; gi + 1 < kCols / 8; gi += 2) mh = fmax3(mh, mg[gi], mg[gi + 1]);
      if ((kCols / 8) % 2 == 0) mh = fmaxf(mh, mg[kCols / 8 - 1]);
    }
    sm.red[b & 1][hf][i] = mh;
    if (!pair_meet(bars, q, lane, meets++)) {
      ok = false;
      break;
    }
    float mrow = sm.red[b & 1][0][i];
#pragma unroll
    for (int k = 1; k < kNH; ++k) mrow = fmaxf(mrow, sm.red[b & 1][k][i]);
    const float mb = mrow * c;                   // the block's largest logit, log2 units
    // integer running maximum, moved only by more than kLazy (then p may
    // reach 2^kLazy in between, harmless in fp32)
    const float m_new = mb > m + kLazy ? ceilf(mb) : m;
    const bool moved = m_new != m;
    const float dm = m - m_new;                  // an integer, or -inf on the first block
    const float alpha = moved ? (dm < -126.0f ? 0.0f : exp2i((int)dm)) : 1.0f;
    m = m_new;
    // P's power-of-2 block scale 2^e: the smallest e with 2^(mb - m) <= 448 2^e
    int e = (int)ceilf((mb - m) - kLog2_448);
    e = max(-127, min(127, e));
    const float sp = e == -127 ? __uint_as_float(0x00400000u) : exp2i(e);
    const float2 c2 = make_float2(c, c);
    const float off = -(m + (float)e);
    const float2 nm2 = make_float2(off, off);
    float2 ps2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int j = 0; j < kCols; j += 2) {
      const int u = j >> 5, k = j & 31;
      const float2 z = ffma2(make_float2(__uint_as_float(r[u][k]), __uint_as_float(r[u][k + 1])), c2, nm2);
      const float2 pj = make_float2(ex2(z.x), ex2(z.y));
      r[u][k] = __float_as_uint(pj.x);
      r[u][k + 1] = __float_as_uint(pj.y);
      ps2[(j >> 1) & 3] = fadd2(ps2[(j >> 1) & 3], pj);
    }
    const float2 psum = fadd2(fadd2(ps2[0], ps2[1]), fadd2(ps2[2], ps2[3]));
    lh = lh * alpha + sp * (psum.x + psum.y);
    uint32_t w[kCols / 4];
#pragma unroll
    for (int j = 0; j < kCols / 4; ++j) {
      const int u = j >> 3, k = 4 * (j & 7);
      w[j] = cvt_e4m3x2(__uint_as_float(r[u][k]), __uint_as_float(r[u][k + 1])) |
             (cvt_e4m3x2(__uint_as_float(r[u][k + 2]), __uint_as_float(r[u][k + 3])) << 16);
    }
    if (!warp_wait(smem_u32(&bars->p_empty[b & 1]), ((b >> 1) & 1) ^ 1)) {
      ok = false;
      break;
    }
    // row i of the P tile: 16-byte chunk c at c ^ (i & 7) (128-byte swizzle)
    uint8_t* prow = sm.p[b & 1] + i * 128;
#pragma unroll
    for (int cc = 0; cc < kCols / 16; ++cc)
      *reinterpret_cast<uint4*>(prow + (((hf * (kCols / 16) + cc) ^ (i & 7)) << 4)) =
          make_uint4(w[4 * cc], w[4 * cc + 1], w[4 * cc + 2], w[4 * cc + 3]);
    if (hf == 0) sm.sfp[b & 1].w[i & 31][i >> 5] = (uint32_t)(e + 127) * 0x01010101u;
    if (b >= 1) {
      // the previous P.V is complete; rescale O if a row of this warp moved
      if (!warp_wait(smem_u32(&bars->o_full), (b - 1) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (__any_sync(0xffffffffu, moved)) {
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          uint32_t o[32];
          const uint32_t to = tmem + lane_off + kMxO + col0 + 32 * u;
          tmem_ld32(to, o);
          tmem_wait_ld();
          tmem_fence_regs(o);
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
          tmem_st32(to, o);
        }
        tmem_wait_st();
      }
    }
    fence_proxy_async_smem();   // the P tile and scale bytes, for the MMA
    tc_fence_before();          // the rescaled O, for the MMA that accumulates onto it
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars->p_full[b & 1]));
    if (bars->abort) ok = false;
  }
  if (ok && !warp_wait(smem_u32(&bars->o_full), (nb - 1) & 1)) ok = false;
  tc_fence_after();
  if (!ok) raise_attn_timeout(bars);
  // row sum of the kNH parts, then O / l in bf16 (padding rows: 0)
  sm.lsum[hf][i] = lh;
  if (!pair_meet(bars, q, lane, meets++)) ok = false;
  float l = sm.lsum[0][i];
#pragma unroll
  for (int k = 1; k < kNH; ++k) l += sm.lsum[k][i];
  const bool real = t < jreal && ok;
  const float il = real ? __fdiv_rn(1.0f, l) : 0.0f;
  uint16_t* orow = a.o + (size_t)h * kD + (size_t)t * ((size_t)a.Hq * kD) + col0;
#pragma unroll
  for (int u = 0; u < kU; ++u) {
    uint32_t o[32];
    tmem_ld32(tmem + lane_off + kMxO + col0 + 32 * u, o);
    tmem_wait_ld();
    tmem_fence_regs(o);
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      uint32_t o8[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        o8[j] = real ? pack_bf16x2(__uint_as_float(o[16 * cc + 2 * j]) * il,
                                   __uint_as_float(o[16 * cc + 2 * j + 1]) * il)
                     : 0u;
      st_global_v8(orow + 32 * u + 16 * cc, make_uint4(o8[0], o8[1], o8[2], o8[3]),
                   make_uint4(o8[4], o8[5], o8[6], o8[7]));
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    k_attn_fwd_mx(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  AttnSmemMx& sm = *reinterpret_cast<AttnSmemMx*>(smem_align1024(smem_raw));
  AttnBarsMx* bars = &sm.bars;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ int s_seg;
  const AttnBlock wk = attn_block<kThreads>(a, &s_seg);
  if (wk.done) return;
  const int h = wk.h, g = wk.g, q0 = wk.q0, jreal = wk.jreal;
  const int kb_first = wk.kb_first, nb = wk.nb;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_u32(&bars->kv_full[i]), 1);
      mbar_init(smem_u32(&bars->kv_empty[i]), 1);
    }
    for (int i = 0; i < kScSlots; ++i) {
      mbar_init(smem_u32(&bars->sc_full[i]), 1);
      mbar_init(smem_u32(&bars->sc_empty[i]), 1);   // read by the scale converter only
    }
    mbar_init(smem_u32(&bars->sfq_full), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars->sfkv_full[i]), 1);
      mbar_init(smem_u32(&bars->sfkv_empty[i]), 1);
      mbar_init(smem_u32(&bars->s_full[i]), 1);
      mbar_init(smem_u32(&bars->s_empty[i]), kSoftWarps);
      mbar_init(smem_u32(&bars->p_full[i]), kSoftWarps);
      mbar_init(smem_u32(&bars->p_empty[i]), 1);
    }
    mbar_init(smem_u32(&bars->o_full), 1);
    for (int i = 0; i < 4; ++i) mbar_init(smem_u32(&bars->pair[i]), kNH);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp < 4) {
  regs_dec<kRegsLow>();
  if (warp == 0) {
    // ---------------------------------------------------- TMA producer ----
    if (lane == 0) attn_producer<1>(sm, bars, &tmQ, &tmK, &tmV, a, h, g, q0, kb_first, nb);
  } else if (warp == 1) {
    // ----------------------------------------------------- MMA issuer -----
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_mx(128, 128, 0);   // E4M3 x E4M3, UE8M0 scales, byte 0
      bool ok = mbar_wait(smem_u32(&bars->q_full), 0) && mbar_wait(smem_u32(&bars->sfq_full), 0);
      tc_fence_after();
      if (ok) tmem_cp_32x128b_x4(tmem + kMxSfq, sdesc_k_noswz_16B(smem_u32(&sm.sfq.w[0][0])));
      const uint64_t dq = sdesc_k_sw128(smem_u32(sm.q));
      for (int b = 0; ok && b <= nb; ++b) {
        if (b < nb) {
          const int s = b % kStages;
          if (!mbar_wait(smem_u32(&bars->kv_full[s]), (b / kStages) & 1) ||
              !mbar_wait(smem_u32(&bars->s_empty[b & 1]), ((b >> 1) & 1) ^ 1) ||
              !mbar_wait(smem_u32(&bars->sfkv_full[b & 1]), (b >> 1) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t tk = tmem + kMxSfk + 4 * (b & 1);
          tmem_cp_32x128b_x4(tk, sdesc_k_noswz_16B(smem_u32(&sm.sfk[b & 1].w[0][0])));
          const uint64_t dk = sdesc_k_sw128(smem_u32(sm.kv[s][0]));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_mx(tmem + (b & 1) * 128, dq + 2 * kk, dk + 2 * kk, idesc, tmem + kMxSfq, tk, kk > 0 ? 1u : 0u);
          umma_commit(smem_u32(&bars->s_full[b & 1]));
        }
        if (b >= 1) {
          const int c = b - 1, s = c % kStages;
          if (!mbar_wait(smem_u32(&bars->p_full[c & 1]), (c >> 1) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t tp = tmem + kMxSfp + 4 * (c & 1), tv = tmem + kMxSfv + 4 * (c & 1);
          tmem_cp_32x128b_x4(tp, sdesc_k_noswz_16B(smem_u32(&sm.sfp[c & 1].w[0][0])));
          tmem_cp_32x128b_x4(tv, sdesc_k_noswz_16B(smem_u32(&sm.sfv[c & 1].w[0][0])));
          const uint64_t dp = sdesc_k_sw128(smem_u32(sm.p[c & 1]));
          const uint64_t dv = sdesc_k_sw128(smem_u32(sm.kv[s][1]));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_mx(tmem + kMxO, dp + 2 * kk, dv + 2 * kk, idesc, tp, tv, (c > 0 || kk > 0) ? 1u : 0u);
          umma_commit(smem_u32(&bars->p_empty[c & 1]));
          umma_commit(smem_u32(&bars->kv_empty[s]));
          umma_commit(smem_u32(&bars->sfkv_empty[c & 1]));
          umma_commit(smem_u32(&bars->o_full));
        }
        if (bars->abort) break;
      }
      if (!ok) raise_attn_timeout(bars);
    }
  } else if (warp == 2) {
    // ------------------------------------------------ scale converter -----
    bool bad = sf_tile(a.sq + (size_t)h * a.T + q0, &sm.sfq, lane);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars->sfq_full));
    for (int b = 0; b < nb; ++b) {
      const int sl = b % kScSlots;
      if (!warp_wait(smem_u32(&bars->sc_full[sl]), (b / kScSlots) & 1) ||
          !warp_wait(smem_u32(&bars->sfkv_empty[b & 1]), ((b >> 1) & 1) ^ 1)) {
        if (lane == 0) raise_attn_timeout(bars);
        break;
      }
      bad |= sf_tile(sm.sc[sl].sk, &sm.sfk[b & 1], lane);
      bad |= sf_tile(sm.sc[sl].sv, &sm.sfv[b & 1], lane);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&bars->sfkv_full[b & 1]));
        mbar_arrive(smem_u32(&bars->sc_empty[sl]));
      }
      if (bars->abort) break;
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&g_attn_error, DEV_ERR_CHECK);
  }
  } else {
    regs_inc<kRegsHigh>();
    attn_softmax_mx(sm, bars, tmem, a, warp, lane, h, q0, jreal, kb_first, nb);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------
// Power-of-2 scales, two query heads per CTA.  With one query tile, the two
// softmax warps of a TMEM lane quarter run the same phases at the same time
// (they meet on every block's maximum), so the MUFU idles while they load S,
// reduce, store P and rescale.  Here a CTA takes one 128-query block of two
// query heads h, h+1 of the same KV group (they read the same K and V tiles
// and share the causal mask), and each head has its own four softmax warps,
// one per lane quarter, a thread owning a whole row (128 columns, no
// meeting).  The two heads' warps share the schedulers, so one head's
// exponentials overlap the other's remaining phases.  Per key block the MMA
// warp computes S_A, S_B (one S buffer in TMEM, taken in turn: S_B is
// issued once head A has read S_A), then O_A += P_A V^T and O_B += P_B V^T
// for the previous block.  Numerics as in k_attn_fwd_mx (every scale
// applied by the block-scaled MMA, integer running maximum, P codes against
// it).  TMEM: S at 0, O_A at 128, O_B at 256, scale tiles (4 columns each)
// from 384: Q (per head), K and V (two slots), P (per head, two slots).
// Launched when Hq / Hkv is even.
constexpr uint32_t kM2S = 0, kM2O = 128;              // O of head tl at kM2O + 128 tl
constexpr uint32_t kM2Sfq = 384, kM2Sfk = 392, kM2Sfv = 400, kM2Sfp = 408;

struct AttnBarsMx2 {
  uint64_t q_full;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t sc_full[kScSlots], sc_empty[kScSlots];
  uint64_t sfq_full, sfkv_full[2], sfkv_empty[2];
  uint64_t s_full[2];              // [head]: its S is in the buffer
  uint64_t s_empty;                // the buffer's last S has been read (four warps)
  uint64_t p_full[2][2], p_empty[2][2];   // [head][slot]
  uint64_t o_full[2];              // [head]: a P.V into its O is complete
  uint32_t tmem_base;
  int32_t abort;
};

struct AttnSmemMx2 {
  uint8_t q[2][kTile];                 // 1024-aligned tiles first
  uint8_t kv[kStages][2][kTile];
  uint8_t p[2][2][kTile];              // [head][slot]
  SfTile sfq[2], sfk[2], sfv[2], sfp[2][2];
  ScSlot sc[kScSlots];
  AttnBarsMx2 bars;
};
static_assert(sizeof(AttnSmemMx2) + 1024 <= 232448, "shared memory budget (two heads)");
static_assert(kM2Sfp + 16 <= 512, "TMEM columns (two heads)");

// Softmax and correction warps of k_attn_fwd_mx2: warps 4-7 own head h0,
// warps 8-11 head h0 + 1; one query row per thread, all 128 columns.  Per
// key block as attn_softmax_mx, without the exchange of partial maxima.
__device__ __forceinline__ void attn_softmax_mx2(AttnSmemMx2& sm, AttnBarsMx2* bars, uint32_t tmem,
                                                 const AttnArgs& a, int warp, int lane, int h0, int q0,
                                                 int jreal, int kb_first, int nb) {
  const int q = warp & 3, tl = (warp - 4) >> 2;   // lane quarter, head of the pair
  const int i = q * 32 + lane, t = q0 + i;
  constexpr float c = kLog2e * 0.08838834764831845f;   // log2(e) / sqrt(128)
  const int jend = a.causal ? min(jreal, t + 1) : jreal;
  const uint32_t lane_off = (uint32_t)(q * 32) << 16;
  const uint32_t to = tmem + lane_off + kM2O + 128 * tl;
  float m = -INFINITY, lh = 0.0f;
  bool ok = true;

  for (int b = 0; b < nb && ok; ++b) {
    const int kb = kb_first + b;
    if (!warp_wait(smem_u32(&bars->s_full[tl]), b & 1)) {
      ok = false;
      break;
    }
    tc_fence_after();
    uint32_t r[4][32];
    tmem_ld64(tmem + lane_off + kM2S, r[0], r[1]);
    tmem_ld64(tmem + lane_off + kM2S + 64, r[2], r[3]);
    tmem_wait_ld();
#pragma unroll
    for (int u = 0; u < 4; ++u) tmem_fence_regs(r[u]);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars->s_empty));

    const int lim = jend - kb * 128;             // columns >= lim are masked
    if (lim < 128) {
#pragma unroll
      for (int j = 0; j < 128; ++j)
        if (j >= lim) r[j >> 5][j & 31] = __float_as_uint(-INFINITY);
    }
    float mh;
    {
      float mg[16];
#pragma unroll
      for (int gi = 0; gi < 16; ++gi) {
        const uint32_t* v = &r[gi >> 2][(8 * gi) & 31];
        mg[gi] = fmax3(fmax3(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2])),
                       fmax3(__uint_as_float(v[3]), __uint_as_float(v[4]), __uint_as_float(v[5])),
                       fmaxf(__uint_as_float(v[6]), __uint_as_float(v[7])));
      }
#pragma unroll
      for (int gi = 0; gi < 8; ++gi) mg[gi] = fmaxf(mg[gi], mg[gi + 8]);
      mh = fmax3(fmax3(mg[0], mg[1], mg[2]), fmax3(mg[3], mg[4], mg[5]), fmaxf(mg[6], mg[7]));
    }
    const float mb = mh * c;                     // the block's largest logit, log2 units
    const float m_new = mb > m + kLazy ? ceilf(mb) : m;
    const bool moved = m_new != m;
    const float dm = m - m_new;                  // an integer, or -inf on the first block
    const float alpha = moved ? (dm < -126.0f ? 0.0f : exp2i((int)dm)) : 1.0f;
    m = m_new;
    // P's power-of-2 block scale 2^e: the smallest e with 2^(mb - m) <= 448 2^e
    int e = (int)ceilf((mb - m) - kLog2_448);
    e = max(-127, min(127, e));
    const float sp = e == -127 ? __uint_as_float(0x00400000u) : exp2i(e);
    const float2 c2 = make_float2(c, c);
    const float off = -(m + (float)e);
    const float2 nm2 = make_float2(off, off);
    float2 ps2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int j = 0; j < 128; j += 2) {
      const int u = j >> 5, k = j & 31;
      const float2 z = ffma2(make_float2(__uint_as_float(r[u][k]), __uint_as_float(r[u][k + 1])), c2, nm2);
      const float2 pj = make_float2(ex2(z.x), ex2(z.y));
      r[u][k] = __float_as_uint(pj.x);
      r[u][k + 1] = __float_as_uint(pj.y);
      ps2[(j >> 1) & 3] = fadd2(ps2[(j >> 1) & 3], pj);
    }
    const float2 psum = fadd2(fadd2(ps2[0], ps2[1]), fadd2(ps2[2], ps2[3]));
    lh = lh * alpha + sp * (psum.x + psum.y);
    uint32_t w[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int u = j >> 3, k = 4 * (j & 7);
      w[j] = cvt_e4m3x2(__uint_as_float(r[u][k]), __uint_as_float(r[u][k + 1])) |
             (cvt_e4m3x2(__uint_as_float(r[u][k + 2]), __uint_as_float(r[u][k + 3])) << 16);
    }
    if (!warp_wait(smem_u32(&bars->p_empty[tl][b & 1]), ((b >> 1) & 1) ^ 1)) {
      ok = false;
      break;
    }
    // row i of the P tile: 16-byte chunk cc at cc ^ (i & 7) (128-byte swizzle)
    uint8_t* prow = sm.p[tl][b & 1] + i * 128;
#pragma unroll
    for (int cc = 0; cc < 8; ++cc)
      *reinterpret_cast<uint4*>(prow + ((cc ^ (i & 7)) << 4)) =
          make_uint4(w[4 * cc], w[4 * cc + 1], w[4 * cc + 2], w[4 * cc + 3]);
    sm.sfp[tl][b & 1].w[i & 31][i >> 5] = (uint32_t)(e + 127) * 0x01010101u;
    if (b >= 1) {
      // the previous P.V of this head is complete; rescale O if a row moved
      if (!warp_wait(smem_u32(&bars->o_full[tl]), (b - 1) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (__any_sync(0xffffffffu, moved)) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint32_t o[32];
          tmem_ld32(to + 32 * u, o);
          tmem_wait_ld();
          tmem_fence_regs(o);
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
          tmem_st32(to + 32 * u, o);
        }
        tmem_wait_st();
      }
    }
    fence_proxy_async_smem();   // the P tile and scale bytes, for the MMA
    tc_fence_before();          // the rescaled O, for the MMA that accumulates onto it
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars->p_full[tl][b & 1]));
    if (bars->abort) ok = false;
  }
  if (ok && !warp_wait(smem_u32(&bars->o_full[tl]), (nb - 1) & 1)) ok = false;
  tc_fence_after();
  if (!ok) raise_attn_timeout(bars);
  const bool real = t < jreal && ok;
  const float il = real ? __fdiv_rn(1.0f, lh) : 0.0f;
  uint16_t* orow = a.o + (size_t)(h0 + tl) * kD + (size_t)t * ((size_t)a.Hq * kD);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    uint32_t o[32];
    tmem_ld32(to + 32 * u, o);
    tmem_wait_ld();
    tmem_fence_regs(o);
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      uint32_t o8[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        o8[j] = real ? pack_bf16x2(__uint_as_float(o[16 * cc + 2 * j]) * il,
                                   __uint_as_float(o[16 * cc + 2 * j + 1]) * il)
                     : 0u;
      st_global_v8(orow + 32 * u + 16 * cc, make_uint4(o8[0], o8[1], o8[2], o8[3]),
                   make_uint4(o8[4], o8[5], o8[6], o8[7]));
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    k_attn_fwd_mx2(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const AttnArgs a) {
  static_assert(kSoftWarps == 8, "four softmax warps per head of the pair");
  extern __shared__ uint8_t smem_raw[];
  AttnSmemMx2& sm = *reinterpret_cast<AttnSmemMx2*>(smem_align1024(smem_raw));
  AttnBarsMx2* bars = &sm.bars;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ int s_seg;
  const AttnBlock wk = attn_block<kThreads, 2>(a, &s_seg);
  if (wk.done) return;
  const int h0 = wk.h, g = wk.g, q0 = wk.q0, jreal = wk.jreal;
  const int kb_first = wk.kb_first, nb = wk.nb;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_u32(&bars->kv_full[i]), 1);
      mbar_init(smem_u32(&bars->kv_empty[i]), 1);
    }
    for (int i = 0; i < kScSlots; ++i) {
      mbar_init(smem_u32(&bars->sc_full[i]), 1);
      mbar_init(smem_u32(&bars->sc_empty[i]), 1);   // read by the scale converter only
    }
    mbar_init(smem_u32(&bars->sfq_full), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars->sfkv_full[i]), 1);
      mbar_init(smem_u32(&bars->sfkv_empty[i]), 1);
      mbar_init(smem_u32(&bars->s_full[i]), 1);
      mbar_init(smem_u32(&bars->o_full[i]), 1);
      for (int j = 0; j < 2; ++j) {
        mbar_init(smem_u32(&bars->p_full[i][j]), 4);
        mbar_init(smem_u32(&bars->p_empty[i][j]), 1);
      }
    }
    mbar_init(smem_u32(&bars->s_empty), 4);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp < 4) {
  regs_dec<kRegsLow>();
  if (warp == 0) {
    // ---------------------------------------------------- TMA producer ----
    if (lane == 0) attn_producer<2>(sm, bars, &tmQ, &tmK, &tmV, a, h0, g, q0, kb_first, nb);
  } else if (warp == 1) {
    // ----------------------------------------------------- MMA issuer -----
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_mx(128, 128, 0);   // E4M3 x E4M3, UE8M0 scales, byte 0
      bool ok = mbar_wait(smem_u32(&bars->q_full), 0) && mbar_wait(smem_u32(&bars->sfq_full), 0);
      tc_fence_after();
      if (ok) {
        tmem_cp_32x128b_x4(tmem + kM2Sfq, sdesc_k_noswz_16B(smem_u32(&sm.sfq[0].w[0][0])));
        tmem_cp_32x128b_x4(tmem + kM2Sfq + 4, sdesc_k_noswz_16B(smem_u32(&sm.sfq[1].w[0][0])));
      }
      const uint64_t dq0 = sdesc_k_sw128(smem_u32(sm.q[0])), dq1 = sdesc_k_sw128(smem_u32(sm.q[1]));
      uint32_t suse = 0;   // S computations so far (the buffer alternates between the heads)
      for (int b = 0; ok && b <= nb; ++b) {
        if (b < nb) {
          const int s = b % kStages;
          if (!mbar_wait(smem_u32(&bars->kv_full[s]), (b / kStages) & 1) ||
              !mbar_wait(smem_u32(&bars->sfkv_full[b & 1]), (b >> 1) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t tk = tmem + kM2Sfk + 4 * (b & 1);
          tmem_cp_32x128b_x4(tk, sdesc_k_noswz_16B(smem_u32(&sm.sfk[b & 1].w[0][0])));
          const uint64_t dk = sdesc_k_sw128(smem_u32(sm.kv[s][0]));
          for (int tl = 0; tl < 2 && ok; ++tl) {
            // the previous S (the other head's, or this one's last block) has been read
            if (!mbar_wait(smem_u32(&bars->s_empty), (suse & 1) ^ 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_mx(tmem + kM2S, (tl ? dq1 : dq0) + 2 * kk, dk + 2 * kk, idesc, tmem + kM2Sfq + 4 * tl, tk,
                      kk > 0 ? 1u : 0u);
            umma_commit(smem_u32(&bars->s_full[tl]));
            ++suse;
          }
          if (!ok) break;
        }
        if (b >= 1) {
          const int c = b - 1, s = c % kStages;
          const uint32_t tv = tmem + kM2Sfv + 4 * (c & 1);
          const uint64_t dv = sdesc_k_sw128(smem_u32(sm.kv[s][1]));
          for (int tl = 0; tl < 2 && ok; ++tl) {
            if (!mbar_wait(smem_u32(&bars->p_full[tl][c & 1]), (c >> 1) & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t tp = tmem + kM2Sfp + 8 * tl + 4 * (c & 1);
            tmem_cp_32x128b_x4(tp, sdesc_k_noswz_16B(smem_u32(&sm.sfp[tl][c & 1].w[0][0])));
            if (tl == 0) tmem_cp_32x128b_x4(tv, sdesc_k_noswz_16B(smem_u32(&sm.sfv[c & 1].w[0][0])));
            const uint64_t dp = sdesc_k_sw128(smem_u32(sm.p[tl][c & 1]));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_mx(tmem + kM2O + 128 * tl, dp + 2 * kk, dv + 2 * kk, idesc, tp, tv,
                      (c > 0 || kk > 0) ? 1u : 0u);
            umma_commit(smem_u32(&bars->p_empty[tl][c & 1]));
            umma_commit(smem_u32(&bars->o_full[tl]));
          }
          if (!ok) break;
          umma_commit(smem_u32(&bars->kv_empty[s]));
          umma_commit(smem_u32(&bars->sfkv_empty[c & 1]));
        }
        if (bars->abort) break;
      }
      if (!ok) raise_attn_timeout(bars);
    }
  } else if (warp == 2) {
    // ------------------------------------------------ scale converter -----
    bool bad = sf_tile(a.sq + (size_t)h0 * a.T + q0, &sm.sfq[0], lane);
    bad |= sf_tile(a.sq + (size_t)(h0 + 1) * a.T + q0, &sm.sfq[1], lane);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars->sfq_full));
    for (int b = 0; b < nb; ++b) {
      const int sl = b % kScSlots;
      if (!warp_wait(smem_u32(&bars->sc_full[sl]), (b / kScSlots) & 1) ||
          !warp_wait(smem_u32(&bars->sfkv_empty[b & 1]), ((b >> 1) & 1) ^ 1)) {
        if (lane == 0) raise_attn_timeout(bars);
        break;
      }
      bad |= sf_tile(sm.sc[sl].sk, &sm.sfk[b & 1], lane);
      bad |= sf_tile(sm.sc[sl].sv, &sm.sfv[b & 1], lane);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&bars->sfkv_full[b & 1]));
        mbar_arrive(smem_u32(&bars->sc_empty[sl]));
      }
      if (bars->abort) break;
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&g_attn_error, DEV_ERR_CHECK);
  }
  } else {
    regs_inc<kRegsHigh>();
    attn_softmax_mx2(sm, bars, tmem, a, warp, lane, h0, q0, jreal, kb_first, nb);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_attention_fwd(int64_t T, int Hq, int Hkv, int nseg, const int32_t* d_off,
                                 const int32_t* d_len, int causal, int mode, const uint8_t* q, const float* sq,
                                 const uint8_t* k, const float* sk, const uint8_t* vT, const float* sv,
                                 void* o, cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q, (uint64_t)Hq * kD, (uint64_t)T,
                (uint64_t)Hq * kD, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!make_map(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, k, (uint64_t)Hkv * kD, (uint64_t)T,
                (uint64_t)Hkv * kD, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!make_map(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, vT, (uint64_t)T, (uint64_t)Hkv * kD,
                (uint64_t)T, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  AttnArgs a;
  a.T = (int)T;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.nseg = nseg;
  a.causal = causal;
  a.off = d_off;
  a.len = d_len;
  a.sq = sq;
  a.sk = sk;
  a.sv = sv;
  a.o = static_cast<uint16_t*>(o);
  const bool mx = mode == FP8BW_SCALE_POW2;
  const bool pair = (Hq / Hkv) % 2 == 0;   // two query heads of one KV group per CTA
  const void* kern = mx ? (pair ? reinterpret_cast<const void*>(k_attn_fwd_mx2)
                                : reinterpret_cast<const void*>(k_attn_fwd_mx))
                        : (pair ? reinterpret_cast<const void*>(k_attn_fwd2)
                                : reinterpret_cast<const void*>(k_attn_fwd));
  const size_t smem = (mx ? (pair ? sizeof(AttnSmemMx2) : sizeof(AttnSmemMx))
                          : (pair ? sizeof(AttnSmem2) : sizeof(AttnSmem))) + 1024;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes attr;
  e = cudaFuncGetAttributes(&attr, kern);
  if (e != cudaSuccess) return e;
  // setmaxnreg draws on the launch allocation: refuse to launch if the
  // compiled register count could not cover the split.
  if (attr.numRegs < kRegsLaunch) return cudaErrorInvalidConfiguration;
  const unsigned grid = (unsigned)((T / 128) * (pair ? Hq / 2 : Hq));
  if (mx && pair) k_attn_fwd_mx2<<<grid, kThreads, smem, st>>>(tq, tk, tv, a);
  else if (mx) k_attn_fwd_mx<<<grid, kThreads, smem, st>>>(tq, tk, tv, a);
  else if (pair) k_attn_fwd2<<<grid, kThreads, smem, st>>>(tq, tk, tv, a);
  else k_attn_fwd<<<grid, kThreads, smem, st>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

cudaError_t attn_read_clear_error(uint32_t* out, cudaStream_t st) {
  uint32_t v = 0, z = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_attn_error, sizeof v, 0, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess && v) e = cudaMemcpyToSymbolAsync(g_attn_error, &z, sizeof z, 0, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  *out = v;
  return e;
}

}  // namespace fp8bw

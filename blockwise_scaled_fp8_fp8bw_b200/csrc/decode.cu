// FP8 KV-cache decode attention for sm_100a: one new query token per
// sequence attends to its cached keys, K and V stored as E4M3 codes with one
// fp32 scale per token and KV head (the row-wise 1x128 quantization of the
// cache's token matrix [B*Lmax][Hkv*128]).
//
// Method: "NVIDIA NeMo RL erreicht 48% ..." section "Leistungsgewinne in der
// Praxis": the recipe extends FP8 to the KV cache and the attention
// operations of generation.  The query stays bf16; logits, softmax and P.V
// are fp32 (no tensor core: per key the work is 2 x 128 x G multiply-adds
// against 256 bytes of cache, so the kernel is bound by HBM, not by
// arithmetic).
//
// One cluster of kNS CTAs per (sequence, KV head); CTA r takes the r-th
// contiguous slice of the sequence's keys for all G = Hq / Hkv query heads
// of the group, in 32-key tiles.  Warp 0 (one thread) loads the tiles with
// TMA: the K and V tiles [32 keys][128] of the KV head (128-byte swizzle)
// and the tile's 32 key and 32 value scales (bulk copies), into kSlots
// shared-memory slots per consumer warp, tile t going to consumer warp
// t % kCW.  The
// consumer warps:
//   logits   lane = key: its K row from shared memory (eight conflict-free
//            16-byte loads thanks to the swizzle), decoded four codes of a
//            word at a time (E4M3 -> f16x2 -> f32, the word's 16-bit halves
//            taken in place) and dotted with the G query rows held as
//            [dim][head] (broadcast loads; head pairs on packed fp32
//            lanes), times the key's scale;
//   softmax  per head, online in log2 units (the query is pre-scaled by
//            log2(e) / sqrt(128)): tile maximum across the warp, running
//            maximum, p = 2^(z - m), per-lane partial sums;
//   P.V      lane = channels 4 lane .. 4 lane + 3: per key of the tile, its
//            p * s_V from shared memory (broadcast) and the row's four codes.
// The warps' states (m, l, o) are merged in shared memory, the cluster's
// CTAs' states through distributed shared memory, each CTA combining and
// writing (O / l in bf16) its share of the outputs.  A sequence with length 0 gives zeros.  Every mbarrier wait
// is bounded (a timeout latches an error bit); the producer waits, bounded,
// for each of its copies before the CTA leaves; the two cluster barriers
// are reached by every CTA of the cluster.

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "tmap.cuh"

namespace fp8bw {

__device__ uint32_t g_dec_error;

namespace {

constexpr int kD = 128;
// CTAs per (sequence, KV head): one cluster.  Four measured faster than
// eight (3.11-3.13 against 2.66-2.67 TB/s on the 64 x 16K rollout batch,
// with the first round of loads issued before the query staging): a CTA's
// fixed costs (barrier setup, query staging, the first loads' latency, the
// merges) then spread over twice the keys.  Two ran the same as four, three
// and six slower.
constexpr int kNS = 4;
// Eight consumer warps with one ring slot each (two CTAs per SM, 16
// consumer warps): measured faster than four warps with two slots (2.11 vs
// 1.97 TB/s on the 64 x 16K rollout batch) and than eight with two (one CTA
// per SM, 1.51 TB/s).
constexpr int kCW = 8;                 // consumer warps
constexpr int kSlots = 1;              // ring slots per consumer warp
constexpr int kThreads = 32 * (kCW + 1);
constexpr uint32_t kTileB = 32 * kD;   // one 32-key tile of K or V codes
constexpr float kQScale = 1.4426950408889634f * 0.08838834764831845f;   // log2(e) / sqrt(128)

struct DecArgs {
  int B, Hq, Hkv;
  int64_t Lmax, T;        // T = B * Lmax cache rows
  const int32_t* len;     // device [B]
  const uint16_t* q;      // bf16 [B][Hq*128]
  const float* sk;        // [Hkv][T]
  const float* sv;
  uint16_t* o;            // bf16 [B][Hq*128]
};

struct DecBars {
  uint64_t full[kCW][kSlots], empty[kCW][kSlots];
};

template <int G>
struct DecSmem {
  uint8_t kt[kCW][kSlots][kTileB];   // 1024-aligned tiles first (128-byte swizzle)
  uint8_t vt[kCW][kSlots][kTileB];
  float ks[kCW][kSlots][32], vs[kCW][kSlots][32];
  float qs[kD][G];                   // query rows * log2(e)/sqrt(128), [dim][head]
  float pw[kCW][32][G];              // p * s_V of the warp's 32 keys
  float wm[kCW][G], wl[kCW][G];
  float wo[kCW][G][kD];              // the warps' partial outputs
  float cm[G], cl[G];                // the CTA's state, read by every CTA of the cluster
  float co[G][kD];
  DecBars bars;
};

// Four E4M3 codes (byte i of w is code i) to floats, exactly (E4M3 -> f16
// is exact, f16 -> f32 too).  The word's 16-bit halves are taken as they
// sit in the register (no mask or shift).
__device__ __forceinline__ float4 dec4(uint32_t w) {
  float4 r;
  asm("{\n\t.reg .b16 lo, hi, a, b, c, d;\n\t.reg .b32 h01, h23;\n\t"
      "mov.b32 {lo, hi}, %4;\n\t"
      "cvt.rn.f16x2.e4m3x2 h01, lo;\n\t"
      "cvt.rn.f16x2.e4m3x2 h23, hi;\n\t"
      "mov.b32 {a, b}, h01;\n\t"
      "mov.b32 {c, d}, h23;\n\t"
      "cvt.f32.f16 %0, a;\n\t"
      "cvt.f32.f16 %1, b;\n\t"
      "cvt.f32.f16 %2, c;\n\t"
      "cvt.f32.f16 %3, d;\n\t}"
      : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
      : "r"(w));
  return r;
}

__device__ __forceinline__ float ld_dsmem(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ bool warp_wait_dec(uint32_t bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}

template <int G>
__global__ void __launch_bounds__(kThreads) k_attn_decode(const __grid_constant__ CUtensorMap tmK,
                                                          const __grid_constant__ CUtensorMap tmV,
                                                          const DecArgs a) {
  extern __shared__ uint8_t smem_raw[];
  DecSmem<G>& sm = *reinterpret_cast<DecSmem<G>*>(smem_align1024(smem_raw));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int cl = (int)(blockIdx.x / kNS);          // cluster = (sequence, KV head)
  const int b = cl / a.Hkv, g = cl % a.Hkv;
  int L = a.len[b];
  if (L < 0 || L > a.Lmax) {
    if (threadIdx.x == 0 && rank == 0) atomicOr(&g_dec_error, DEV_ERR_CHECK);
    L = -1;                                         // nothing is written for this sequence
  }
  // this CTA's keys [lo, hi): the rank-th slice, in whole 32-key tiles
  const int Lc = L > 0 ? L : 0;
  const int chunk = ((Lc + 32 * kNS - 1) / (32 * kNS)) * 32;
  const int lo = min(Lc, (int)rank * chunk), hi = min(Lc, lo + chunk);
  const int ntile = (hi - lo + 31) / 32;
  const int64_t row0 = (int64_t)b * a.Lmax;         // the sequence's first cache row
  const int h0 = g * G;

  const float* skg = a.sk + (size_t)g * a.T + row0;
  const float* svg = a.sv + (size_t)g * a.T + row0;
  // tile t of this CTA (keys lo + 32 t ..): K and V boxes and both scale
  // rows into consumer warp t % kCW's slot
  auto issue = [&](int t) {
    const int w = t % kCW, s = (t / kCW) % kSlots, j0 = lo + 32 * t;
    const uint32_t full = smem_u32(&sm.bars.full[w][s]);
    mbar_arrive_expect_tx(full, 2 * kTileB + 256);
    tma_load_2d(smem_u32(sm.kt[w][s]), &tmK, full, g * kD, (int)(row0 + j0));
    tma_load_2d(smem_u32(sm.vt[w][s]), &tmV, full, g * kD, (int)(row0 + j0));
    bulk_load(smem_u32(sm.ks[w][s]), skg + j0, 128, full);
    bulk_load(smem_u32(sm.vs[w][s]), svg + j0, 128, full);
  };
  const int first = min(ntile, kCW * kSlots);   // the first round: every slot starts empty
  if (threadIdx.x == 0) {
    for (int w = 0; w < kCW; ++w)
      for (int s = 0; s < kSlots; ++s) {
        mbar_init(smem_u32(&sm.bars.full[w][s]), 1);
        mbar_init(smem_u32(&sm.bars.empty[w][s]), 1);
      }
    fence_barrier_init();
    // the first round's loads go out while the query rows are staged
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    for (int t = 0; t < first; ++t) issue(t);
  }
  for (int i = threadIdx.x; i < G * kD; i += kThreads) {
    const int h = i / kD, d = i % kD;
    sm.qs[d][h] = __uint_as_float((uint32_t)a.q[(size_t)b * a.Hq * kD + (size_t)(h0 + h) * kD + d] << 16) *
                  kQScale;
  }
  __syncthreads();

  if (warp == 0) {
    // ---------------------------------------------------- TMA producer ----
    if (lane == 0) {
      int t = first;
      for (; t < ntile; ++t) {
        const int w = t % kCW, i = t / kCW, s = i % kSlots;
        if (!mbar_wait(smem_u32(&sm.bars.empty[w][s]), ((i / kSlots) & 1) ^ 1)) {
          atomicOr(&g_dec_error, DEV_ERR_TIMEOUT);
          break;
        }
        issue(t);
      }
      // every copy issued has landed before the CTA goes on (bounded)
      for (int w = 0; w < kCW; ++w)
        for (int s = 0; s < kSlots; ++s) {
          const int uses = t > w + kCW * s ? (t - w - kCW * s + kCW * kSlots - 1) / (kCW * kSlots) : 0;
          if (uses > 0) (void)mbar_wait(smem_u32(&sm.bars.full[w][s]), (uses - 1) & 1);
        }
    }
  } else {
    // ------------------------------------------------- consumer warps -----
    const int cw = warp - 1;
    float m[G], lsum[G];
    float2 o01[G], o23[G];   // this lane's channels 4 lane .. 4 lane + 3
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m[h] = -INFINITY;
      lsum[h] = 0.f;
      o01[h] = make_float2(0.f, 0.f);
      o23[h] = make_float2(0.f, 0.f);
    }
    for (int t = cw, i = 0; t < ntile; t += kCW, ++i) {
      const int s = i % kSlots;
      if (!warp_wait_dec(smem_u32(&sm.bars.full[cw][s]), (i / kSlots) & 1)) {
        if (lane == 0) atomicOr(&g_dec_error, DEV_ERR_TIMEOUT);
        break;
      }
      const int n = min(32, hi - (lo + 32 * t));
      const bool valid = lane < n;
      // ---- logits: lane = key; head pairs on packed fp32 lanes, four
      // partial sums per pair (dimensions mod 4) for independent chains
      float2 zp[4][(G + 1) / 2];
#pragma unroll
      for (int e = 0; e < 4; ++e)
#pragma unroll
        for (int h2 = 0; h2 < (G + 1) / 2; ++h2) zp[e][h2] = make_float2(0.f, 0.f);
      const uint8_t* krow = sm.kt[cw][s] + lane * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 kw = *reinterpret_cast<const uint4*>(krow + ((c ^ (lane & 7)) << 4));
        const uint32_t ww[4] = {kw.x, kw.y, kw.z, kw.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float4 k4 = dec4(ww[u]);
          const float kv[4] = {k4.x, k4.y, k4.z, k4.w};
          const int d = 16 * c + 4 * u;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (G == 1) {
              zp[e][0].x = fmaf(sm.qs[d + e][0], kv[e], zp[e][0].x);
            } else {
#pragma unroll
              for (int h2 = 0; h2 < G / 2; ++h2)
                zp[e][h2] = ffma2(make_float2(sm.qs[d + e][2 * h2], sm.qs[d + e][2 * h2 + 1]),
                                  make_float2(kv[e], kv[e]), zp[e][h2]);
            }
          }
        }
      }
      float2 z2[(G + 1) / 2];
#pragma unroll
      for (int h2 = 0; h2 < (G + 1) / 2; ++h2) z2[h2] = fadd2(fadd2(zp[0][h2], zp[1][h2]), fadd2(zp[2][h2], zp[3][h2]));
      const float skj = sm.ks[cw][s][lane], svj = sm.vs[cw][s][lane];
      // ---- online softmax per head (log2 units)
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float zh = ((h & 1) ? z2[h >> 1].y : z2[h >> 1].x) * skj;
        const float tmax = warp_max(valid ? zh : -INFINITY);
        const float m_new = fmaxf(m[h], tmax);
        const float alpha = ex2(m[h] - m_new);       // 0 on the first tile (m = -inf)
        m[h] = m_new;
        const float p = valid ? ex2(zh - m_new) : 0.f;
        lsum[h] = lsum[h] * alpha + p;
        sm.pw[cw][lane][h] = p * svj;
        if (alpha != 1.0f) {
          o01[h] = fmul2(o01[h], make_float2(alpha, alpha));
          o23[h] = fmul2(o23[h], make_float2(alpha, alpha));
        }
      }
      __syncwarp();
      // ---- P.V: lane = channels; row kk's 16-byte chunk lane/4 sits at
      // (lane/4) ^ (kk & 7)
      const uint8_t* vt = sm.vt[cw][s] + 4 * (lane & 3);
#pragma unroll 8
      for (int kk = 0; kk < n; ++kk) {
        const uint32_t vw = *reinterpret_cast<const uint32_t*>(vt + kk * 128 + (((lane >> 2) ^ (kk & 7)) << 4));
        const float4 v4 = dec4(vw);
        const float2 v01 = make_float2(v4.x, v4.y), v23 = make_float2(v4.z, v4.w);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float wk = sm.pw[cw][kk][h];
          o01[h] = ffma2(make_float2(wk, wk), v01, o01[h]);
          o23[h] = ffma2(make_float2(wk, wk), v23, o23[h]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.bars.empty[cw][s]));
    }
    // ---- this warp's state
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float l = warp_sum(lsum[h]);
      if (lane == 0) {
        sm.wm[cw][h] = m[h];
        sm.wl[cw][h] = l;
      }
      *reinterpret_cast<float4*>(&sm.wo[cw][h][4 * lane]) = make_float4(o01[h].x, o01[h].y, o23[h].x, o23[h].y);
    }
  }
  __syncthreads();
  // ---- merge the warps
  for (int i = threadIdx.x; i < G * kD; i += kThreads) {
    const int h = i / kD, d = i % kD;
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kCW; ++w) mx = fmaxf(mx, sm.wm[w][h]);
    float l = 0.f, od = 0.f;
    if (mx != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kCW; ++w) {
        const float f = ex2(sm.wm[w][h] - mx);   // 0 for a warp without keys
        l += sm.wl[w][h] * f;
        od += sm.wo[w][h][d] * f;
      }
    }
    sm.co[h][d] = od;
    if (d == 0) {
      sm.cm[h] = mx;
      sm.cl[h] = l;
    }
  }
  // ---- merge the cluster's CTAs: CTA r combines and writes the r-th
  // kNS-th of the G x 128 outputs, reading every CTA's state through
  // distributed shared memory; then every CTA's shared memory stays alive
  // until all have read it
  cluster_sync();
  if (L >= 0) {
    constexpr int kPer = G * kD / kNS;
    static_assert(G * kD % kNS == 0, "outputs split evenly over the cluster");
    for (int i = (int)rank * kPer + threadIdx.x; i < ((int)rank + 1) * kPer; i += kThreads) {
      const int h = i / kD, d = i % kD;
      float cmr[kNS];
      float mx = -INFINITY;
#pragma unroll
      for (int r = 0; r < kNS; ++r) {
        cmr[r] = ld_dsmem(mapa_shared(smem_u32(&sm.cm[h]), r));
        mx = fmaxf(mx, cmr[r]);
      }
      float l = 0.f, od = 0.f;
      if (mx != -INFINITY) {
#pragma unroll
        for (int r = 0; r < kNS; ++r) {
          const float f = ex2(cmr[r] - mx);
          l += ld_dsmem(mapa_shared(smem_u32(&sm.cl[h]), r)) * f;
          od += ld_dsmem(mapa_shared(smem_u32(&sm.co[h][d]), r)) * f;
        }
      }
      const float y = l > 0.f ? __fdiv_rn(od, l) : 0.f;
      a.o[(size_t)b * a.Hq * kD + (size_t)(h0 + h) * kD + d] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
    }
  }
  cluster_sync();
}

template <int G>
cudaError_t launch_g(const CUtensorMap& tk, const CUtensorMap& tv, const DecArgs& a, cudaStream_t st) {
  const size_t smem = sizeof(DecSmem<G>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(k_attn_decode<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3((unsigned)((int64_t)a.B * a.Hkv * kNS));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kNS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_attn_decode<G>, tk, tv, a);
}

}  // namespace

cudaError_t launch_attention_decode(int B, int Hq, int Hkv, int64_t Lmax, const int32_t* d_len,
                                    const void* q, const uint8_t* k, const float* sk, const uint8_t* v,
                                    const float* sv, void* o, cudaStream_t st) {
  DecArgs a;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Lmax = Lmax;
  a.T = (int64_t)B * Lmax;
  a.len = d_len;
  a.q = static_cast<const uint16_t*>(q);
  a.sk = sk;
  a.sv = sv;
  a.o = static_cast<uint16_t*>(o);
  CUtensorMap tk, tv;
  if (!make_map(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, k, (uint64_t)Hkv * kD, (uint64_t)a.T, (uint64_t)Hkv * kD,
                kD, 32, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, v, (uint64_t)Hkv * kD, (uint64_t)a.T, (uint64_t)Hkv * kD,
                kD, 32, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  cudaError_t e;
  switch (Hq / Hkv) {
    case 1: e = launch_g<1>(tk, tv, a, st); break;
    case 2: e = launch_g<2>(tk, tv, a, st); break;
    case 4: e = launch_g<4>(tk, tv, a, st); break;
    case 8: e = launch_g<8>(tk, tv, a, st); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t dec_read_clear_error(uint32_t* out, cudaStream_t st) {
  uint32_t v = 0, z = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_dec_error, sizeof v, 0, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess && v) e = cudaMemcpyToSymbolAsync(g_dec_error, &z, sizeof z, 0, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  *out = v;
  return e;
}

}  // namespace fp8bw

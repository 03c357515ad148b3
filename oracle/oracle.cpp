// Oracle for the blockwise-scaled FP8 linear layer — TEST INFRASTRUCTURE ONLY.
//
// A plain, slow, CPU implementation of what the library computes, written
// from the pages' statement of the method and from the definitions of the
// formats involved.  It shares no code, header, table or constant with the
// CUDA library and must never be linked into it: only the tests, the smoke
// check and the benchmark's CPU-baseline leg load it.
//
// Sources (page title, section):
//  [P1] "NVIDIA NeMo RL erreicht 48% Geschwindigkeitssteigerung mit End-to-End
//       FP8-Präzisionstraining", section "Der technische Durchbruch": the
//       recipe quantizes to E4M3 with one scale per 128x128 weight block and
//       one per 1x128 activation block; linear layers do FP8 math.
//       Section "Leistungsgewinne in der Praxis": scales are recalibrated
//       after every training step.  Section "Warum dies für die KI-Ökonomie
//       wichtig ist": optional power-of-2 scale factors.
//  [P2] "FP8 Trainingsinfrastructuur", section "Het landschap van numerieke
//       precisie": E4M3 has 4 exponent bits, 3 mantissa bits and values up to
//       +-448.
//
// Readings taken where the pages are silent:
//  * block scale s = fp32(amax / 448) (current scaling), s = 1 for an
//    all-zero block;
//  * power-of-2 mode: s = 2^e with e the smallest integer such that
//    amax <= 448 * 2^e, clamped to [-127, 127]; s = 1 for an all-zero block;
//  * codes: q = E4M3_RNE_satfinite( fp32( fp32(x) / s ) ) — IEEE fp32
//    division, then round-to-nearest-even onto the E4M3 grid, magnitudes
//    beyond 448 saturate to 448, the sign of zero is kept;
//  * GEMM reference: fp64 sum of products of the dequantized operands.
//
// Parity status: every function here is pinned by tests/test_oracle_*.py
// (exhaustive code table, closed-form points, library cross-checks,
// hand-worked blocks, invariants, brute force).  No function is unpinned.
//
// Build: g++ -O2 -std=c++17 -fPIC -shared -ffp-contract=off -fopenmp (no
// -ffast-math: IEEE division and subnormals must be kept).  OpenMP only
// splits independent blocks / output elements across threads; no value's
// arithmetic changes with the thread count.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <cstdlib>
#include <omp.h>

namespace {

// ---------------------------------------------------------------- bf16 ----
// A bf16 value is the upper 16 bits of an IEEE binary32 value.
float bf16_bits_to_float(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return f;
}

// fp32 -> bf16 with round-to-nearest-even (NaN kept as a quiet NaN).
uint16_t float_to_bf16_bits(float f) {
  uint32_t u;
  std::memcpy(&u, &f, sizeof u);
  if (std::isnan(f)) return static_cast<uint16_t>((u >> 16) | 0x40);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return static_cast<uint16_t>(u >> 16);
}

// ---------------------------------------------------------------- E4M3 ----
// E4M3 [P2]: sign bit, 4 exponent bits, 3 mantissa bits, largest value 448.
// 448 = 1.75 * 2^8 is exponent field 15 with mantissa 110, so the exponent
// bias is 7; exponent field 15 with mantissa 111 is NaN (no infinities).
//   field e in 1..15: (1 + m/8) * 2^(e-7)
//   field e == 0    : (m/8) * 2^(1-7) = m * 2^-9   (subnormals)
double e4m3_decode(uint8_t code) {
  int sign = (code >> 7) & 1;
  int e = (code >> 3) & 0xF;
  int m = code & 0x7;
  if (e == 15 && m == 7) return std::nan("");
  double mag;
  if (e == 0)
    mag = std::ldexp(static_cast<double>(m), -9);
  else
    mag = std::ldexp(1.0 + m / 8.0, e - 7);
  return sign ? -mag : mag;
}

// Round a finite fp32 value to the E4M3 grid, ties to even, saturating to
// +-448.  The grid spacing in [2^E, 2^(E+1)) is 2^(E-3) for E >= -6 and 2^-9
// below 2^-6 (the subnormal range), so v / spacing is an integer k whose
// parity is the parity of the mantissa field.  Rounding k to the nearest
// integer with ties to even is therefore the E4M3 round-to-nearest-even.
uint8_t e4m3_encode(float v) {
  uint8_t sign = std::signbit(v) ? 0x80 : 0x00;
  if (std::isnan(v)) return static_cast<uint8_t>(sign | 0x7F);
  double a = std::fabs(static_cast<double>(v));
  if (a >= 448.0) return static_cast<uint8_t>(sign | 0x7E);  // saturate
  if (a == 0.0) return sign;
  int E;  // a = f * 2^E2 with f in [0.5,1)  =>  a in [2^(E2-1), 2^E2)
  std::frexp(a, &E);
  E -= 1;                          // a in [2^E, 2^(E+1))
  int spacing_exp = (E < -6) ? -9 : E - 3;
  double k = std::ldexp(a, -spacing_exp);      // exact (power-of-2 scaling)
  double r = std::nearbyint(k);                // default mode: ties to even
  // r * 2^spacing_exp is the rounded magnitude, never above 448.
  //  subnormal range: value r * 2^-9, r in 0..8; r == 8 is 2^-6, the first
  //    normal (field 1, mantissa 0), which is also code 8;
  //  normal range: value (r/8) * 2^E, r in 8..16; the code is
  //    (E + 7) * 8 + (r - 8), and r == 16 carries into the next exponent.
  long r_int = static_cast<long>(r);
  if (r_int == 0) return sign;
  long code = (E < -6) ? r_int : (E + 7) * 8 + (r_int - 8);
  return static_cast<uint8_t>(sign | code);
}

// ---------------------------------------------------------------- E5M2 ----
// E5M2 ([P2] "Het landschap van numerieke precisie": the gradient format of
// the per-tensor recipe): sign bit, 5 exponent bits (bias 15), 2 mantissa
// bits; exponent field 31 holds +-inf (mantissa 0) and NaN; the largest
// finite value is 1.75 * 2^15 = 57344.
//   field e in 1..30: (1 + m/4) * 2^(e-15)
//   field e == 0    : (m/4) * 2^(1-15) = m * 2^-16   (subnormals)
double e5m2_decode(uint8_t code) {
  int sign = (code >> 7) & 1;
  int e = (code >> 2) & 0x1F;
  int m = code & 0x3;
  double mag;
  if (e == 31) {
    if (m != 0) return std::nan("");
    mag = INFINITY;
  } else if (e == 0) {
    mag = std::ldexp(static_cast<double>(m), -16);
  } else {
    mag = std::ldexp(1.0 + m / 4.0, e - 15);
  }
  return sign ? -mag : mag;
}

// Round a finite fp32 value to the E5M2 grid, ties to even, saturating to
// +-57344 (as the E4M3 encoder: the spacing in [2^E, 2^(E+1)) is 2^(E-2)
// for E >= -14 and 2^-16 below, and the parity of v / spacing is the parity
// of the mantissa field).  NaN keeps its sign with code 0x7F.
uint8_t e5m2_encode(float v) {
  uint8_t sign = std::signbit(v) ? 0x80 : 0x00;
  if (std::isnan(v)) return static_cast<uint8_t>(sign | 0x7F);
  double a = std::fabs(static_cast<double>(v));
  if (a >= 57344.0) return static_cast<uint8_t>(sign | 0x7B);  // saturate
  if (a == 0.0) return sign;
  int E;
  std::frexp(a, &E);
  E -= 1;                          // a in [2^E, 2^(E+1))
  int spacing_exp = (E < -14) ? -16 : E - 2;
  double k = std::ldexp(a, -spacing_exp);
  double r = std::nearbyint(k);    // ties to even
  //  subnormal range: r * 2^-16, r in 0..4 (r == 4 is 2^-14 = code 4);
  //  normal range: (r/4) * 2^E, r in 4..8, code (E + 15) * 4 + (r - 4).
  long r_int = static_cast<long>(r);
  if (r_int == 0) return sign;
  long code = (E < -14) ? r_int : (E + 15) * 4 + (r_int - 4);
  return static_cast<uint8_t>(sign | code);
}

// Element formats: 0 = E4M3 (largest value 448), 1 = E5M2 (57344).
constexpr int FMT_E4M3 = 0;
constexpr int FMT_E5M2 = 1;

double fmt_max(int fmt) { return fmt == FMT_E5M2 ? 57344.0 : 448.0; }
double decode(uint8_t code, int fmt) { return fmt == FMT_E5M2 ? e5m2_decode(code) : e4m3_decode(code); }
uint8_t encode(float v, int fmt) { return fmt == FMT_E5M2 ? e5m2_encode(v) : e4m3_encode(v); }

// ------------------------------------------------------------ block scale --
constexpr int MODE_FP32 = 0;
constexpr int MODE_POW2 = 1;

float block_scale(float amax, int mode, int fmt = FMT_E4M3) {
  if (amax == 0.0f) return 1.0f;
  const float qmax = static_cast<float>(fmt_max(fmt));
  if (mode == MODE_FP32) return amax / qmax;  // IEEE fp32 division
  // Power of two: the smallest e with amax <= qmax * 2^e (found by search,
  // which is the definition), clamped to the UE8M0-representable [-127,127].
  int e = -127;
  while (e < 127 && static_cast<double>(amax) > std::ldexp(static_cast<double>(qmax), e)) ++e;
  return static_cast<float>(std::ldexp(1.0, e));
}

uint8_t quant_one(uint16_t xb, float s, int fmt = FMT_E4M3) {
  float x = bf16_bits_to_float(xb);
  float t = x / s;  // IEEE fp32 division, round to nearest even
  return encode(t, fmt);
}

}  // namespace

extern "C" {

// Thread count of the OpenMP loops below (timing of the CPU baseline only;
// no value depends on it).
void orc_set_threads(int n) { omp_set_num_threads(n > 0 ? n : 1); }
int orc_max_threads() { return omp_get_max_threads(); }

double orc_e4m3_decode(uint8_t code) { return e4m3_decode(code); }
uint8_t orc_e4m3_encode(float v) { return e4m3_encode(v); }
double orc_e5m2_decode(uint8_t code) { return e5m2_decode(code); }
uint8_t orc_e5m2_encode(float v) { return e5m2_encode(v); }
float orc_block_scale(float amax, int mode) { return block_scale(amax, mode); }
float orc_block_scale_fmt(float amax, int mode, int fmt) { return block_scale(amax, mode, fmt); }
float orc_bf16_to_float(uint16_t b) { return bf16_bits_to_float(b); }
uint16_t orc_float_to_bf16(float f) { return float_to_bf16_bits(f); }

void orc_e4m3_encode_array(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_encode(v[i]);
}

void orc_e5m2_encode_array(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e5m2_encode(v[i]);
}

// Activation quantization, 1x128 blocks [P1 "Der technische Durchbruch"].
//   x      : bf16 bits, row-major [M][ldx] (first K columns used)
//   q_row  : [M][K] codes; s_row : [K/128][M] scales (chunk-major)
//   q_col  : [K][M] codes of the column-wise copy, whose blocks are 128
//            consecutive rows of one column; s_col : [M/128][K].
//   The column-wise copy is quantized from x itself, not from q_row.
//   q_col/s_col may be null (row-wise only).
//   fmt: element format of the codes (0 = E4M3, 1 = E5M2).
void orc_quant_act_1x128_fmt(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                             int mode, int fmt, uint8_t* q_row, float* s_row,
                             uint8_t* q_col, float* s_col) {
  const int64_t nK = K / 128;
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t kb = 0; kb < nK; ++kb) {
      float amax = 0.0f;
      for (int64_t j = 0; j < 128; ++j) {
        float a = std::fabs(bf16_bits_to_float(x[m * ldx + kb * 128 + j]));
        if (a > amax) amax = a;
      }
      float s = block_scale(amax, mode, fmt);
      s_row[kb * M + m] = s;
      for (int64_t j = 0; j < 128; ++j)
        q_row[m * K + kb * 128 + j] = quant_one(x[m * ldx + kb * 128 + j], s, fmt);
    }
  }
  if (!q_col) return;
  const int64_t nM = M / 128;
#pragma omp parallel for schedule(static)
  for (int64_t k = 0; k < K; ++k) {
    for (int64_t mb = 0; mb < nM; ++mb) {
      float amax = 0.0f;
      for (int64_t i = 0; i < 128; ++i) {
        float a = std::fabs(bf16_bits_to_float(x[(mb * 128 + i) * ldx + k]));
        if (a > amax) amax = a;
      }
      float s = block_scale(amax, mode, fmt);
      s_col[mb * K + k] = s;
      for (int64_t i = 0; i < 128; ++i)
        q_col[k * M + mb * 128 + i] = quant_one(x[(mb * 128 + i) * ldx + k], s, fmt);
    }
  }
}

void orc_quant_act_1x128(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                         int mode, uint8_t* q_row, float* s_row,
                         uint8_t* q_col, float* s_col) {
  orc_quant_act_1x128_fmt(x, M, K, ldx, mode, FMT_E4M3, q_row, s_row, q_col, s_col);
}

// Weight quantization, 128x128 blocks [P1 "Der technische Durchbruch"].
//   w  : bf16 bits [N][ldw]; q : [N][K]; s : [N/128][K/128];
//   qT : [K][N], the exact byte transpose of q (may be null).
void orc_quant_weight_128x128(const uint16_t* w, int64_t N, int64_t K,
                              int64_t ldw, int mode, uint8_t* q, float* s,
                              uint8_t* qT) {
  const int64_t nN = N / 128, nK = K / 128;
#pragma omp parallel for schedule(static)
  for (int64_t nb = 0; nb < nN; ++nb) {
    for (int64_t kb = 0; kb < nK; ++kb) {
      float amax = 0.0f;
      for (int64_t i = 0; i < 128; ++i)
        for (int64_t j = 0; j < 128; ++j) {
          float a = std::fabs(
              bf16_bits_to_float(w[(nb * 128 + i) * ldw + kb * 128 + j]));
          if (a > amax) amax = a;
        }
      float sc = block_scale(amax, mode);
      s[nb * nK + kb] = sc;
      for (int64_t i = 0; i < 128; ++i)
        for (int64_t j = 0; j < 128; ++j)
          q[(nb * 128 + i) * K + kb * 128 + j] =
              quant_one(w[(nb * 128 + i) * ldw + kb * 128 + j], sc);
    }
  }
  if (!qT) return;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) qT[k * N + n] = q[n * K + k];
}

// Per-tensor delayed scaling [P2 "Transformer Engine: de softwarebasis" and
// "Scaling-strategieën en stabiliteit"]: one scale for the whole tensor,
// taken from the largest absolute values observed in earlier iterations
// (the page's recipe keeps a history of 16 and takes its maximum, margin 0),
// not from the tensor being quantized; this call's amax then enters the
// history.  The scale rule applied to that maximum is the block rule above.
//   x     : bf16 bits [M][ldx], first K columns
//   hist  : [H] amax history, newest first, updated in place:
//           hist'[0] = amax(x), hist'[i] = hist[i-1] for 0 < i < H
//   q     : [M][K] codes, q = encode(fp32(x) / s); values beyond the
//           format's largest saturate (the history may under-estimate)
//   qT    : [K][M] the byte transpose of q (one scale: the column-wise copy
//           is the transpose), may be null
//   scale : s = block_scale(max(hist), mode, fmt)
//   amax  : max |x| of this call
// A NaN, in x or in hist, never wins a maximum (the comparisons below are
// false for NaN).
void orc_quant_tensor_delayed(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                              int mode, int fmt, float* hist, int32_t H, uint8_t* q,
                              uint8_t* qT, float* scale, float* amax) {
  float h = 0.0f;
  for (int32_t i = 0; i < H; ++i)
    if (hist[i] > h) h = hist[i];
  const float s = block_scale(h, mode, fmt);
  float a = 0.0f;
  for (int64_t m = 0; m < M; ++m)
    for (int64_t k = 0; k < K; ++k) {
      const float v = std::fabs(bf16_bits_to_float(x[m * ldx + k]));
      if (v > a) a = v;
      q[m * K + k] = quant_one(x[m * ldx + k], s, fmt);
    }
  if (qT)
    for (int64_t m = 0; m < M; ++m)
      for (int64_t k = 0; k < K; ++k) qT[k * M + m] = q[m * K + k];
  for (int32_t i = H - 1; i > 0; --i) hist[i] = hist[i - 1];
  if (H > 0) hist[0] = a;
  *scale = s;
  *amax = a;
}

// Scale of operand B for output column n at K-chunk kb, per GEMM kind:
//   kind 0 (fprop): 128x128 block grid [N/128][K/128]
//   kind 1 (dgrad): the weight's own grid, read transposed: [K/128][N/128]
//   kind 2 (wgrad): 1x128 blocks along the contraction, [K/128][N]
static double b_scale(int kind, const float* sB, int64_t N, int64_t K,
                      int64_t n, int64_t kb) {
  if (kind == 0) return sB[(n / 128) * (K / 128) + kb];
  if (kind == 1) return sB[kb * (N / 128) + n / 128];
  return sB[kb * N + n];
}

// The decoded value of every code of one format, taken from the decoder
// above once (a lookup saves the per-product decode in the GEMM references;
// the values are the decoder's own).
struct DecodeTable {
  double v[2][256];
  DecodeTable() {
    for (int c = 0; c < 256; ++c) {
      v[FMT_E4M3][c] = e4m3_decode(static_cast<uint8_t>(c));
      v[FMT_E5M2][c] = e5m2_decode(static_cast<uint8_t>(c));
    }
  }
};

static const double* decode_table(int fmt) {
  static const DecodeTable t;  // initialised once, thread-safe
  return t.v[fmt == FMT_E5M2 ? FMT_E5M2 : FMT_E4M3];
}

// One output element of the GEMM reference over K-chunks [kb0, kb1):
// sum_k (qA[m][k] * sA[k/128][m]) * (qB[n][k] * sB(n, k/128)) in fp64 from
// the dequantized operands, and sum_k |a * b|.
// fa / fb: element formats of the A and B codes (0 = E4M3, 1 = E5M2).
static void ref_element(int kind, int64_t M, int64_t N, int64_t K,
                        const uint8_t* A, const float* sA, const uint8_t* B,
                        const float* sB, int64_t kb0, int64_t kb1, int64_t m,
                        int64_t n, double* y, double* yabs, int fa = FMT_E4M3,
                        int fb = FMT_E4M3) {
  const double* da = decode_table(fa);
  const double* db = decode_table(fb);
  double acc = 0.0, aacc = 0.0;
  for (int64_t kb = kb0; kb < kb1; ++kb) {
    double sa = sA[kb * M + m];
    double sb = b_scale(kind, sB, N, K, n, kb);
    for (int64_t j = 0; j < 128; ++j) {
      int64_t k = kb * 128 + j;
      double a = da[A[m * K + k]] * sa;
      double b = db[B[n * K + k]] * sb;
      acc += a * b;
      aacc += std::fabs(a * b);
    }
  }
  *y = acc;
  *yabs = aacc;
}

// GEMM reference [P1 "Der technische Durchbruch": linear layers do FP8 math]
// over rows [m0,m1) x cols [n0,n1); y/yabs laid out [m1-m0][n1-n0].
//   A : [M][K] codes (K-major), sA : [K/128][M]
//   B : [N][K] codes (K-major), sB : per kind (see b_scale)
void orc_gemm_ref_tile_fmt(int kind, int fa, int fb, int64_t M, int64_t N, int64_t K,
                           const uint8_t* A, const float* sA, const uint8_t* B,
                           const float* sB, int64_t m0, int64_t m1, int64_t n0,
                           int64_t n1, double* y, double* yabs) {
  const int64_t W = n1 - n0;
#pragma omp parallel for schedule(static)
  for (int64_t m = m0; m < m1; ++m)
    for (int64_t n = n0; n < n1; ++n)
      ref_element(kind, M, N, K, A, sA, B, sB, 0, K / 128, m, n,
                  &y[(m - m0) * W + (n - n0)], &yabs[(m - m0) * W + (n - n0)], fa, fb);
}

void orc_gemm_ref_tile(int kind, int64_t M, int64_t N, int64_t K,
                       const uint8_t* A, const float* sA, const uint8_t* B,
                       const float* sB, int64_t m0, int64_t m1, int64_t n0,
                       int64_t n1, double* y, double* yabs) {
  orc_gemm_ref_tile_fmt(kind, FMT_E4M3, FMT_E4M3, M, N, K, A, sA, B, sB, m0, m1, n0, n1, y, yabs);
}

// Grouped (MoE expert) GEMM reference [P1 "Leistungsgewinne in der Praxis":
// the recipe also trains the Qwen3-30B mixture-of-experts model].  Expert g
// owns token rows [off[g], off[g+1]) of the permuted token matrix; every
// offset is a multiple of 128 (segments zero-padded to whole blocks).
//   kind 0/1: rows m of the output use expert g(m)'s weight
//             B + g*N*K, sB + g*(N/128)*(K/128); y over rows [m0,m1)
//             (rows at or beyond off[G] are not part of the result).
//   kind 2  : output dW_g [N][K] for one expert g = `expert`: the
//             contraction runs over that expert's token chunks only; A is
//             [N][Mtot] (K-major in tokens), sA [Mtot/128][N], B [K][Mtot],
//             sB [Mtot/128][K]; y over rows [m0,m1) x cols [n0,n1) of dW_g.
//             An empty expert gives exact zeros.
void orc_grouped_gemm_ref_tile(int kind, int32_t G, const int32_t* off,
                               int64_t Mtot, int64_t N, int64_t K,
                               const uint8_t* A, const float* sA,
                               const uint8_t* B, const float* sB,
                               int32_t expert, int64_t m0, int64_t m1,
                               int64_t n0, int64_t n1, double* y,
                               double* yabs) {
  const int64_t W = n1 - n0;
  if (kind == 2) {
    // GEMM dims: rows N, cols K, contraction Mtot.
    int64_t kb0 = off[expert] / 128, kb1 = off[expert + 1] / 128;
#pragma omp parallel for schedule(static)
    for (int64_t m = m0; m < m1; ++m)
      for (int64_t n = n0; n < n1; ++n)
        ref_element(2, N, K, Mtot, A, sA, B, sB, kb0, kb1, m, n,
                    &y[(m - m0) * W + (n - n0)],
                    &yabs[(m - m0) * W + (n - n0)]);
    return;
  }
#pragma omp parallel for schedule(static)
  for (int64_t m = m0; m < m1; ++m) {
    int32_t g = 0;
    while (g < G && !(m >= off[g] && m < off[g + 1])) ++g;
    for (int64_t n = n0; n < n1; ++n) {
      double* py = &y[(m - m0) * W + (n - n0)];
      double* pa = &yabs[(m - m0) * W + (n - n0)];
      if (g == G) { *py = 0.0; *pa = 0.0; continue; }
      const uint8_t* Bg = B + static_cast<int64_t>(g) * N * K;
      const float* sBg = sB + static_cast<int64_t>(g) * (N / 128) * (K / 128);
      ref_element(kind, Mtot, N, K, A, sA, Bg, sBg, 0, K / 128, m, n, py, pa);
    }
  }
}

// Same reference at a list of (m, n) points.
void orc_gemm_ref_points(int kind, int64_t M, int64_t N, int64_t K,
                         const uint8_t* A, const float* sA, const uint8_t* B,
                         const float* sB, const int64_t* pm, const int64_t* pn,
                         int64_t npts, double* y, double* yabs) {
  for (int64_t p = 0; p < npts; ++p)
    orc_gemm_ref_tile(kind, M, N, K, A, sA, B, sB, pm[p], pm[p] + 1, pn[p],
                      pn[p] + 1, y + p, yabs + p);
}

// Diagnostic only (never a gate): the fp32 per-chunk promotion a tensor-core
// kernel performs — fp32 chunk sums, times fp32(sa*sb), accumulated in fp32,
// then rounded to bf16.  Returns bf16 bits [m1-m0][n1-n0].
void orc_gemm_mimic_tile(int kind, int64_t M, int64_t N, int64_t K,
                         const uint8_t* A, const float* sA, const uint8_t* B,
                         const float* sB, int64_t m0, int64_t m1, int64_t n0,
                         int64_t n1, uint16_t* y) {
  const int64_t nK = K / 128;
  const int64_t W = n1 - n0;
  for (int64_t m = m0; m < m1; ++m)
    for (int64_t n = n0; n < n1; ++n) {
      float acc = 0.0f;
      for (int64_t kb = 0; kb < nK; ++kb) {
        float part = 0.0f;
        for (int64_t j = 0; j < 128; ++j) {
          int64_t k = kb * 128 + j;
          part += static_cast<float>(e4m3_decode(A[m * K + k]) *
                                     e4m3_decode(B[n * K + k]));
        }
        float sc = sA[kb * M + m] *
                   static_cast<float>(b_scale(kind, sB, N, K, n, kb));
        acc += part * sc;
      }
      y[(m - m0) * W + (n - n0)] = float_to_bf16_bits(acc);
    }
}

// BF16 reference GEMM (the comparison path): y = sum_k a[m][k] * b[n][k] in
// fp64 over bf16 operands, both K-major.
void orc_gemm_bf16_ref_tile(int64_t M, int64_t N, int64_t K,
                            const uint16_t* A, const uint16_t* B, int64_t m0,
                            int64_t m1, int64_t n0, int64_t n1, double* y,
                            double* yabs) {
  (void)M; (void)N;
  const int64_t W = n1 - n0;
  for (int64_t m = m0; m < m1; ++m)
    for (int64_t n = n0; n < n1; ++n) {
      double acc = 0.0, aacc = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        double p = static_cast<double>(bf16_bits_to_float(A[m * K + k])) *
                   static_cast<double>(bf16_bits_to_float(B[n * K + k]));
        acc += p;
        aacc += std::fabs(p);
      }
      y[(m - m0) * W + (n - n0)] = acc;
      yabs[(m - m0) * W + (n - n0)] = aacc;
    }
}

// One bf16 unit in the last place of v: the gap between the two bf16 values
// around |v| (8 significant bits; smallest subnormal step 2^-133).
double orc_bf16_ulp(double v) {
  double a = std::fabs(v);
  if (a < std::ldexp(1.0, -126)) return std::ldexp(1.0, -133);
  int E;
  std::frexp(a, &E);  // a in [2^(E-1), 2^E)
  return std::ldexp(1.0, E - 1 - 7);
}

// The GEMM acceptance rule: |y - yref| <= rel * yabs + 1 bf16 ulp(yref).
// y are bf16 bits.  Returns the number of violations; the worst ratio of
// error to allowance is written to *worst.
int64_t orc_check_tol(const uint16_t* y, const double* yref,
                      const double* yabs, int64_t n, double rel,
                      double* worst) {
  int64_t bad = 0;
  double w = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    double g = bf16_bits_to_float(y[i]);
    double err = std::fabs(g - yref[i]);
    double allow = rel * yabs[i] + orc_bf16_ulp(yref[i]);
    if (!(err <= allow)) ++bad;
    double r = err / allow;
    if (std::isnan(g)) r = INFINITY;
    if (r > w) w = r;
  }
  if (worst) *worst = w;
  return bad;
}

// -------------------------------------------------------------- attention --
// FP8 attention forward [P1 "Leistungsgewinne in der Praxis": the recipe
// extends FP8 to the KV cache and the attention operations; no granularity
// or numerics are given].  Readings taken, each the recipe's own rule carried
// over:
//  * every FP8 operand is E4M3 with 1x128 blocks along its contraction
//    ("Der technische Durchbruch": 1x128 for activations): Q and K carry one
//    scale per token and head (head dimension 128 = one block), V is the
//    column-wise copy of the activation quantizer (one scale per 128 tokens
//    of one channel, codes stored channel-major [H*128][T]), and the softmax
//    numerator P carries one scale per query row and 128-key block;
//  * logits z_j = (q^ . k^_j) / sqrt(128) from the dequantized operands,
//    p_j = exp(z_j - max_j z_j) over the query's keys, l = sum_j p_j taken
//    from the unquantized p;
//  * P's block scale follows the FP32 rule s_b = amax_b / 448 and its codes
//    are E4M3(fp32(p_j / s_b)); the power-of-two rule is not used for P,
//    because p / amax is what a streaming kernel can reproduce (it meets the
//    keys relative to a running maximum, which scales a block by a constant);
//  * O_d = sum_j p^_j v^_{j,d} / l, p^_j = decode(code_j) * s_b.
// One E4M3 step if the code of tq (tq >= 0) is ambiguous, i.e. tq lies
// within relative distance eta of the rounding midpoint next to its code;
// else 0.
static double midpoint_step(const double* dec, double tq, uint8_t code, double eta) {
  if (!(tq < 448.0)) return 0.0;
  const double v = dec[code];
  const double lo_g = v <= tq ? v : (code > 0 ? dec[code - 1] : 0.0);
  const double hi_g = v <= tq ? (code < 0x7E ? dec[code + 1] : v) : v;
  const double mid = 0.5 * (lo_g + hi_g);
  return (hi_g > lo_g && std::fabs(tq - mid) <= eta * tq) ? hi_g - lo_g : 0.0;
}

// The power-of-2 scale rule on an fp64 amax > 0 (as block_scale: the
// smallest e with amax <= qmax 2^e, found by search, clamped to [-127, 127]).
static int pow2_exponent(double amax, double qmax) {
  int e = -127;
  while (e < 127 && amax > std::ldexp(qmax, e)) ++e;
  return e;
}

// Sequences: segment g covers tokens [off[g], off[g+1]) (multiples of 128),
// of which the first len[g] are real tokens; a query token's keys are the
// real tokens of its segment, and with `causal` only those j <= t.  Query
// head h reads key/value head h / (Hq / Hkv).
//
// For each requested (token, head) row: out[d] = O_d in fp64; oabs[d] =
// sum_j |p^_j v^_{j,d}| / l (the GEMM gate's magnitude term for P.V); and
// oflip[d] = sum over ambiguous codes of (one E4M3 step of p_j/s_b) * s_b *
// |v^_{j,d}| / l.  A code is ambiguous when p_j / s_b lies within eta of an
// E4M3 rounding midpoint, eta bounding the relative error with which an fp32
// kernel forms p_j / s_b: the tensor core's fp32 sum of the 128 code
// products (at most 2^-16 of their absolute sum), the fp32 scaling of the
// logits (2^-21 relative), the exponential (2^-21) and the running maximum
// (the largest logit error of the row).  Either rounding is then correct.
// Padding query rows (t beyond its segment's real tokens) give O = 0.
//
// mode = MODE_FP32: P's block scale is s_b = amax / 448 (the FP32 rule), and
// p_j = e^(z_j - zmax) (the reference maximum cancels out of the codes).
// mode = MODE_POW2 (the recipe's optional power-of-2 scales): s_b is the
// power-of-2 rule on the block's amax, and p_j = 2^(z_j log2 e - M) with
// the integer reference M = ceil(zmax log2 e).  Any integer reference gives
// the same codes, so a kernel may use its running maximum rounded up to an
// integer.  Where the kernel's fp32 amax can fall on the other side of a
// power-of-two boundary, the code under the other scale is also correct;
// oflip then carries the larger of the two outcomes' differences.
void orc_attention_fwd_rows(int64_t T, int32_t Hq, int32_t Hkv, int32_t nseg,
                            const int32_t* off, const int32_t* len, int32_t causal,
                            const uint8_t* q, const float* sq, const uint8_t* k,
                            const float* sk, const uint8_t* vT, const float* sv,
                            int64_t nrows, const int64_t* row_t, const int32_t* row_h,
                            double* out, double* oabs, double* oflip, int32_t mode) {
  const int64_t D = 128;
  const double* dec = decode_table(FMT_E4M3);
  const double inv_sqrt_d = 1.0 / std::sqrt(static_cast<double>(D));
  const int32_t group = Hq / Hkv;
#pragma omp parallel for schedule(dynamic)
  for (int64_t r = 0; r < nrows; ++r) {
    const int64_t t = row_t[r];
    const int32_t h = row_h[r], g = h / group;
    double* o = out + r * D;
    double* oa = oabs + r * D;
    double* of = oflip + r * D;
    for (int64_t d = 0; d < D; ++d) o[d] = oa[d] = of[d] = 0.0;
    int32_t seg = 0;
    while (seg + 1 < nseg && off[seg + 1] <= t) ++seg;
    const int64_t j0 = off[seg], jreal = off[seg] + len[seg];
    if (t >= jreal) continue;                       // a padding row
    const int64_t j1 = causal ? t + 1 : jreal;      // keys [j0, j1)
    const int64_t nk = j1 - j0;
    // logits and their error bounds
    double* z = static_cast<double*>(std::malloc(sizeof(double) * nk * 2));
    double* dz = z + nk;
    const double sqv = sq[static_cast<int64_t>(h) * T + t];
    double zmax = -INFINITY, dzmax = 0.0;
    for (int64_t j = j0; j < j1; ++j) {
      const double skv = sk[static_cast<int64_t>(g) * T + j];
      double acc = 0.0, aabs = 0.0;
      for (int64_t d = 0; d < D; ++d) {
        const double prod = dec[q[t * Hq * D + h * D + d]] * dec[k[j * Hkv * D + g * D + d]];
        acc += prod;
        aabs += std::fabs(prod);
      }
      const double c = sqv * skv * inv_sqrt_d;
      z[j - j0] = acc * c;
      dz[j - j0] = std::fabs(c) * aabs * std::ldexp(1.0, -16) + std::fabs(z[j - j0]) * std::ldexp(1.0, -21);
      if (z[j - j0] > zmax) zmax = z[j - j0];
      if (dz[j - j0] > dzmax) dzmax = dz[j - j0];
    }
    // p_j = e^(z_j - zmax) (FP32 mode); in POW2 mode p_j = 2^(z_j log2 e - M)
    // with the integer reference M = ceil(zmax log2 e): scaling every p by a
    // power of two scales its power-of-2 block scale by the same power, so
    // any integer reference gives the same codes.
    const double kLog2e = 1.0 / std::log(2.0);
    const double ref = mode == MODE_POW2 ? std::ceil(zmax * kLog2e) : 0.0;
    double l = 0.0;
    for (int64_t j = 0; j < nk; ++j) {
      z[j] = mode == MODE_POW2 ? std::exp2(z[j] * kLog2e - ref) : std::exp(z[j] - zmax);   // z now holds p
      l += z[j];
    }
    // P . V block by block (128-key blocks at absolute multiples of 128)
    for (int64_t b0 = (j0 / 128) * 128; b0 < j1; b0 += 128) {
      const int64_t lo = b0 > j0 ? b0 : j0, hi = (b0 + 128 < j1) ? b0 + 128 : j1;
      double amax = 0.0, dzb = 0.0;
      for (int64_t j = lo; j < hi; ++j)
        if (z[j - j0] > amax) { amax = z[j - j0]; dzb = dz[j - j0]; }
      // the block scale by the mode's rule (an all-zero block has s = 1);
      // in POW2 mode a kernel's fp32 amax may land on the other side of a
      // power-of-two boundary (relative error eta_s), giving the other scale
      double sb = 1.0, sb_alt = 0.0;
      if (amax > 0.0) {
        if (mode == MODE_POW2) {
          const int e = pow2_exponent(amax, 448.0);
          sb = std::ldexp(1.0, e);
          const double eta_s = dzb + 2.0 * dzmax + std::ldexp(1.0, -19);
          if (e > -127 && amax <= 448.0 * std::ldexp(1.0, e - 1) * (1.0 + eta_s)) sb_alt = std::ldexp(1.0, e - 1);
          if (e < 127 && amax >= 448.0 * sb * (1.0 - eta_s)) sb_alt = std::ldexp(1.0, e + 1);
        } else {
          // a block whose largest p is so small that amax / 448 underflows
          // (p below ~2e-321, far below fp32's range) is treated like an
          // all-zero block (s = 1): its codes are 0 under any positive scale
          sb = amax / 448.0;
          if (!(sb > 0.0)) sb = 1.0;
        }
      }
      const float* svb = sv + (b0 / 128) * (static_cast<int64_t>(Hkv) * D) + static_cast<int64_t>(g) * D;
      for (int64_t j = lo; j < hi; ++j) {
        const double pj = z[j - j0];
        const double eta = dz[j - j0] + dzb + 2.0 * dzmax + std::ldexp(1.0, -19);
        const double tq = pj / sb;
        const uint8_t code = e4m3_encode(static_cast<float>(tq));
        const double phat = dec[code] * sb;
        double amb = midpoint_step(dec, tq, code, eta) * sb;   // either rounding is correct
        if (sb_alt > 0.0) {
          const double tq2 = pj / sb_alt;
          const uint8_t code2 = e4m3_encode(static_cast<float>(tq2));
          const double d2 = std::fabs(dec[code2] * sb_alt - phat) + midpoint_step(dec, tq2, code2, eta) * sb_alt;
          if (d2 > amb) amb = d2;
        }
        for (int64_t d = 0; d < D; ++d) {
          const double vv = dec[vT[(static_cast<int64_t>(g) * D + d) * T + j]] * svb[d];
          o[d] += phat * vv;
          oa[d] += std::fabs(phat * vv);
          of[d] += amb * std::fabs(vv);
        }
      }
    }
    for (int64_t d = 0; d < D; ++d) {
      o[d] /= l;
      oa[d] /= l;
      of[d] /= l;
    }
    std::free(z);
  }
}

// FP8 KV-cache decode attention ["NVIDIA NeMo RL erreicht 48% ...",
// "Leistungsgewinne in der Praxis": FP8 KV cache and attention in
// generation].  One new query token per sequence attends to its cached keys.
// The cache is the row-wise 1x128 quantization of the token matrix
// [B*Lmax][Hkv*128]: one E4M3 code row and one fp32 scale per (token, KV
// head), for K and for V alike; sequence b holds tokens b*Lmax .. b*Lmax +
// len[b] - 1.  Scales are laid out [Hkv][B*Lmax].  The query is bf16
// [B][Hq*128]; query head h reads KV head h / (Hq / Hkv).
//   z_j = (q . k^_j) / sqrt(128),  k^_j = decode(k_j) * s_k,j
//   O = sum_j e^(z_j - max z) v^_j / sum_j e^(z_j - max z)
// in fp64, for every (b, h): out[(b*Hq + h)*128 + d].  A sequence with
// len = 0 gives zeros.  oabs = sum_j p_j |v^_j| / l; oerr = 4 dzmax * oabs,
// dzmax bounding the logit error of an fp32 kernel (the fp32 sum of the 128
// exact products q_d * code, at most 2^-16 of their absolute sum, and the
// two fp32 scalings, 2^-21 of |z|): each p and the sum l then carry at most
// 2 dzmax relative error.
void orc_attention_decode(int32_t B, int32_t Hq, int32_t Hkv, int64_t Lmax, const int32_t* len,
                          const uint16_t* q, const uint8_t* k, const float* sk, const uint8_t* v,
                          const float* sv, double* out, double* oabs, double* oerr) {
  const int64_t D = 128;
  const double* dec = decode_table(FMT_E4M3);
  const double inv_sqrt_d = 1.0 / std::sqrt(static_cast<double>(D));
  const int32_t group = Hq / Hkv;
  const int64_t ld = static_cast<int64_t>(Hkv) * D;    // bytes per cache token row
  const int64_t T = static_cast<int64_t>(B) * Lmax;    // tokens in the cache
#pragma omp parallel for schedule(dynamic)
  for (int64_t r = 0; r < static_cast<int64_t>(B) * Hq; ++r) {
    const int64_t b = r / Hq;
    const int32_t h = static_cast<int32_t>(r % Hq), g = h / group;
    double* o = out + r * D;
    double* oa = oabs + r * D;
    double* oe = oerr + r * D;
    for (int64_t d = 0; d < D; ++d) o[d] = oa[d] = oe[d] = 0.0;
    const int64_t L = len[b];
    if (L <= 0) continue;
    double qd[128];
    for (int64_t d = 0; d < D; ++d) qd[d] = bf16_bits_to_float(q[b * Hq * D + h * D + d]);
    double* z = static_cast<double*>(std::malloc(sizeof(double) * L));
    double zmax = -INFINITY, dzmax = 0.0;
    for (int64_t j = 0; j < L; ++j) {
      const int64_t row = b * Lmax + j;
      double acc = 0.0, aabs = 0.0;
      for (int64_t d = 0; d < D; ++d) {
        const double prod = qd[d] * dec[k[row * ld + g * D + d]];
        acc += prod;
        aabs += std::fabs(prod);
      }
      const double c = static_cast<double>(sk[static_cast<int64_t>(g) * T + row]) * inv_sqrt_d;
      z[j] = acc * c;
      const double dz = std::fabs(c) * aabs * std::ldexp(1.0, -16) + std::fabs(z[j]) * std::ldexp(1.0, -21);
      if (z[j] > zmax) zmax = z[j];
      if (dz > dzmax) dzmax = dz;
    }
    double l = 0.0;
    for (int64_t j = 0; j < L; ++j) {
      z[j] = std::exp(z[j] - zmax);   // z now holds p
      l += z[j];
    }
    for (int64_t j = 0; j < L; ++j) {
      const int64_t row = b * Lmax + j;
      const double svj = sv[static_cast<int64_t>(g) * T + row];
      for (int64_t d = 0; d < D; ++d) {
        const double vv = dec[v[row * ld + g * D + d]] * svj;
        o[d] += z[j] * vv;
        oa[d] += z[j] * std::fabs(vv);
      }
    }
    for (int64_t d = 0; d < D; ++d) {
      o[d] /= l;
      oa[d] /= l;
      oe[d] = 4.0 * dzmax * oa[d];
    }
    std::free(z);
  }
}

}  // extern "C"

/*
 * fp8bw — blockwise-scaled FP8 linear layer for B200 (sm_100a).
 *
 * The method (page "NVIDIA NeMo RL erreicht 48% Geschwindigkeitssteigerung
 * mit End-to-End FP8-Präzisionstraining", section "Der technische
 * Durchbruch"): linear layers run FP8 math on E4M3 operands that carry one
 * scale per 128x128 block of a weight and one per 1x128 block of an
 * activation; section "Leistungsgewinne in der Praxis": the weight scales are
 * recalibrated after every training step; section "Warum dies für die
 * KI-Ökonomie wichtig ist": optionally the scales are powers of two.  E4M3
 * itself (page "FP8 Trainingsinfrastructuur", section "Het landschap van
 * numerieke precisie"): 4 exponent bits, 3 mantissa bits, values up to +-448.
 *
 * Conventions for every call below
 *  - All tensor arguments are DEVICE pointers to caller-owned memory; the
 *    library allocates no device memory and keeps no pointer after the call.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).  The returned status covers host-side validation and
 *    launch errors; errors seen inside a kernel (a bounded wait that ran out,
 *    a failed device-side check) are latched in a device error word and read
 *    with fp8bw_last_device_error().
 *  - Shapes: M, N, K are multiples of 128 (else FP8BW_ERR_ALIGNMENT), and
 *    every pointer is 16-byte aligned with leading dimensions that keep rows
 *    16-byte aligned (32-byte where a call says so: the activation
 *    quantizers' code outputs, the per-tensor quantizer's input and codes).
 *    Invalid arguments never reach the GPU.
 *  - bf16 tensors are IEEE bfloat16 bit patterns; E4M3 codes are bytes
 *    (sign | 4-bit exponent field, bias 7 | 3-bit mantissa; 0x7F/0xFF NaN).
 *  - Scale rule (identical in every quantizer): amax = max |x| over the block;
 *      FP8BW_SCALE_FP32: s = fp32(amax / 448)
 *      FP8BW_SCALE_POW2: s = 2^e, e the smallest integer with amax <= 448*2^e,
 *                        clamped to [-127, 127]
 *      an all-zero block has s = 1;
 *    codes q = E4M3(fp32(x / s)) with IEEE fp32 division, round to nearest
 *    even, magnitudes above 448 saturating to 448, the sign of zero kept.
 *    Dequantized value = decode(q) * s.
 */
#ifndef FP8BW_H_
#define FP8BW_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define FP8BW_API __attribute__((visibility("default")))
#else
#define FP8BW_API
#endif

typedef struct CUstream_st* fp8bw_stream_t; /* same type as cudaStream_t */

typedef enum {
  FP8BW_OK = 0,
  FP8BW_ERR_INVALID_ARG = 1,     /* null pointer, bad enum, negative size   */
  FP8BW_ERR_ALIGNMENT = 2,       /* size not a multiple of 128, misaligned  */
  FP8BW_ERR_UNSUPPORTED_ARCH = 3,/* device is not compute capability 10.0   */
  FP8BW_ERR_CUDA = 4,            /* a CUDA runtime/driver call failed       */
  FP8BW_ERR_TIMEOUT = 5,         /* a device-side bounded wait ran out      */
  FP8BW_ERR_DEVICE_CHECK = 6,    /* a device-side argument check failed     */
  FP8BW_ERR_TOO_LARGE = 7        /* a size exceeds a documented maximum     */
} fp8bw_status;

typedef enum { FP8BW_SCALE_FP32 = 0, FP8BW_SCALE_POW2 = 1 } fp8bw_scale_mode;

typedef enum { FP8BW_FPROP = 0, FP8BW_DGRAD = 1, FP8BW_WGRAD = 2 } fp8bw_gemm_kind;

/* Element format of the FP8 codes.  E4M3 is the method's; E5M2 (5 exponent
 * bits, 2 mantissa bits, bias 15, largest finite value 57344; page "FP8
 * Trainingsinfrastructuur", section "Het landschap van numerieke precisie":
 * the gradient format of the per-tensor recipe) is offered for activation
 * gradients as a comparison point.  Block scales then use 57344 in place of
 * 448 (FP32: s = fp32(amax / 57344); POW2: the smallest 2^e with
 * amax <= 57344 * 2^e). */
typedef enum { FP8BW_FMT_E4M3 = 0, FP8BW_FMT_E5M2 = 1 } fp8bw_format;

/* Checks that `device` is an sm_100 part and caches its SM count.  Called
 * implicitly by every entry point for the current device; calling it
 * explicitly first keeps that one-time query out of timed regions. */
FP8BW_API fp8bw_status fp8bw_init(int device);

/* Static, human-readable name of a status. */
FP8BW_API const char* fp8bw_status_string(fp8bw_status s);

/* Synchronizes `stream`, then returns (and clears) the device error words of
 * the current device (one each for the GEMMs, the quantizers and attention):
 * FP8BW_ERR_TIMEOUT if a kernel's bounded wait ran out, FP8BW_ERR_DEVICE_CHECK
 * if a kernel rejected its device-side arguments (grouped offsets, or
 * FP8BW_SCALE_POW2 scales that are not powers of two), else FP8BW_OK.
 * FP8BW_ERR_CUDA if the sync failed. */
FP8BW_API fp8bw_status fp8bw_last_device_error(fp8bw_stream_t stream);

/* Testing hook for the failure path (not part of the method): the next FP8
 * GEMM launch of the process (any fp8bw_gemm* / fp8bw_grouped_* call, from
 * any host thread) has its first CTA's operand producer skip K-chunk number
 * `chunk` (counted over that CTA's tiles), so the kernel's bounded waits run
 * out: it abandons its loops within a few seconds, writes an incomplete
 * result and latches FP8BW_ERR_TIMEOUT for fp8bw_last_device_error(); the
 * context stays usable.  The pending stall is one process-wide value with no
 * synchronization: set it only while no other host thread launches GEMMs.
 * chunk = -1 cancels a pending stall.  FP8BW_ERR_INVALID_ARG if chunk < -1. */
FP8BW_API fp8bw_status fp8bw_testing_stall_next_gemm(int32_t chunk);

/* Activation quantization with 1x128 blocks ("Der technische Durchbruch":
 * 1x128 granularity for activations), plus the column-wise copy the weight
 * gradient needs.
 *   x      [M][ldx] bf16, row-major; the first K columns are quantized.
 *   q_row  [M][K]   E4M3 codes; block (m, kb) = x[m][128kb .. 128kb+127]
 *   s_row  [K/128][M] fp32 scales, chunk-major (s_row[kb*M + m])
 *   q_col  [K][M]   E4M3 codes of the column-wise copy: block (mb, k) =
 *                   x[128mb .. 128mb+127][k], quantized from x itself and
 *                   stored transposed (q_col[k*M + m]) so that the weight
 *                   gradient reads it K-major in tokens
 *   s_col  [M/128][K] fp32 scales of the column-wise copy
 *   q_col and s_col are both NULL for a row-wise-only call.
 * For mixture-of-experts tokens grouped by expert, pad each expert's segment
 * to a multiple of 128 rows (zero rows): column blocks then never straddle
 * two experts and zero rows change no block's amax.
 * Requires M, K multiples of 128, ldx >= K, ldx a multiple of 8, and q_row,
 * q_col 32-byte aligned (the codes leave in 32-byte stores). */
FP8BW_API fp8bw_status fp8bw_quant_act_1x128(const void* x, int64_t M, int64_t K, int64_t ldx,
                                   fp8bw_scale_mode mode, uint8_t* q_row, float* s_row,
                                   uint8_t* q_col, float* s_col, fp8bw_stream_t stream);

/* Weight quantization with 128x128 blocks ("Der technische Durchbruch":
 * 128x128 granularity for weights).
 *   w   [N][ldw] bf16 row-major (nn.Linear layout: N = out, K = in features)
 *   q   [N][K]   E4M3 codes
 *   s   [N/128][K/128] fp32 scales, row-major
 *   qT  [K][N]   the exact byte transpose of q (the data-gradient operand),
 *                or NULL.  Its scale grid is s read transposed.
 * Requires N, K multiples of 128, ldw >= K, ldw a multiple of 8. */
FP8BW_API fp8bw_status fp8bw_quant_weight_128x128(const void* w, int64_t N, int64_t K, int64_t ldw,
                                        fp8bw_scale_mode mode, uint8_t* q, float* s,
                                        uint8_t* qT, fp8bw_stream_t stream);

/* One weight of a batched requantization. */
typedef struct {
  const void* w;   /* [N][ldw] bf16 */
  int64_t N, K, ldw;
  uint8_t* q;      /* [N][K]            */
  float* s;        /* [N/128][K/128]    */
  uint8_t* qT;     /* [K][N] or NULL    */
} fp8bw_weight_desc;

/* Per-step scale recalibration ("Leistungsgewinne in der Praxis": the scales
 * are recalibrated after every training step): requantizes every weight in
 * `descs` (a HOST array of n descriptors, read during the call only) exactly
 * as fp8bw_quant_weight_128x128 would, in one launch per up to
 * FP8BW_REQUANT_MAX_PER_LAUNCH weights.  Output is bit-identical to n
 * separate fp8bw_quant_weight_128x128 calls. */
#define FP8BW_REQUANT_MAX_PER_LAUNCH 256
FP8BW_API fp8bw_status fp8bw_requant_weights(const fp8bw_weight_desc* descs, int32_t n,
                                   fp8bw_scale_mode mode, fp8bw_stream_t stream);

/* Blockwise-scaled FP8 GEMM ("Der technische Durchbruch": linear layers run
 * FP8 math), FP32 accumulation, bf16 output:
 *   D[m][n] = bf16( sum_kb sA(m,kb) * sB(n,kb) * sum_{k in chunk kb} A[m][k] B[n][k] )
 * with codes decoded from E4M3 and chunk kb = columns 128kb .. 128kb+127.
 * M, N, K are the GEMM's own sizes:
 *   FPROP  Y  = X W^T : A = q_row(X) [M][K], sA = s_row(X); B = q(W) [N][K],
 *                       sB = s(W) [N/128][K/128]
 *   DGRAD  dX = dY W  : A = q_row(dY) [M][K=out], sA = s_row(dY);
 *                       B = qT(W) [N=in][K=out], sB = s(W) of the layer,
 *                       i.e. [K/128][N/128] in this call's sizes
 *   WGRAD  dW = dY^T X: A = q_col(dY) [M=out][K=tokens], sA = s_col(dY);
 *                       B = q_col(X) [N=in][K=tokens], sB = s_col(X) [K/128][N]
 *   A  [M][K] codes, K-major; sA [K/128][M]
 *   B  [N][K] codes, K-major; sB as above
 *   D  [M][ldd] bf16; ldd >= N, a multiple of 8
 * `mode` states how the scales were made; FP8BW_SCALE_POW2 promises exact
 * powers of two in [2^-127, 2^127] (the kernel then folds them into the
 * tensor-core MMA as UE8M0 scale factors).  A POW2 scale that is not a power
 * of two latches FP8BW_ERR_DEVICE_CHECK and leaves D undefined (written with
 * the scale's exponent only).
 * The result is within |D - ref| <= 1e-2 * sum_k |a_k b_k| + 1 bf16 ulp(ref)
 * of the fp64 product of the dequantized operands.  K = 0 writes exact zeros;
 * M = 0 or N = 0 does nothing. */
FP8BW_API fp8bw_status fp8bw_gemm(fp8bw_gemm_kind kind, int64_t M, int64_t N, int64_t K,
                        const uint8_t* A, const float* sA, const uint8_t* B, const float* sB,
                        void* D, int64_t ldd, fp8bw_scale_mode mode, fp8bw_stream_t stream);

/* fp8bw_quant_act_1x128 with the element format chosen: FP8BW_FMT_E4M3
 * gives exactly fp8bw_quant_act_1x128's result; FP8BW_FMT_E5M2 encodes E5M2
 * codes (round to nearest even, saturating to 57344) with the E5M2 scale
 * rule above.  Arguments, layouts and errors as in fp8bw_quant_act_1x128. */
FP8BW_API fp8bw_status fp8bw_quant_act_1x128_fmt(const void* x, int64_t M, int64_t K, int64_t ldx,
                                       fp8bw_scale_mode mode, fp8bw_format fmt,
                                       uint8_t* q_row, float* s_row, uint8_t* q_col,
                                       float* s_col, fp8bw_stream_t stream);

/* fp8bw_gemm with the element formats of A and B given (codes decoded as
 * E4M3 or E5M2; e.g. dgrad/wgrad with E5M2 activation gradients against
 * E4M3 weights or activations).  Everything else as in fp8bw_gemm. */
FP8BW_API fp8bw_status fp8bw_gemm_fmt(fp8bw_gemm_kind kind, int64_t M, int64_t N, int64_t K,
                            const uint8_t* A, const float* sA, fp8bw_format a_fmt,
                            const uint8_t* B, const float* sB, fp8bw_format b_fmt,
                            void* D, int64_t ldd, fp8bw_scale_mode mode,
                            fp8bw_stream_t stream);

/* The same GEMM with an fp32 output, for the weight gradient's fp32 main
 * gradient of mixed-precision training (the optimizer step after which the
 * weights are requantized, "Leistungsgewinne in der Praxis", keeps fp32
 * master state):
 *   accumulate = 0:  D[m][n]  = sum_kb sA(m,kb) sB(n,kb) sum_k A[m][k] B[n][k]
 *   accumulate = 1:  D[m][n] += the same sum (one fp32 rounding of the add,
 *                    done in L2; no bf16 rounding anywhere)
 * Operands, kinds and scale layouts as in fp8bw_gemm.  D [M][ldd] fp32,
 * 16-byte aligned, ldd >= N and a multiple of 4 (16-byte rows).  The
 * result is within |D - ref| <= 1e-2 * sum_k |a_k b_k| + 2^-22 |ref| of the
 * fp64 reference (plus the prior D when accumulating).  Calls on one stream
 * accumulate in order; no two calls may write the same D concurrently. */
FP8BW_API fp8bw_status fp8bw_gemm_f32(fp8bw_gemm_kind kind, int64_t M, int64_t N, int64_t K,
                            const uint8_t* A, const float* sA, const uint8_t* B,
                            const float* sB, float* D, int64_t ldd, int32_t accumulate,
                            fp8bw_scale_mode mode, fp8bw_stream_t stream);

/* The GEMM with its output quantized in the epilogue, for an output that is
 * the next FP8 GEMM's operand ("Der technische Durchbruch": activations and
 * activation gradients enter the FP8 linear layers as 1x128 blocks;
 * "Leistungsgewinne in der Praxis": quantization-kernel overhead is part of
 * the gap between 2x and the measured gain, and fusing the quantizer into
 * the producer removes the bf16 round trip through HBM).
 * Computes D = bf16(sum_kb sA sB sum_k A B) exactly as fp8bw_gemm with
 * FP8BW_SCALE_FP32 (the operand scales may be any fp32 values, powers of two
 * included), then writes what fp8bw_quant_act_1x128(D, out_mode) writes:
 *   q_row [M][N] E4M3 codes, s_row [N/128][M]   (1x128 row blocks)
 *   q_col [N][M] codes, s_col [M/128][N]        (column-wise copy; both
 *                                                NULL for row-wise only)
 *   D     [M][ldd] bf16, or NULL to skip it (ldd a multiple of 8 if given).
 * Bit for bit, the codes and scales equal fp8bw_quant_act_1x128 applied to
 * this call's D.  Operands, kinds and scale layouts as in fp8bw_gemm.
 * Requires M, N, K multiples of 128 and K > 0 (else FP8BW_ERR_ALIGNMENT /
 * FP8BW_ERR_INVALID_ARG), q_row and q_col 32-byte aligned. */
FP8BW_API fp8bw_status fp8bw_gemm_quant(fp8bw_gemm_kind kind, int64_t M, int64_t N, int64_t K,
                                        const uint8_t* A, const float* sA, const uint8_t* B,
                                        const float* sB, fp8bw_scale_mode out_mode, void* D, int64_t ldd,
                                        uint8_t* q_row, float* s_row, uint8_t* q_col, float* s_col,
                                        fp8bw_stream_t stream);

/* Grouped GEMM for mixture-of-experts layers ("Leistungsgewinne in der
 * Praxis": the recipe also trains the Qwen3-30B MoE model).  Tokens are
 * grouped by expert: expert g owns rows [off[g], off[g+1]) of the permuted
 * token matrix, with every offset a multiple of 128 (segments zero-padded),
 * off[0] = 0 and off[G] <= M_total_pad.  `d_offsets` is a DEVICE array of
 * G+1 int32 values, so routing never synchronizes the host; a kernel that
 * finds them invalid writes nothing and latches FP8BW_ERR_DEVICE_CHECK.
 *   FPROP/DGRAD: A [M_total_pad][K], sA [K/128][M_total_pad];
 *                B [G][N][K] (FPROP: q(W_g); DGRAD: qT(W_g)),
 *                sB [G][...] the per-expert grid as in fp8bw_gemm;
 *                D [M_total_pad][N]; rows at or beyond off[G] are untouched.
 *   WGRAD:       A = q_col(dY) [N][M_total_pad], sA [M_total_pad/128][N];
 *                B = q_col(X)  [K][M_total_pad], sB [M_total_pad/128][K];
 *                D [G][N][K]: expert g contracts only its own tokens; an
 *                expert with no tokens gets exact zeros.
 * Requires G <= FP8BW_MAX_EXPERTS.  FPROP/DGRAD with K = 0 return
 * FP8BW_ERR_INVALID_ARG (the routed rows are known only on the device, so
 * the host cannot zero them); M_total_pad = 0 or N = 0 does nothing, and
 * WGRAD with N = 0 or K = 0 does nothing.  Scales as in fp8bw_gemm. */
#define FP8BW_MAX_EXPERTS 512
FP8BW_API fp8bw_status fp8bw_grouped_gemm(fp8bw_gemm_kind kind, int32_t G, const int32_t* d_offsets,
                                int64_t M_total_pad, int64_t N, int64_t K,
                                const uint8_t* A, const float* sA, const uint8_t* B,
                                const float* sB, void* D, fp8bw_scale_mode mode,
                                fp8bw_stream_t stream);

/* Grouped weight gradient with an fp32 output, for mixture-of-experts
 * layers' fp32 main gradients: operands, offsets and checks as in
 * fp8bw_grouped_gemm with kind FP8BW_WGRAD; D [G][N][K] fp32 (16-byte
 * aligned), accumulate as in fp8bw_gemm_f32 (an expert with no tokens adds
 * zeros, or stores zeros when accumulate = 0). */
FP8BW_API fp8bw_status fp8bw_grouped_wgrad_f32(int32_t G, const int32_t* d_offsets,
                                     int64_t M_total_pad, int64_t N, int64_t K,
                                     const uint8_t* A, const float* sA, const uint8_t* B,
                                     const float* sB, float* D, int32_t accumulate,
                                     fp8bw_scale_mode mode, fp8bw_stream_t stream);

/* BF16 GEMM, the comparison path of "Der technische Durchbruch" (FP8 linear
 * layers have twice the BF16 peak): D[m][n] = bf16( sum_k A[m][k] B[n][k] )
 * with FP32 accumulation.  A [M][K], B [N][K] bf16, K-major (dense rows);
 * D [M][ldd] bf16.  M, N, K multiples of 128. */
FP8BW_API fp8bw_status fp8bw_gemm_bf16(int64_t M, int64_t N, int64_t K, const void* A, const void* B,
                             void* D, int64_t ldd, fp8bw_stream_t stream);

/* Per-tensor delayed scaling, the comparison recipe of "FP8
 * Trainingsinfrastructuur" (sections "Transformer Engine: de softwarebasis":
 * a history of 16 amax values, the "max" rule, margin 0, E4M3 forward and
 * E5M2 backward; "Scaling-strategieën en stabiliteit": one scale per tensor,
 * chosen from earlier iterations so that no reduction over the current
 * tensor precedes its quantization).
 *   x        [M][ldx] bf16, row-major; the first K columns are quantized.
 *   hist     [H] fp32 amax history, newest first, read and updated:
 *            s = scale rule of `fmt` and `mode` applied to max(hist)
 *            (s = 1 while the history holds no positive value); after the
 *            tensor is quantized hist[i] = hist[i-1] for i = H-1 .. 1 and
 *            hist[0] = amax.  Zero-initialise it before the first call.
 *   q        [M][K] codes, q = encode(fp32(x) / s); a tensor that outgrew its
 *            history saturates to the format's largest value.
 *   qT       [K][M] the byte transpose of q (one scale: the column-wise copy
 *            the weight gradient reads), or NULL.
 *   scale    one fp32, the s this call used.
 *   amax     one fp32, max |x| of this call (NaN elements are ignored).
 *   s_grid   NULL, or s_grid_len fp32 values all set to s: a constant scale
 *            grid, so that (q, s_grid) or (qT, s_grid) feed the blockwise
 *            GEMMs (fp8bw_gemm, fp8bw_gemm_fmt) as an operand whose every
 *            block carries s.  A grid of M*K/128 values serves both
 *            activation layouts; a weight needs N*K/16384.
 * All outputs are device memory; hist, scale, amax and s_grid must not
 * overlap each other or the tensors.  The history is read and rewritten in
 * stream order (a 4-byte memset of amax, the quantizing kernel, a one-thread
 * history push), so calls that share a history must be ordered: the same
 * stream, or events between streams.  An empty tensor (M or K zero; x, q,
 * qT may then be NULL) still sets scale, amax = 0, s_grid and the history.
 * Requires M, K multiples of 128, ldx >= K and a multiple of 16, x, q and qT
 * 32-byte aligned, hist, scale, amax, s_grid 4-byte aligned,
 * 1 <= H <= FP8BW_MAX_HISTORY; else FP8BW_ERR_INVALID_ARG or
 * FP8BW_ERR_ALIGNMENT, with nothing launched. */
#define FP8BW_MAX_HISTORY 1024
FP8BW_API fp8bw_status fp8bw_quant_tensor_delayed(const void* x, int64_t M, int64_t K, int64_t ldx,
                                        fp8bw_format fmt, fp8bw_scale_mode mode, float* hist,
                                        int32_t H, uint8_t* q, uint8_t* qT, float* scale,
                                        float* amax, float* s_grid, int64_t s_grid_len,
                                        fp8bw_stream_t stream);

/* FP8 attention forward ("NVIDIA NeMo RL erreicht 48% ...", section
 * "Leistungsgewinne in der Praxis": the recipe extends FP8 to the KV cache
 * and the attention operations).  Head dimension 128.  Every operand is
 * E4M3 with one scale per 128 elements along its contraction, as the
 * activation quantizer makes them:
 *   q   [T][Hq*128] codes, sq [Hq][T]: fp8bw_quant_act_1x128 of Q [T][Hq*128]
 *       (row-wise; one scale per token and head)
 *   k   [T][Hkv*128] codes, sk [Hkv][T]: the same for K (the key cache)
 *   vT  [Hkv*128][T] codes, sv [T/128][Hkv*128]: the column-wise copy
 *       (q_col, s_col) of V [T][Hkv*128] (one scale per 128 tokens of one
 *       channel; the value cache, channel-major)
 *   o   [T][Hq*128] bf16 output, 32-byte aligned.
 * Query head h reads key/value head h / (Hq / Hkv).  Tokens are packed
 * sequences: segment s covers tokens [off[s], off[s+1]) (DEVICE arrays
 * d_seg_off [nseg+1], d_seg_len [nseg]; offsets non-decreasing multiples of
 * 128, off[0] = 0, off[nseg] <= T), of which the first len[s] are real.  A
 * real query token t attends to the real tokens of its segment (causal = 1:
 * only those j <= t).  Per query row: logits z_j = (q^ . k^_j) / sqrt(128)
 * (q^, k^ dequantized), p_j = exp(z_j - max z), l = sum_j p_j; P is
 * quantized to E4M3 per 128-key block with the FP32 scale rule s = amax/448
 * (codes E4M3(p / s)); o = sum_j p^_j v^_j / l in bf16.  Padding rows (past
 * len[s], or past off[nseg]) are written as zeros.  The result is within
 * |o - ref| <= 1e-2 * sum_j |p^_j v^_j| / l + (one E4M3 step of each p_j
 * whose p / s lies within the kernel's fp32 error of a rounding midpoint)
 * + 1 bf16 ulp of the fp64 reference of the same definition.
 * mode = FP8BW_SCALE_POW2 (the recipe's optional power-of-2 scales,
 * "Warum dies für die KI-Ökonomie wichtig ist"): sq, sk and sv must be
 * powers of two, as fp8bw_quant_act_1x128 makes them in that mode; the
 * tensor core then applies every scale itself (block-scaled MMA), and P's
 * block scale is the power-of-2 rule on its amax, p taken against an integer
 * power-of-two reference maximum (any such reference gives the same codes).
 * The result is within the gate above, widened where the block amax sits
 * within the kernel's error of a power-of-two boundary (either scale is
 * correct there).  A scale that is not a power of two latches
 * FP8BW_ERR_DEVICE_CHECK and leaves o undefined.
 * Requires T a multiple of 128, Hq a multiple of Hkv, Hq <=
 * FP8BW_ATTN_MAX_HEADS, 1 <= nseg <= FP8BW_ATTN_MAX_SEGMENTS, 16-byte
 * aligned codes and scales.  Invalid offsets are rejected on the device:
 * nothing is written and fp8bw_last_device_error() reports
 * FP8BW_ERR_DEVICE_CHECK. */
#define FP8BW_ATTN_MAX_SEGMENTS 65536
#define FP8BW_ATTN_MAX_HEADS 1024
FP8BW_API fp8bw_status fp8bw_attention_fwd(int64_t T, int32_t Hq, int32_t Hkv, int32_t nseg,
                                           const int32_t* d_seg_off, const int32_t* d_seg_len,
                                           int32_t causal, fp8bw_scale_mode mode,
                                           const uint8_t* q, const float* sq,
                                           const uint8_t* k, const float* sk, const uint8_t* vT,
                                           const float* sv, void* o, fp8bw_stream_t stream);

/* FP8 KV-cache decode attention ("NVIDIA NeMo RL erreicht 48% ...", section
 * "Leistungsgewinne in der Praxis": FP8 for the KV cache and the attention
 * operations of generation).  One new query token per sequence attends to
 * the keys cached for it.  Head dimension 128.  The cache is the row-wise
 * 1x128 quantization of its token matrix, as fp8bw_quant_act_1x128 (FP32 or
 * power-of-2 scales, row-wise only) makes it:
 *   k  [B*Lmax][Hkv*128] E4M3 codes, sk [Hkv][B*Lmax] fp32 scales (one per
 *      token and KV head); sequence b owns rows b*Lmax .. b*Lmax + Lmax - 1,
 *      of which the first len[b] are its cached tokens
 *   v, sv  the same for V
 *   q  [B][Hq*128] bf16, the new tokens' queries (not quantized)
 *   o  [B][Hq*128] bf16 output.
 * d_len is a DEVICE array [B] with 0 <= len[b] <= Lmax.  Query head h reads
 * KV head h / (Hq / Hkv).  Per (b, h): z_j = (q . k^_j) / sqrt(128) with
 * k^_j = E4M3(k_j) * s_k,j, p_j = exp(z_j - max z), o = sum_j p_j v^_j /
 * sum_j p_j in bf16; len[b] = 0 gives zeros.  The kernel computes in fp32;
 * the result is within |o - ref| <= 2^-10 * sum_j p_j |v^_j| / l + 4 dz *
 * sum_j p_j |v^_j| / l + 1 bf16 ulp of the fp64 reference, dz = max_j
 * (2^-16 |s_k,j| / sqrt(128) * sum_d |q_d E4M3(k_j,d)| + 2^-21 |z_j|) (the
 * fp32 logit error).  A length outside [0, Lmax] latches
 * FP8BW_ERR_DEVICE_CHECK and that sequence's output is not written.
 * Requires Lmax a positive multiple of 128, Hq a multiple of Hkv with Hq / Hkv in
 * {1, 2, 4, 8}, 16-byte aligned k, v, q, sk and sv, 4-byte aligned d_len,
 * 2-byte aligned o.  All buffers are the caller's; nothing is allocated. */
FP8BW_API fp8bw_status fp8bw_attention_decode(int32_t B, int32_t Hq, int32_t Hkv, int64_t Lmax,
                                              const int32_t* d_len, const void* q,
                                              const uint8_t* k, const float* sk,
                                              const uint8_t* v, const float* sv, void* o,
                                              fp8bw_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FP8BW_H_ */

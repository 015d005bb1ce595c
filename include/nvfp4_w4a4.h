/*
 * nvfp4_w4a4.h -- NVFP4 x NVFP4 (W4A4) prefill GEMM for NVIDIA B200 (sm_100a),
 * beside the weight-only entry points of nvfp4.h (same library, status codes
 * and conventions: device pointers owned by the caller, asynchronous on
 * `stream`, host-side validation, nothing allocated, no synchronization).
 *
 * The operation (imp docs/quantization.md: the dense-layer pipeline's prefill
 * "CUTLASS NVFP4 GEMM" with the weight micro-scales rearranged once into the
 * tensor core's scale-factor layout, "Phase 3b"; the Modelopt row's
 * "NVFP4 x NVFP4 prefill").  The pages give no rule for the activations; here
 * X takes the weights' own format and rule (nvfp4.h, nvfp4_quantize):
 *   g_x = x_amax / 2688 (fp32), x_amax = max |X| (dynamic) or a given,
 *         calibrated amax (static);
 *   (qx, sx) = RTN NVFP4 of X with the tensor scale g_x;
 *   Y[m, n] = bf16_rn( g * g_x * sum_k (sx * e2m1(qx))[m, k] * (s * e2m1(q))[n, k] )
 * on the block-scaled FP4 tensor cores with fp32 accumulation.
 *
 * Layouts:
 *   X   BF16 [M, K], leading dimension ldx (elements)
 *   qx  u8   [M, K/2] row-major codes (element 2j in the low nibble of byte j)
 *   q   u8   [N, K/2] weight codes as in nvfp4.h
 *   scale-factor ("MMA") layout of a [R, K/16] E4M3 scale matrix: rows padded
 *       with zero scales to a multiple of P; one 512-byte atom per 128 rows and
 *       64 k, atom (r / 128, k / 64) at ((r / 128) * (K / 64) + k / 64) * 512,
 *       the scale of row r and elements 16j .. 16j+15 of the 64 at byte
 *       (r % 32) * 16 + ((r % 128) / 32) * 4 + j of its atom.
 *       Weights: P = 128 (nvfp4_w4a4_weight_scales_bytes); activations: P = 256
 *       (nvfp4_w4a4_x_scales_bytes).
 *   Y   BF16 [M, N], leading dimension ldy
 *
 * K must be a positive multiple of 256 and at most 2^24; N >= 1; 1 <= M <= 2^24;
 * ceil(N / 128) * ceil(M / 256) < 2^31 (the GEMM's tile count).
 * X, q, qx, scale buffers and the workspace are 16-byte aligned, ldx a
 * multiple of 8; g and x_amax 4-byte aligned; Y 2-byte aligned.
 */
#ifndef NVFP4_W4A4_H_
#define NVFP4_W4A4_H_

#include "nvfp4.h"

#ifdef __cplusplus
extern "C" {
#endif

/* x_amax is an input (a calibrated amax) instead of being computed from X. */
#define NVFP4_W4A4_GIVEN_AMAX 2u

/* Floats of the x_amax buffer of a dynamic-amax nvfp4_w4a4_quantize_x:
 * element 0 receives max |X|, the rest holds per-CTA partial maxima. */
#define NVFP4_W4A4_AMAX_FLOATS 260

/* Bytes of the weight scales [N, K/16] in the MMA layout (rows padded to 128). */
NVFP4_API size_t nvfp4_w4a4_weight_scales_bytes(int64_t N, int64_t K);

/* Bytes of the activation scales [M, K/16] in the MMA layout (rows padded to 256). */
NVFP4_API size_t nvfp4_w4a4_x_scales_bytes(int64_t M, int64_t K);

/*
 * Rearrange the row-major weight scales s [N, K/16] (nvfp4_quantize output)
 * into s_mma (nvfp4_w4a4_weight_scales_bytes(N, K) bytes), once per weight
 * tensor.  s_mma must not overlap s.  N == 0 is a no-op.
 */
NVFP4_API nvfp4_status nvfp4_w4a4_prepare_weights(const uint8_t* s, int64_t N, int64_t K, uint8_t* s_mma,
                                                  nvfp4_stream_t stream);

/*
 * Quantize X [M, K] for the W4A4 GEMM: codes qx [M, K/2] and scales sx in the
 * MMA layout (nvfp4_w4a4_x_scales_bytes(M, K) bytes).  Without
 * NVFP4_W4A4_GIVEN_AMAX in flags, x_amax points to NVFP4_W4A4_AMAX_FLOATS
 * floats and x_amax[0] receives max |X| (two kernels: per-CTA maxima, then the
 * quantizer, which reduces them); with it, only x_amax[0] is read.  qx, sx and
 * the x_amax floats must not overlap X or each other.  M == 0 is a no-op.
 */
NVFP4_API nvfp4_status nvfp4_w4a4_quantize_x(const uint16_t* X, int64_t ldx, int64_t M, int64_t K, uint8_t* qx,
                                             uint8_t* sx, float* x_amax, uint32_t flags, nvfp4_stream_t stream);

/*
 * Y = bf16(g * (x_amax / 2688) * Xq . Wq^T) from quantized activations (qx,
 * sx, x_amax as nvfp4_w4a4_quantize_x leaves them) and weights (q, s_mma from
 * nvfp4_w4a4_prepare_weights, g).  flags: NVFP4_FLAG_STATIC_WEIGHTS and
 * NVFP4_FLAG_W4A4_PAIR (nvfp4.h).
 * Y must not overlap any input.  M == 0 or N == 0 is a no-op.
 */
NVFP4_API nvfp4_status nvfp4_w4a4_gemm(const uint8_t* qx, const uint8_t* sx, const float* x_amax, const uint8_t* q,
                                       const uint8_t* s_mma, const float* g, uint16_t* Y, int64_t ldy, int64_t M,
                                       int64_t N, int64_t K, uint32_t flags, nvfp4_stream_t stream);

/* Workspace of nvfp4_w4a4_linear: qx, sx and the dynamic x_amax floats. */
NVFP4_API size_t nvfp4_w4a4_workspace_size(int64_t M, int64_t K);

/*
 * nvfp4_w4a4_quantize_x into the workspace, then nvfp4_w4a4_gemm.  x_amax:
 * NULL for the dynamic max |X|, else a device pointer to a calibrated amax.
 * flags: NVFP4_FLAG_STATIC_WEIGHTS, NVFP4_FLAG_W4A4_PAIR.  The workspace (at least
 * nvfp4_w4a4_workspace_size(M, K) bytes) must not overlap the other buffers;
 * calls that share it must be ordered on one stream.
 */
NVFP4_API nvfp4_status nvfp4_w4a4_linear(const uint16_t* X, int64_t ldx, const float* x_amax, const uint8_t* q,
                                         const uint8_t* s_mma, const float* g, uint16_t* Y, int64_t ldy, int64_t M,
                                         int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                                         uint32_t flags, nvfp4_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif  // NVFP4_W4A4_H_

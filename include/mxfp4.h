/*
 * mxfp4.h -- MXFP4 weight-only (W4A16) quantizer and decode GEMV for NVIDIA
 * B200 (sm_100a), beside the NVFP4 entry points of nvfp4.h (same library,
 * same status codes, same conventions: device pointers owned by the caller,
 * asynchronous on `stream`, host-side validation, nothing allocated).
 *
 * The format (imp docs/quantization.md, the MXFP4 paragraph after the NVFP4
 * pipelines, and the MXFP4 row of the format table): the same E2M1 nibble
 * layout as NVFP4, one UE8M0 micro-scale per 32 elements, no separate tensor
 * scale; quantization is round-to-nearest.
 *
 * Layouts (row-major):
 *   W  BF16 [N, K] with leading dimension ldw (elements)
 *   q  u8   [N, K/2]  as in nvfp4.h: element 2j in the low nibble of byte j
 *   s  u8   [N, K/32] UE8M0 scale of elements 32j .. 32j+31 of row n: byte b
 *                     means 2^(b - 127) (255 is NaN)
 *   y[n] = bf16_rn( sum_j 2^(s[n, j] - 127) * sum_i e2m1(q[n, 32j+i]) * x[32j+i] )
 *   accumulated in fp32.
 *
 * Quantizer contract (bit-exact; the pages give no scale formula, this is the
 * shared-exponent rule of the microscaling convention): for each 32-block,
 *   amax_b = max |w|;  e = floor(log2(amax_b)) - 2   (2 = largest E2M1 exponent)
 *   s = clamp(e + 127, 0, 254), and s = 0 when amax_b == 0
 *   code = E2M1_rne_satfinite(w / 2^(s - 127))   (ties to the even code, sign
 *          kept, |.| > 6 saturates to 6; w == +-0 gives 0x0 / 0x8)
 *
 * K must be a positive multiple of 32.  Pointers: W, x, q 16-byte aligned
 * (ldw a multiple of 8); s 16-byte aligned; y 2-byte aligned.
 */
#ifndef MXFP4_H_
#define MXFP4_H_

#include "nvfp4.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Round-to-nearest BF16 -> MXFP4 of W [N, K] (no tensor amax pass: each
 * block's scale depends on the block alone).  q, s must not overlap W or each
 * other.  N == 0 is a no-op.
 */
NVFP4_API nvfp4_status mxfp4_quantize(const uint16_t* w, int64_t N, int64_t K, int64_t ldw, uint8_t* q,
                                      uint8_t* s, nvfp4_stream_t stream);

/*
 * MXFP4 batch-1 decode GEMV, y = x . W^T as above.  x: BF16 [K]; y: BF16 [N],
 * not overlapping x, q or s.  K <= 49152.  N == 0 is a no-op.
 */
NVFP4_API nvfp4_status mxfp4_gemv(const uint16_t* x, const uint8_t* q, const uint8_t* s, uint16_t* y,
                                  int64_t N, int64_t K, nvfp4_stream_t stream);

/* mxfp4_gemv with flags (NVFP4_FLAG_*, as for nvfp4_gemv_ex). */
NVFP4_API nvfp4_status mxfp4_gemv_ex(const uint16_t* x, const uint8_t* q, const uint8_t* s, uint16_t* y,
                                     int64_t N, int64_t K, uint32_t flags, nvfp4_stream_t stream);

/*
 * MXFP4 weights on the NVFP4 kernels (nvfp4_gemm, nvfp4_gemv, ...): the codes q
 * are shared, and the scales are restated once (weights are static) as NVFP4
 * scales s_nv [N, K/16] with a power-of-two tensor scale *g_out:
 *   G = (largest k = s_mx - 127 over blocks with a non-zero code) - 8,
 *   s_nv of both 16-element halves of a 32-block = E4M3(2^(k - G)), g = 2^G,
 * which reproduces the MXFP4 weights exactly when every non-zero block lies
 * within 17 binades of the largest (E4M3 holds 2^-9 .. 2^8).  Blocks whose
 * codes are all zero get scale 0.  Blocks with the NaN scale byte 255 (which
 * take no part in G) and non-zero blocks outside the window get scale 0 and
 * are counted: nvfp4_check_device_errors then returns NVFP4_ERR_INVALID_ARG.  q, s_mx, s_nv 16-byte aligned and
 * contiguous; g_out 4-byte aligned (it also holds the reduction while the call
 * runs).  N == 0 is a no-op.
 */
NVFP4_API nvfp4_status mxfp4_to_nvfp4_scales(const uint8_t* q, const uint8_t* s_mx, int64_t N, int64_t K,
                                             uint8_t* s_nv, float* g_out, nvfp4_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif  // MXFP4_H_

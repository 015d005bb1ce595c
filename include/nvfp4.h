/*
 * nvfp4.h -- C ABI of the NVFP4 weight-only (W4A16) linear-layer library for
 * NVIDIA B200 (sm_100a).
 *
 * The operation (web pages, by title and section):
 *   - "Raphael Friedmann" home page, NVFP4 bit-level graphic: a weight is an
 *     E2M1 nibble (1 sign, 2 exponent, 1 mantissa bit), every 16 values share
 *     an FP8 scale and the tensor has one FP32 scale.
 *   - imp docs/quantization.md, format table and "imp-quantize" section: the
 *     packed layout (.weight U8 nibbles, .weight_scale F8_E4M3 per 16,
 *     .weight_scale_2 F32) and plain round-to-nearest from the block absmax;
 *     "Dense layers" pipeline: decode GEMV and prefill GEMM read it directly.
 *   - model card "Qwen3.8-27B-NVFP4 (compressed-tensors)", "What is quantized"
 *     and the paragraph after it: weight-only (activations stay BF16), group
 *     size 16, merged q/k/v and gate/up layers share one tensor scale.
 *
 * Layouts (all row-major, no padding inside a row):
 *   W  BF16 [N, K]  with leading dimension ldw (elements)       (quantizer input)
 *   q  u8   [N, K/2] byte j of row n holds element 2j in its low nibble and
 *                    element 2j+1 in its high nibble (E2M1 codes)
 *   s  u8   [N, K/16] E4M3 scale of elements 16j .. 16j+15 of row n
 *   g  fp32 scalar   dequantization multiplier, g = amax / (6 * 448)
 *   X  BF16 [M, K] with leading dimension ldx;  Y BF16 [M, N] with ldy
 *   Y[m, n] = bf16_rn( g * sum_j e4m3(s[n, j]) * sum_i e2m1(q[n, 16j+i]) * X[m, 16j+i] )
 *   accumulated in fp32.
 *
 * Conventions of every entry point:
 *   - Pointers to tensors are DEVICE pointers owned by the caller; the library
 *     keeps no pointer after the call returns and allocates no device memory.
 *     BF16 tensors are passed as uint16_t bit patterns.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and runs asynchronously; the call does not synchronize.
 *   - Arguments are validated on the host before anything is launched.  On
 *     failure nothing is enqueued, a status other than NVFP4_OK is returned and
 *     nvfp4_last_error() describes it.  No call aborts or throws.
 *   - Input tensor pointers (W, X, x, q, s) and the quantizer outputs q, s
 *     must be 16-byte aligned, with leading dimensions ldw, ldx multiples of 8
 *     elements; the BF16 outputs y, Y need 2-byte alignment and any ldy >= N;
 *     scalar pointers (g, amax) need 4-byte alignment.  K is a positive
 *     multiple of 16 (one scale per 16).
 *   - Calls on the same stream are ordered; calls on different streams that
 *     write the same buffers race.
 */
#ifndef NVFP4_H_
#define NVFP4_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t, kept opaque so that this header needs no CUDA headers. */
typedef void* nvfp4_stream_t;

typedef enum nvfp4_status {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1, /* null pointer, negative size, aliasing outputs */
  NVFP4_ERR_SHAPE = 2,       /* K not a positive multiple of 16, M/N < 0, size too large */
  NVFP4_ERR_ALIGNMENT = 3,   /* pointer under-aligned, leading dimension not a multiple of 8 */
  NVFP4_ERR_UNSUPPORTED = 4, /* current device is not compute capability 10.0 (B200) */
  NVFP4_ERR_CUDA = 5,        /* a CUDA runtime call or kernel launch failed */
  NVFP4_ERR_WORKSPACE = 6,   /* workspace missing or smaller than nvfp4_gemm_workspace_size() */
  NVFP4_ERR_TIMEOUT = 7      /* a kernel's bounded pipeline wait gave up (see nvfp4_check_device_errors) */
} nvfp4_status;

/*
 * Flags of the *_ex entry points.
 * NVFP4_FLAG_STATIC_WEIGHTS: q, s and g are not written by any work that is
 *   still running on the stream when the call is made (model weights loaded
 *   once).  The kernel may then start streaming them while the preceding
 *   kernel on the stream is still finishing (programmatic dependent launch);
 *   x / X are still read, and y / Y written, only after the preceding work has
 *   completed.  Without the flag, every global access waits for it.
 */
#define NVFP4_FLAG_STATIC_WEIGHTS 1u

/*
 * Decode GEMV only (nvfp4_gemv_ex, mxfp4_gemv_ex): NVFP4_FLAG_KSPLIT(c) with c
 * in {1, 2, 4, 8} fixes how many CTAs share each block of output rows by
 * splitting K ("K-parallel" decode GEMV of imp docs/quantization.md, "Dense
 * layers" pipeline).  The split points fall on 512-element boundaries, so no
 * 16- or 32-element scale block is cut; the c CTAs form a thread-block cluster
 * and add their fp32 partial sums in a fixed order through distributed shared
 * memory (results are deterministic, no workspace).  Without the flag the
 * library picks c per shape (skinny layers with large K get c > 1).  A c that
 * does not fit the shape (fewer than c 512-element columns, more than 11520
 * elements of x per CTA, K not a multiple of 256 / 512 for MXFP4) gives
 * NVFP4_ERR_SHAPE; c = 1 forbids splitting.
 */
#define NVFP4_FLAG_KSPLIT(c) (((uint32_t)(c) & 15u) << 8)
#define NVFP4_FLAG_KSPLIT_MASK (15u << 8)

/*
 * W4A4 GEMM only (nvfp4_w4a4_gemm, nvfp4_w4a4_linear): NVFP4_FLAG_W4A4_PAIR
 * runs the GEMM on tiles of 256 weight rows x 256 tokens, each on a pair of
 * SMs (a 2-CTA cluster whose even CTA issues tcgen05.mma.cta_group::2 for
 * both): a token tile then crosses from L2 into the SMs once per 256 weight
 * rows instead of once per 128.  The result is the same as without the flag
 * (same products, same fp32 accumulation order per output).  On one B200 the
 * [17408, 5120] layer at M = 512 ran at 28.5 us per call with the flag and
 * 27.8 us without (each stage then waits for the later of two CTAs' loads),
 * so it is off by default.
 */
#define NVFP4_FLAG_W4A4_PAIR (1u << 12)

/* Version of this ABI (major * 10000 + minor * 100 + patch). */
NVFP4_API int nvfp4_version(void);

/* Message of the most recent failed call made by this host thread ("" if none).
 * The string is owned by the library and stays valid until the thread's next
 * failing call. */
NVFP4_API const char* nvfp4_last_error(void);

/* Short name of a status code. */
NVFP4_API const char* nvfp4_status_string(nvfp4_status status);

/*
 * Tensor amax: *amax_inout = max(*amax_inout, max |W|) over a BF16 [rows, cols]
 * matrix (leading dimension ldw).  Follows the FP32 per-tensor scale of the
 * NVFP4 graphic on the "Raphael Friedmann" home page and the shared-scale rule
 * of the model card "Qwen3.8-27B-NVFP4" (merged members share one amax): zero
 * *amax_inout once, then call this once per member to get the merged amax.
 * amax_inout is one device fp32; the update is an atomic max, so concurrent
 * calls on one accumulator are safe.  cols must be a multiple of 8.
 * rows == 0 or cols == 0 is a no-op.
 */
NVFP4_API nvfp4_status nvfp4_amax(const uint16_t* w, int64_t rows, int64_t cols, int64_t ldw,
                        float* amax_inout, nvfp4_stream_t stream);

/*
 * Round-to-nearest NVFP4 quantization (imp docs/quantization.md, "imp-quantize":
 * plain round-to-nearest from the block absmax, no calibration) of a BF16
 * W [N, K] (leading dimension ldw) into q [N, K/2] and s [N, K/16].
 *
 * Arithmetic (IEEE fp32, round to nearest even, no contraction), per 16-block b
 * of row n with amax_b = max |w| over the block:
 *   g   = amax / 2688                      (written to *g_out)
 *   s   = E4M3_rne_satfinite((amax_b / 6) / g),   s = 0 when g == 0
 *   d   = e4m3(s) * g;   all 16 codes 0x0 when d == 0, else with r = 1 / d:
 *   code = E2M1_rne_satfinite(w * r)  (ties to the even code, sign kept,
 *          |w * r| > 6 saturates to 6; w == +-0 gives 0x0 / 0x8)
 *
 * amax: device fp32 holding the tensor amax to use (for a merged layer, the max
 *   over all members, as accumulated by nvfp4_amax).  NULL = compute this
 *   tensor's own amax first (then g_out is used as the accumulator and is
 *   overwritten with g at the end).  amax must not alias g_out.
 * g_out: device fp32 receiving g.  May be NULL when amax is given.
 * Output bytes are bit-exact functions of the inputs (deterministic).
 * N == 0 is a no-op apart from writing *g_out.
 */
NVFP4_API nvfp4_status nvfp4_quantize(const uint16_t* w, int64_t N, int64_t K, int64_t ldw,
                            const float* amax, uint8_t* q, uint8_t* s, float* g_out,
                            nvfp4_stream_t stream);

/*
 * Micro-scale search (MSE) quantization (imp docs/quantization.md, micro-scale
 * search paragraph: each block's FP8 micro-scale chosen by the least
 * reconstruction error over candidates around the absmax one; measured there
 * and reverted, kept here as the measured alternative to nvfp4_quantize).
 * Arguments, layouts, the amax / g_out handling and g are those of
 * nvfp4_quantize; per 16-block, with c0 the scale byte nvfp4_quantize writes:
 *   candidates: E4M3 codes c with |c - c0| <= window, clamped to 1..126
 *     (window 8 = one binade either side; window 0 is nvfp4_quantize);
 *   each candidate quantizes the block by nvfp4_quantize's element rule with
 *     d = e4m3(c) * g; its error sum_i (w_i - e2m1(code_i) * d)^2 is formed in
 *     IEEE fp64, each operation rounded on its own, in index order;
 *   the least error wins; ties go to the code nearest c0, then to the smaller;
 *   blocks with c0 == 0 get scale 0 and zero codes.
 * Output bytes are bit-exact functions of the inputs.  window outside 0..125
 * gives NVFP4_ERR_INVALID_ARG.  About 17 candidates of fp64 arithmetic per
 * block: several times the cost of nvfp4_quantize.
 */
NVFP4_API nvfp4_status nvfp4_quantize_mse(const uint16_t* w, int64_t N, int64_t K, int64_t ldw,
                                          const float* amax, int32_t window, uint8_t* q, uint8_t* s,
                                          float* g_out, nvfp4_stream_t stream);

/*
 * Batch-1 decode GEMV, y[n] = bf16_rn(g * sum_k W_deq[n, k] * x[k]) with fp32
 * accumulation ("Dense layers" pipeline of imp docs/quantization.md: the decode
 * path reads packed FP4 directly; weight-only per the model card).
 * x: BF16 [K]; q, s as above; g: device fp32; y: BF16 [N].
 * y must not overlap x, q or s.  N == 0 is a no-op.
 * Limits: K <= 49152 (x is staged in shared memory).
 */
NVFP4_API nvfp4_status nvfp4_gemv(const uint16_t* x, const uint8_t* q, const uint8_t* s,
                        const float* g, uint16_t* y, int64_t N, int64_t K,
                        nvfp4_stream_t stream);

/* nvfp4_gemv with flags (NVFP4_FLAG_*); nvfp4_gemv(...) is this with flags 0.
 * Unknown flag bits give NVFP4_ERR_INVALID_ARG. */
NVFP4_API nvfp4_status nvfp4_gemv_ex(const uint16_t* x, const uint8_t* q, const uint8_t* s,
                                     const float* g, uint16_t* y, int64_t N, int64_t K,
                                     uint32_t flags, nvfp4_stream_t stream);

/*
 * GEMM Y = X . W^T for M >= 1 rows of activations (32-user batched decode and
 * 512-token prefill of the model card "Qwen3.8-27B-NVFP4", "Measurements"),
 * same arithmetic as nvfp4_gemv per output.  M == 1 runs the GEMV.  M >= 2 with
 * K % 256 == 0 runs on the tensor cores (tcgen05, fp32 accumulation in tensor
 * memory): every product is exact, because the dequantized weights
 * e2m1 * e4m3 are exact f16 values and each row of X is copied to f16 scaled
 * by a power of two; rows whose non-zero magnitudes span more than 2^32 (or
 * that are not finite) are recomputed exactly in fp32 on CUDA cores.  g and the
 * row scale are applied in fp32 in the epilogue.  Other K (<= 49152) run one
 * GEMV per row of X.
 * workspace: device scratch of at least nvfp4_gemm_workspace_size(M, N, K)
 *   bytes, 16-byte aligned, not overlapping any argument (it receives the f16
 *   copy of X and the row scales); may be NULL when that size is 0.  Too small
 *   a workspace gives NVFP4_ERR_WORKSPACE.  Calls that share a workspace must
 *   be ordered (one stream).
 * Y must not overlap X, q or s.  M == 0 or N == 0 is a no-op.
 */
NVFP4_API nvfp4_status nvfp4_gemm(const uint16_t* X, int64_t ldx, const uint8_t* q, const uint8_t* s,
                        const float* g, uint16_t* Y, int64_t ldy, int64_t M, int64_t N,
                        int64_t K, void* workspace, size_t workspace_bytes,
                        nvfp4_stream_t stream);

/* nvfp4_gemm with flags (NVFP4_FLAG_*); nvfp4_gemm(...) is this with flags 0. */
NVFP4_API nvfp4_status nvfp4_gemm_ex(const uint16_t* X, int64_t ldx, const uint8_t* q, const uint8_t* s,
                                     const float* g, uint16_t* Y, int64_t ldy, int64_t M, int64_t N,
                                     int64_t K, void* workspace, size_t workspace_bytes, uint32_t flags,
                                     nvfp4_stream_t stream);

/* Bytes of workspace nvfp4_gemm needs for this shape (0 if none). */
NVFP4_API size_t nvfp4_gemm_workspace_size(int64_t M, int64_t N, int64_t K);

/* Size of the scratch array built into the library for nvfp4_gemm_noalloc. */
#define NVFP4_GEMM_NOALLOC_SCRATCH_BYTES (((size_t)8 << 20) + 4096)

/*
 * nvfp4_gemm_ex without a workspace argument: the scratch comes from an
 * 8 MiB + 4 KiB array compiled into the library (one per device), so the call
 * allocates nothing.  The pages have no counterpart of this entry point; it
 * is for callers that cannot allocate device memory (no allocator of their
 * own, or one that is closed while a step runs).
 * Arguments, layouts, flags and results are those of nvfp4_gemm_ex.
 * Limit: shapes whose nvfp4_gemm_workspace_size(M, N, K) exceeds
 *   NVFP4_GEMM_NOALLOC_SCRATCH_BYTES are rejected with NVFP4_ERR_WORKSPACE
 *   and launch nothing; every shape with M <= 1024 and M * K <= 2^22 fits
 *   (e.g. M = 512, K = 8192).
 * Set-up: the first call in each CUDA context (normally the device's primary
 *   context, current when the call is made) looks up the array's device
 *   address and caches it under the context's unique id; make that call
 *   before any stream capture in the context begins.  A call in a new context
 *   (after cudaDeviceReset, or with another context made current) looks the
 *   address up again.
 * Sharing: every call on a device uses the same array, which keeps what the
 *   last call wrote (nothing in it needs to start at zero).  Calls whose work
 *   overlaps on the GPU race on it: order them (e.g. one stream).
 */
NVFP4_API nvfp4_status nvfp4_gemm_noalloc(const uint16_t* X, int64_t ldx, const uint8_t* q, const uint8_t* s,
                                          const float* g, uint16_t* Y, int64_t ldy, int64_t M, int64_t N,
                                          int64_t K, uint32_t flags, nvfp4_stream_t stream);

/*
 * Grouped (MoE) decode GEMV over stacked experts ("MoE layers" pipeline of imp
 * docs/quantization.md: one contiguous [ne, N, K_packed] buffer per layer and
 * projection, read by the decode fast path).  For p = 0 .. P-1:
 *   Y[p, n] = bf16_rn( g[e] * sum_j e4m3(s[e, n, j]) * sum_i e2m1(q[e, n, 16j+i]) * X[t, 16j+i] )
 *   with e = expert_ids[p], t = token_ids[p].
 * X: BF16 [T, K], leading dimension ldx (elements, multiple of 8); q: [E, N, K/2];
 * s: [E, N, K/16]; g: fp32 [E] (each expert's own tensor scale); expert_ids,
 * token_ids: device int32 [P] (e.g. written by a router kernel earlier on the
 * stream: they are read after it completes); Y: BF16 [P, N], leading dimension
 * ldy >= N.  A problem whose ids are out of range gets a zero output row and is
 * counted for nvfp4_check_device_errors (NVFP4_ERR_INVALID_ARG).  P == 0 is a
 * no-op; P <= 65535; K <= 49152.  flags: NVFP4_FLAG_* (the static-weights flag
 * changes nothing here: the expert is known only after the previous kernel).
 */
NVFP4_API nvfp4_status nvfp4_gemv_grouped(const uint16_t* X, int64_t ldx, const uint8_t* q, const uint8_t* s,
                                          const float* g, const int32_t* expert_ids, const int32_t* token_ids,
                                          uint16_t* Y, int64_t ldy, int64_t P, int64_t E, int64_t T, int64_t N,
                                          int64_t K, uint32_t flags, nvfp4_stream_t stream);

/*
 * Diagnostic: every wait inside the pipelined kernels (the tensor-core GEMMs,
 * the W4A4 GEMM of nvfp4_w4a4.h and the TMA-fed decode GEMV) is bounded
 * (about 2 s); a CTA that gives up records it in a device counter and finishes
 * without hanging, leaving its outputs undefined.  This call reads and clears
 * those counters for the current device (it waits for prior work on the
 * legacy default stream) and returns NVFP4_ERR_TIMEOUT if one was non-zero,
 * else NVFP4_ERR_INVALID_ARG if grouped GEMVs met out-of-range ids or MXFP4
 * scales could not be restated (mxfp4.h, mxfp4_to_nvfp4_scales).
 */
NVFP4_API nvfp4_status nvfp4_check_device_errors(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H_ */

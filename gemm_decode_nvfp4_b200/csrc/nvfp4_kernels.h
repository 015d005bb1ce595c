// nvfp4_kernels.h -- internal launchers behind the C ABI (include/nvfp4.h).
// Each returns the CUDA error of its launch; arguments are validated by the
// caller in abi.cu before any of these runs.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "nvfp4.h"

namespace nvfp4 {

cudaError_t launch_amax(const uint16_t* w, int64_t rows, int64_t cols, int64_t ldw, float* amax,
                        cudaStream_t stream, int sms);
cudaError_t launch_quantize(const uint16_t* w, int64_t N, int64_t K, int64_t ldw,
                            const float* amax, uint8_t* q, uint8_t* s, float* g_out,
                            cudaStream_t stream, int sms);
cudaError_t launch_finalize_scale(float* amax_then_g, cudaStream_t stream);
// Micro-scale search (MSE) quantizer (quantize.cu): the quantize arithmetic with
// each block's scale chosen among the E4M3 codes within `window` of the
// round-to-nearest one by the least fp64 squared error.
cudaError_t launch_quantize_mse(const uint16_t* w, int64_t N, int64_t K, int64_t ldw, const float* amax, int window,
                                uint8_t* q, uint8_t* s, float* g_out, cudaStream_t stream, int sms);
// Decode GEMV (gemv.cu).  static_weights: q, s and g are not written by work
// still running on the stream, so they may be read before it completes
// (programmatic dependent launch).  splits: 0 lets the launcher choose how many
// CTAs of a cluster split K (1, 2, 4 or 8); a value fixes it, and a split that
// does not fit the shape returns cudaErrorInvalidConfiguration (1 = no split).
cudaError_t launch_gemv(const uint16_t* x, const uint8_t* q, const uint8_t* s, const float* g,
                        uint16_t* y, int64_t N, int64_t K, int sms, bool static_weights, cudaStream_t stream,
                        int splits = 0);
// MXFP4 decode GEMV (gemv.cu): one UE8M0 scale per 32 elements, no tensor
// scale; K a multiple of 32.
cudaError_t launch_gemv_mx(const uint16_t* x, const uint8_t* q, const uint8_t* s, uint16_t* y, int64_t N,
                           int64_t K, int sms, bool static_weights, cudaStream_t stream, int splits = 0);
// Whether the split-K decode GEMV can run this shape with the given split.
bool gemv_split_fits(int64_t N, int64_t K, int sms, bool mx, int splits);
// Grouped (MoE) decode GEMV (gemv.cu): problem p multiplies expert expert_ids[p]
// of the stacked weights q [E, N, K/2], s [E, N, K/16], g [E] by row
// token_ids[p] of X [T, K] (leading dimension ldx) into row p of Y (ldy).
cudaError_t launch_gemv_grouped(const uint16_t* X, int64_t ldx, const uint8_t* q, const uint8_t* s,
                                const float* g, const int* expert_ids, const int* token_ids, uint16_t* Y,
                                int64_t ldy, int64_t P, int64_t E, int64_t T, int64_t N, int64_t K, int sms,
                                cudaStream_t stream);
// Problems of grouped GEMVs whose ids were out of range since the last read.
cudaError_t read_and_clear_gemv_bad_ids(unsigned int* count);
// W4A4 (gemm_w4a4.cu): X quantized by the weights' rule with
// g_x = *x_amax / 2688 into row-major codes qx [M, K/2] and scales sx in the
// tensor core's scale-factor layout (512-byte atoms per 128 rows x 64 k,
// rows padded with zero scales to a multiple of 256); the weight scales
// rearranged once into the same layout (rows padded to a multiple of 128);
// the block-scaled FP4 GEMM Y = bf16(g * g_x * sum sx sw qx qw).
// amax: given ? amax[0] is read : amax[0] receives max |X| and amax[1 .. 256]
// hold per-CTA partial maxima (NVFP4_W4A4_AMAX_FLOATS floats in all).
cudaError_t launch_quantize_x_mma(const uint16_t* X, int64_t ldx, int64_t M, int64_t K, float* amax, bool given,
                                  uint8_t* qx, uint8_t* sx, cudaStream_t stream, int sms);
cudaError_t launch_scales_to_mma(const uint8_t* s, int64_t N, int64_t K, uint8_t* s_mma, cudaStream_t stream,
                                 int sms);
cudaError_t launch_gemm_w4a4(const uint8_t* qx, const uint8_t* sx, const float* x_amax, const uint8_t* q,
                             const uint8_t* s_mma, const float* g, uint16_t* Y, int64_t ldy, int64_t M, int64_t N,
                             int64_t K, bool static_weights, bool pair, cudaStream_t stream, int sms);
cudaError_t read_and_clear_w4a4_timeouts(unsigned int* count);
// MXFP4 scales restated as NVFP4 scales s_nv [N, K/16] and a power-of-two
// tensor scale g (quantize.cu); non-zero blocks outside the E4M3 window are
// counted (read_and_clear_mx_out_of_window).
cudaError_t launch_mx_to_nvfp4(const uint8_t* q, const uint8_t* s_mx, int64_t N, int64_t K, uint8_t* s_nv,
                               float* g, cudaStream_t stream, int sms);
cudaError_t read_and_clear_mx_out_of_window(unsigned int* count);
// MXFP4 round-to-nearest quantizer (quantize.cu); K a multiple of 32.
cudaError_t launch_mx_quantize(const uint16_t* w, int64_t N, int64_t K, int64_t ldw, uint8_t* q, uint8_t* s,
                               cudaStream_t stream, int sms);
// CTAs of the decode GEMV whose bounded pipeline wait gave up since the last read.
cudaError_t read_and_clear_gemv_timeouts(unsigned int* count);

// Tensor-core GEMM (gemm_tc.cu): shapes it covers, the launcher, and the count
// of CTAs whose bounded pipeline wait gave up since the last read.
// The workspace holds the per-row exponents and the f16 copy of X (see
// gemm_tc_workspace_bytes); it must be 16-byte aligned.
bool gemm_tc_supported(int64_t M, int64_t N, int64_t K);
size_t gemm_tc_workspace_bytes(int64_t M, int64_t K);
cudaError_t launch_gemm_tc(const uint16_t* X, int64_t ldx, const uint8_t* q, const uint8_t* s, const float* g,
                           uint16_t* Y, int64_t ldy, int64_t M, int64_t N, int64_t K, void* workspace,
                           bool static_weights, cudaStream_t stream);
cudaError_t read_and_clear_gemm_timeouts(unsigned int* count);

// X pre-pass of the tensor-core GEMMs (gemm_tc.cu): per-row exponents and the
// exact f16 copy of X, written into `workspace` (gemm_prep_workspace_bytes).
size_t gemm_prep_workspace_bytes(int64_t M, int64_t K);
cudaError_t launch_gemm_prep(const uint16_t* X, int64_t ldx, int64_t M, int64_t K, void* workspace, int** info,
                             uint16_t** xh, cudaStream_t stream);

// Decode GEMV and small-M GEMM (gemm_small.cu, 1 <= M <= 64, K % 256 == 0):
// dequantized weights in tensor memory.  M <= 8 needs no workspace (the kernel
// converts X itself); larger M use the X pre-pass.
bool gemm_small_supported(int64_t M, int64_t N, int64_t K);
size_t gemm_small_workspace_bytes(int64_t M, int64_t K);
cudaError_t launch_gemm_small(const uint16_t* X, int64_t ldx, const uint8_t* q, const uint8_t* s, const float* g,
                              uint16_t* Y, int64_t ldy, int64_t M, int64_t N, int64_t K, void* workspace,
                              bool static_weights, cudaStream_t stream);
cudaError_t read_and_clear_small_timeouts(unsigned int* count);

// Record a message for nvfp4_last_error() on this thread and return st (or
// NVFP4_ERR_CUDA for a CUDA error), for entry points defined outside abi.cu.
nvfp4_status report_error(nvfp4_status st, const char* fmt, ...);
nvfp4_status report_cuda_error(cudaError_t e, const char* what);

// Largest K the GEMV accepts (x is staged in shared memory as fp32).
constexpr int64_t kGemvMaxK = 49152;

}  // namespace nvfp4

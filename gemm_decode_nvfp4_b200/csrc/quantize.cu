// quantize.cu -- tensor amax and round-to-nearest BF16 -> NVFP4 quantization.
//
// Follows imp docs/quantization.md, "imp-quantize" section (plain
// round-to-nearest from the absmax of each 16-block, E4M3 micro-scale, FP32
// tensor scale) and the model card "Qwen3.8-27B-NVFP4", paragraph after
// "What is quantized" (merged layers share the tensor scale: the caller
// accumulates one amax over all members).
//
// Both kernels stream HBM once: amax reads W (2 B/element); quantize reads W
// and writes 0.5 + 1/16 B/element.  Each thread owns whole 16-element blocks
// (32 B in, 8 B of codes + 1 scale byte out), so loads are 16-byte vectors
// that are contiguous across a warp and blocks never straddle threads.
#include "nvfp4_kernels.h"
#include "nvfp4_device.cuh"
#include "nvfp4_quant.cuh"

namespace nvfp4 {

namespace {

// amax over rows x cols (cols % 8 == 0), atomically max-merged into *out.
__global__ void __launch_bounds__(256) amax_kernel(const uint16_t* __restrict__ w, int64_t rows,
                                                   int64_t cols, int64_t ldw,
                                                   float* __restrict__ out) {
  __shared__ float red[8];
  const int64_t vpr = cols / 8;
  const int64_t total = rows * vpr;
  float m = 0.0f;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (ldw == cols) {
    // contiguous rows: one flat array, four independent 16-byte loads in flight
    const uint4* wv = reinterpret_cast<const uint4*>(w);
    for (; t + 3 * stride < total; t += 4 * stride) {
      const uint4 a = ld_stream_v4(wv + t), b = ld_stream_v4(wv + t + stride);
      const uint4 c = ld_stream_v4(wv + t + 2 * stride), d = ld_stream_v4(wv + t + 3 * stride);
      m = absmax8(d, absmax8(c, absmax8(b, absmax8(a, m))));
    }
    for (; t < total; t += stride) m = absmax8(ld_stream_v4(wv + t), m);
  } else {
    for (; t < total; t += stride) {
      const int64_t r = t / vpr, c = (t - r * vpr) * 8;
      m = absmax8(ld_stream_v4(w + r * ldw + c), m);
    }
  }
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
    m = warp_max(m);
    // non-negative floats order like their bit patterns
    if (threadIdx.x == 0) atomicMax(reinterpret_cast<unsigned int*>(out), __float_as_uint(m));
  }
}

// Quantize the 16 BF16 values of (v0, v1) and store 8 code bytes and the scale.
__device__ __forceinline__ void quantize_store(uint4 v0, uint4 v1, float g, uint8_t* qd, uint8_t* sd) {
  const uint32_t wv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
  float f[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    f[2 * i] = bf16lo_to_float(wv[i]);
    f[2 * i + 1] = bf16hi_to_float(wv[i]);
  }
  uint32_t sc;
  uint2 codes;
  quantize_block(f, g, sc, codes);
  *reinterpret_cast<uint2*>(qd) = codes;
  *sd = static_cast<uint8_t>(sc);
}

__global__ void __launch_bounds__(256) quantize_kernel(const uint16_t* __restrict__ w, int64_t N,
                                                       int64_t K, int64_t ldw,
                                                       const float* __restrict__ amax,
                                                       uint8_t* __restrict__ q,
                                                       uint8_t* __restrict__ s,
                                                       float* __restrict__ g_out) {
  const float g = __fdiv_rn(*amax, 2688.0f);
  if (g_out != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *g_out = g;
  const int64_t bpr = K / 16;
  const int64_t total = N * bpr;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (ldw == K) {
    // contiguous rows: block t reads w[16t ..], writes q[8t ..] and s[t]; two
    // blocks (four 16-byte loads) in flight per thread
    for (; t + stride < total; t += 2 * stride) {
      const uint4* s0 = reinterpret_cast<const uint4*>(w + t * 16);
      const uint4* s1 = reinterpret_cast<const uint4*>(w + (t + stride) * 16);
      const uint4 a0 = ld_stream_v4(s0), a1 = ld_stream_v4(s0 + 1);
      const uint4 b0 = ld_stream_v4(s1), b1 = ld_stream_v4(s1 + 1);
      quantize_store(a0, a1, g, q + t * 8, s + t);
      quantize_store(b0, b1, g, q + (t + stride) * 8, s + t + stride);
    }
    if (t < total) {
      const uint4* s0 = reinterpret_cast<const uint4*>(w + t * 16);
      quantize_store(ld_stream_v4(s0), ld_stream_v4(s0 + 1), g, q + t * 8, s + t);
    }
    return;
  }
  for (; t < total; t += stride) {
    const int64_t n = t / bpr, b = t - n * bpr;
    const uint16_t* src = w + n * ldw + b * 16;
    const uint4 v0 = ld_stream_v4(src), v1 = ld_stream_v4(src + 8);
    const uint32_t wv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    float f[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      f[2 * i] = bf16lo_to_float(wv[i]);
      f[2 * i + 1] = bf16hi_to_float(wv[i]);
    }
    uint32_t sc;
    uint2 codes;
    quantize_block(f, g, sc, codes);
    *reinterpret_cast<uint2*>(q + n * (K / 2) + b * 8) = codes;
    s[n * bpr + b] = static_cast<uint8_t>(sc);
  }
}

// ---------------------------------------------------------------------- MXFP4
//
// imp docs/quantization.md, MXFP4 paragraph: the NVFP4 nibble layout with one
// UE8M0 (power-of-two) micro-scale per 32 elements and no tensor scale,
// quantized round-to-nearest.  Scale rule (the pages give none; this is the
// shared-exponent rule of the microscaling convention): X = 2^(floor(log2
// amax_b) - 2), so the block maximum lands in [4, 8) before rounding and 6
// clips it; byte = that exponent + 127, at least 0.  For a finite amax with
// biased fp32 exponent field ef, floor(log2 amax) = ef - 127 when ef > 0, so
// byte = max(ef - 2, 0), and zero or subnormal maxima give byte 0.
// Elements are multiplied by 2^(127 - byte), a normal fp32 for every byte
// 0..252 (exact), and rounded to E2M1 by the same RNE, saturating, sign-keeping
// conversion as NVFP4.

// One 32-element block: 16 code bytes and the UE8M0 byte.
__device__ __forceinline__ void mx_quantize_store(const uint4 (&v)[4], uint8_t* qd, uint8_t* sd) {
  float f[32];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t w4[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[8 * j + 2 * i] = bf16lo_to_float(w4[i]);
      f[8 * j + 2 * i + 1] = bf16hi_to_float(w4[i]);
    }
  }
  float amax_b = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax_b = fmaxf(amax_b, fabsf(f[i]));
  const uint32_t ef = (__float_as_uint(amax_b) >> 23) & 0xFFu;
  const uint32_t byte = ef >= 2u ? ef - 2u : 0u;
  const float m = __uint_as_float((254u - byte) << 23);  // 2^(127 - byte)
  uint32_t c[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) c[i] = float2_to_e2m1x2_satfinite(__fmul_rn(f[2 * i], m), __fmul_rn(f[2 * i + 1], m));
  uint4 codes;
  codes.x = c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24);
  codes.y = c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24);
  codes.z = c[8] | (c[9] << 8) | (c[10] << 16) | (c[11] << 24);
  codes.w = c[12] | (c[13] << 8) | (c[14] << 16) | (c[15] << 24);
  *reinterpret_cast<uint4*>(qd) = codes;
  *sd = static_cast<uint8_t>(byte);
}

// Thread t owns 32-element blocks t, t + stride, ...: 64 bytes in (four 16-byte
// loads), 16 code bytes and one scale byte out.
__global__ void __launch_bounds__(256) mx_quantize_kernel(const uint16_t* __restrict__ w, int64_t N, int64_t K,
                                                          int64_t ldw, uint8_t* __restrict__ q,
                                                          uint8_t* __restrict__ s) {
  const int64_t bpr = K / 32;
  const int64_t total = N * bpr;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (ldw == K) {
    // contiguous rows: blocks t and t + stride together, eight 16-byte loads in flight
    for (; t + stride < total; t += 2 * stride) {
      const uint4* a = reinterpret_cast<const uint4*>(w + t * 32);
      const uint4* b = reinterpret_cast<const uint4*>(w + (t + stride) * 32);
      uint4 va[4], vb[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        va[j] = ld_stream_v4(a + j);
        vb[j] = ld_stream_v4(b + j);
      }
      mx_quantize_store(va, q + t * 16, s + t);
      mx_quantize_store(vb, q + (t + stride) * 16, s + t + stride);
    }
  }
  for (; t < total; t += stride) {
    const int64_t n = t / bpr, b = t - n * bpr;
    const uint4* src = reinterpret_cast<const uint4*>(w + n * ldw + b * 32);
    uint4 v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = ld_stream_v4(src + j);
    mx_quantize_store(v, q + t * 16, s + t);
  }
}

// ----------------------------------------------- MXFP4 scales as NVFP4 scales
//
// The two formats share the nibble layout, so MXFP4 weights run on the NVFP4
// GEMMs once their scales are restated: with g = 2^G, a UE8M0 block scale 2^k
// is the E4M3 scale 2^(k - G) of both 16-element halves of its 32-block (E4M3
// holds the powers 2^-9 .. 2^8).  G = (largest k of a block with a non-zero
// code) - 8, found by a max-reduction into the g slot itself (as an int,
// starting from the byte pattern 0x80808080), so no scratch memory is needed.

// Blocks with the NaN scale byte 255, and non-zero blocks whose scale fell
// outside the E4M3 window.
__device__ unsigned int g_mx_out_of_window = 0;

constexpr int kNoBlock = (int)0x80808080;  // the reduction's start value: no non-zero block yet

__device__ __forceinline__ bool mx_block_nonzero(const uint8_t* q, int64_t b) {
  const uint4 w = *reinterpret_cast<const uint4*>(q + 16 * b);
  return ((w.x | w.y | w.z | w.w) & 0x77777777u) != 0u;  // any magnitude bits (codes 0x0 / 0x8 are zeros)
}

__global__ void __launch_bounds__(256) mx_kmax_kernel(const uint8_t* __restrict__ q, const uint8_t* __restrict__ s,
                                                      int64_t nblocks, int* __restrict__ kmax) {
  int m = kNoBlock;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; b < nblocks; b += stride)
    if (s[b] != 255u && mx_block_nonzero(q, b)) m = max(m, (int)s[b] - 127);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0 && m != kNoBlock) atomicMax(kmax, m);
}

__device__ __forceinline__ int mx_tensor_exponent(int kmax) { return kmax == kNoBlock ? 0 : kmax - 8; }

__global__ void __launch_bounds__(256) mx_to_nv_kernel(const uint8_t* __restrict__ q, const uint8_t* __restrict__ s,
                                                       int64_t nblocks, const int* __restrict__ kmax,
                                                       uint8_t* __restrict__ s_nv) {
  const int G = mx_tensor_exponent(*kmax);
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; b < nblocks; b += stride) {
    uint32_t byte = 0;
    if (s[b] == 255u) {  // NaN scale: no finite NVFP4 scale holds it
      atomicAdd(&g_mx_out_of_window, 1u);
    } else if (mx_block_nonzero(q, b)) {
      const int j = (int)s[b] - 127 - G;
      if (j < -9)
        atomicAdd(&g_mx_out_of_window, 1u);
      else
        byte = j >= -6 ? (uint32_t)(j + 7) << 3 : 1u << (j + 9);  // 2^j in E4M3 (subnormal below 2^-6)
    }
    *reinterpret_cast<uint16_t*>(s_nv + 2 * b) = (uint16_t)(byte | (byte << 8));
  }
}

__global__ void mx_g_kernel(float* g) {  // the reduced exponent in the g slot -> g = 2^G
  const int G = mx_tensor_exponent(*reinterpret_cast<const int*>(g));
  *g = G >= -126 ? __uint_as_float((uint32_t)(G + 127) << 23) : __uint_as_float(1u << (G + 149));
}

// ------------------------------------------------- micro-scale search (MSE)
//
// imp docs/quantization.md, micro-scale search paragraph: each block's E4M3
// micro-scale is chosen by the least reconstruction error over FP8 candidates
// around the absmax scale (the pages measured it at about 6x the cost of the
// round-to-nearest quantizer for a 0.7% perplexity change and reverted it).
// The pages give no window, precision or tie rule; the readings taken here:
//   - candidates: the E4M3 codes c with |c - c0| <= window, clamped to
//     1..126, where c0 is the round-to-nearest scale of quantize_block;
//   - each candidate quantizes the block by the round-to-nearest element rule
//     with its own d = e4m3(c) * g (r = 1 / d, E2M1 RNE of w * r, zeros keep
//     their sign); candidates with d == 0 are skipped;
//   - its error is sum_i (w_i - e2m1(code_i) * d)^2 in IEEE fp64, each
//     product, difference and sum rounded on its own, in index order (so that
//     every comparison below is a deterministic function of the inputs);
//   - the least error wins, ties to the code nearest c0, then to the smaller
//     code (candidates are visited in increasing order);
//   - a block whose c0 is 0 (zero block, or g = 0) keeps scale 0 and zero codes.
// window = 0 gives the round-to-nearest quantizer.  The error loop is fp64
// work (about 64 operations per candidate): this kernel is bound by the FP64
// pipe, not by HBM.
__device__ __forceinline__ void quantize_block_mse(const float (&f)[16], float g, int window, uint32_t& scale,
                                                   uint2& codes) {
  float amax_b = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax_b = fmaxf(amax_b, fabsf(f[i]));
  int c0 = 0;
  if (g != 0.0f) c0 = (int)float_to_e4m3_satfinite(__fdiv_rn(__fdiv_rn(amax_b, 6.0f), g));
  int best_c = 0;
  uint32_t best[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (c0 != 0) {
    double best_err = __longlong_as_double(0x7FF0000000000000ll);  // +inf
    const int lo = max(1, c0 - window), hi = min(126, c0 + window);
    for (int c = lo; c <= hi; ++c) {
      const float d = __fmul_rn(e4m3_to_float((uint32_t)c), g);
      if (d == 0.0f) continue;
      const float r = __frcp_rn(d);
      const double dd = (double)d;
      uint32_t cc[8];
      double err = 0.0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float a = (f[2 * i] == 0.0f) ? f[2 * i] : __fmul_rn(f[2 * i], r);
        const float b = (f[2 * i + 1] == 0.0f) ? f[2 * i + 1] : __fmul_rn(f[2 * i + 1], r);
        cc[i] = float2_to_e2m1x2_satfinite(a, b);
        const float2 v = f16x2_to_float2(e2m1x2_to_f16x2(cc[i]));  // the two quantized values / d
        const double e0 = __dsub_rn((double)f[2 * i], __dmul_rn((double)v.x, dd));
        err = __dadd_rn(err, __dmul_rn(e0, e0));
        const double e1 = __dsub_rn((double)f[2 * i + 1], __dmul_rn((double)v.y, dd));
        err = __dadd_rn(err, __dmul_rn(e1, e1));
      }
      const int dc = abs(c - c0), db = abs(best_c - c0);
      if (err < best_err || (err == best_err && (dc < db || (dc == db && c < best_c)))) {
        best_err = err;
        best_c = c;
#pragma unroll
        for (int i = 0; i < 8; ++i) best[i] = cc[i];
      }
    }
  }
  scale = (uint32_t)best_c;
  codes.x = best[0] | (best[1] << 8) | (best[2] << 16) | (best[3] << 24);
  codes.y = best[4] | (best[5] << 8) | (best[6] << 16) | (best[7] << 24);
}

// One thread per 16-element block (grid-stride): 32 bytes in, 8 code bytes
// and the scale byte out.
__global__ void __launch_bounds__(256) quantize_mse_kernel(const uint16_t* __restrict__ w, int64_t N, int64_t K,
                                                           int64_t ldw, const float* __restrict__ amax, int window,
                                                           uint8_t* __restrict__ q, uint8_t* __restrict__ s,
                                                           float* __restrict__ g_out) {
  const float g = __fdiv_rn(*amax, 2688.0f);
  if (g_out != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *g_out = g;
  const int64_t bpr = K / 16;
  const int64_t total = N * bpr;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total; t += stride) {
    const int64_t n = t / bpr, b = t - n * bpr;
    const uint16_t* src = w + n * ldw + b * 16;
    const uint4 v0 = ld_stream_v4(src), v1 = ld_stream_v4(src + 8);
    const uint32_t wv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    float f[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      f[2 * i] = bf16lo_to_float(wv[i]);
      f[2 * i + 1] = bf16hi_to_float(wv[i]);
    }
    uint32_t sc;
    uint2 codes;
    quantize_block_mse(f, g, window, sc, codes);
    *reinterpret_cast<uint2*>(q + n * (K / 2) + b * 8) = codes;
    s[n * bpr + b] = static_cast<uint8_t>(sc);
  }
}

__global__ void finalize_scale_kernel(float* amax_then_g) {
  *amax_then_g = __fdiv_rn(*amax_then_g, 2688.0f);
}

int grid_for(int64_t work_items, int sms) {
  const int64_t blocks = (work_items + 255) / 256;
  const int64_t cap = (int64_t)sms * 8;
  return (int)(blocks < 1 ? 1 : (blocks < cap ? blocks : cap));
}

}  // namespace

cudaError_t launch_amax(const uint16_t* w, int64_t rows, int64_t cols, int64_t ldw, float* amax,
                        cudaStream_t stream, int sms) {
  const int grid = grid_for(rows * (cols / 8), sms);
  amax_kernel<<<grid, 256, 0, stream>>>(w, rows, cols, ldw, amax);
  return cudaGetLastError();
}

cudaError_t launch_quantize(const uint16_t* w, int64_t N, int64_t K, int64_t ldw,
                            const float* amax, uint8_t* q, uint8_t* s, float* g_out,
                            cudaStream_t stream, int sms) {
  const int grid = grid_for(N * (K / 16), sms);
  quantize_kernel<<<grid, 256, 0, stream>>>(w, N, K, ldw, amax, q, s, g_out);
  return cudaGetLastError();
}

cudaError_t launch_quantize_mse(const uint16_t* w, int64_t N, int64_t K, int64_t ldw, const float* amax, int window,
                                uint8_t* q, uint8_t* s, float* g_out, cudaStream_t stream, int sms) {
  const int grid = grid_for(N * (K / 16), sms);
  quantize_mse_kernel<<<grid, 256, 0, stream>>>(w, N, K, ldw, amax, window, q, s, g_out);
  return cudaGetLastError();
}

cudaError_t launch_mx_quantize(const uint16_t* w, int64_t N, int64_t K, int64_t ldw, uint8_t* q, uint8_t* s,
                               cudaStream_t stream, int sms) {
  const int grid = grid_for(N * (K / 32), sms);
  mx_quantize_kernel<<<grid, 256, 0, stream>>>(w, N, K, ldw, q, s);
  return cudaGetLastError();
}

cudaError_t launch_mx_to_nvfp4(const uint8_t* q, const uint8_t* s_mx, int64_t N, int64_t K, uint8_t* s_nv,
                               float* g, cudaStream_t stream, int sms) {
  const int64_t nblocks = N * (K / 32);
  cudaError_t e = cudaMemsetAsync(g, 0x80, sizeof(float), stream);  // kNoBlock
  if (e != cudaSuccess) return e;
  const int grid = grid_for(nblocks, sms);
  mx_kmax_kernel<<<grid, 256, 0, stream>>>(q, s_mx, nblocks, reinterpret_cast<int*>(g));
  mx_to_nv_kernel<<<grid, 256, 0, stream>>>(q, s_mx, nblocks, reinterpret_cast<const int*>(g), s_nv);
  mx_g_kernel<<<1, 1, 0, stream>>>(g);
  return cudaGetLastError();
}

cudaError_t read_and_clear_mx_out_of_window(unsigned int* count) {
  cudaError_t e = cudaMemcpyFromSymbol(count, g_mx_out_of_window, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  const unsigned int zero = 0;
  return cudaMemcpyToSymbol(g_mx_out_of_window, &zero, sizeof(unsigned int));
}

cudaError_t launch_finalize_scale(float* amax_then_g, cudaStream_t stream) {
  finalize_scale_kernel<<<1, 1, 0, stream>>>(amax_then_g);
  return cudaGetLastError();
}

}  // namespace nvfp4

// gemv.cu -- batch-1 decode GEMV over packed NVFP4 weights (W4A16).
//
// The decode path of imp docs/quantization.md ("Dense layers" pipeline: an
// NVFP4 GEMV reading the packed nibbles, E4M3 micro-scales and FP32 tensor
// scale directly) with BF16 activations (model card "Qwen3.8-27B-NVFP4",
// "What is quantized": weight-only).  The pages' kernel targets sm_120 with a
// prmt register LUT; here the sm_100a cvt.rn.f16x2.e2m1x2 instruction decodes
// two codes per instruction (exactly, sign included) and the products are
// accumulated with packed fp32x2 FMAs.
//
// Work split: a warp owns R consecutive rows; lane l reads the 16-byte chunks
// l, l+32, ... of each row (512 contiguous bytes per warp-load, one 16-bit
// scale load per chunk).  x is staged once per CTA in shared memory as fp32.
// Per chunk and row: 8 cvt + 16 f16->f32 + 16 FFMA2 for 32 weights, plus two
// block sums and two scale FMAs.  The weight stream (0.5625 B/weight) is the
// roofline: HBM bandwidth.
#include "nvfp4_kernels.h"
#include "nvfp4_device.cuh"

namespace nvfp4 {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

// CB = bytes of packed codes per lane per step (16, or 8 when K % 32 != 0).
template <int R, int CB>
__global__ void __launch_bounds__(kThreads) gemv_kernel(const uint16_t* __restrict__ x,
                                                        const uint8_t* __restrict__ q,
                                                        const uint8_t* __restrict__ s,
                                                        const float* __restrict__ g,
                                                        uint16_t* __restrict__ y, int N, int K) {
  extern __shared__ __align__(16) float xs[];  // K fp32
  constexpr int kElems = 2 * CB;               // weights per lane-chunk
  constexpr int kBlocks = kElems / 16;         // scales per lane-chunk (2 or 1)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = (blockIdx.x * kWarps + warp) * R;
  const int row_bytes = K >> 1;
  const int row_scales = K >> 4;
  const int steps = (row_bytes + 32 * CB - 1) / (32 * CB);

  auto load = [&](int step, uint32_t (&wq)[R][CB / 4], uint32_t (&ws)[R]) {
    const int off = step * 32 * CB + lane * CB;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int row = row0 + r;
      if (row < N && off < row_bytes) {
        const uint8_t* pq = q + (int64_t)row * row_bytes + off;
        const uint8_t* ps = s + (int64_t)row * row_scales + off / 8;
        if constexpr (CB == 16) {
          const uint4 v = ld_stream_v4(pq);
          wq[r][0] = v.x; wq[r][1] = v.y; wq[r][2] = v.z; wq[r][3] = v.w;
          ws[r] = *reinterpret_cast<const uint16_t*>(ps);
        } else {
          const uint2 v = ld_stream_v2(pq);
          wq[r][0] = v.x; wq[r][1] = v.y;
          ws[r] = *ps;
        }
      } else {
#pragma unroll
        for (int i = 0; i < CB / 4; ++i) wq[r][i] = 0;
        ws[r] = 0;
      }
    }
  };

  uint32_t wq[R][CB / 4], ws[R];
  load(0, wq, ws);  // first weights in flight before x is staged

  for (int i = threadIdx.x; i < (K >> 3); i += kThreads) {
    const uint4 v = *reinterpret_cast<const uint4*>(x + 8 * i);
    float4* dst = reinterpret_cast<float4*>(xs) + 2 * i;
    dst[0] = make_float4(bf16lo_to_float(v.x), bf16hi_to_float(v.x), bf16lo_to_float(v.y),
                         bf16hi_to_float(v.y));
    dst[1] = make_float4(bf16lo_to_float(v.z), bf16hi_to_float(v.z), bf16lo_to_float(v.w),
                         bf16hi_to_float(v.w));
  }
  __syncthreads();

  float acc[R];
#pragma unroll
  for (int r = 0; r < R; ++r) acc[r] = 0.0f;

  for (int step = 0; step < steps; ++step) {
    uint32_t nq[R][CB / 4], ns[R];
    if (step + 1 < steps) load(step + 1, nq, ns);
    const int off = step * 32 * CB + lane * CB;
    if (off < row_bytes) {
      const float* xp = xs + 2 * off;
      float2 part[R][kBlocks];
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int b = 0; b < kBlocks; ++b) part[r][b] = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int wi = 0; wi < CB / 4; ++wi) {  // 8 weights per 32-bit word
        const float4 xa = reinterpret_cast<const float4*>(xp)[2 * wi];
        const float4 xb = reinterpret_cast<const float4*>(xp)[2 * wi + 1];
        const float2 x01 = make_float2(xa.x, xa.y), x23 = make_float2(xa.z, xa.w);
        const float2 x45 = make_float2(xb.x, xb.y), x67 = make_float2(xb.z, xb.w);
        const int b = wi / 2;  // two words per 16-block
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const uint32_t word = wq[r][wi];
          float2& p = part[r][b];
          p = __ffma2_rn(f16x2_to_float2(e2m1x2_byte_to_f16x2<0>(word)), x01, p);
          p = __ffma2_rn(f16x2_to_float2(e2m1x2_byte_to_f16x2<1>(word)), x23, p);
          p = __ffma2_rn(f16x2_to_float2(e2m1x2_byte_to_f16x2<2>(word)), x45, p);
          p = __ffma2_rn(f16x2_to_float2(e2m1x2_byte_to_f16x2<3>(word)), x67, p);
        }
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float2 sc = f16x2_to_float2(e4m3x2_to_f16x2(ws[r]));
        acc[r] = fmaf(part[r][0].x + part[r][0].y, sc.x, acc[r]);
        if constexpr (kBlocks == 2) acc[r] = fmaf(part[r][1].x + part[r][1].y, sc.y, acc[r]);
      }
    }
    if (step + 1 < steps) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
#pragma unroll
        for (int i = 0; i < CB / 4; ++i) wq[r][i] = nq[r][i];
        ws[r] = ns[r];
      }
    }
  }

  const float gv = *g;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    float v = acc[r];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    acc[r] = v;
  }
  if (lane < R) {
    float v = acc[0];
#pragma unroll
    for (int r = 1; r < R; ++r)
      if (lane == r) v = acc[r];
    const int row = row0 + lane;
    if (row < N) {
      const __nv_bfloat16 o = __float2bfloat16_rn(v * gv);
      y[row] = *reinterpret_cast<const uint16_t*>(&o);
    }
  }
}

template <int R, int CB>
cudaError_t launch(const uint16_t* x, const uint8_t* q, const uint8_t* s, const float* g,
                   uint16_t* y, int N, int K, cudaStream_t stream) {
  const size_t smem = (size_t)K * sizeof(float);
  auto kern = gemv_kernel<R, CB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int rows_per_cta = kWarps * R;
  const int grid = (N + rows_per_cta - 1) / rows_per_cta;
  kern<<<grid, kThreads, smem, stream>>>(x, q, s, g, y, N, K);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemv(const uint16_t* x, const uint8_t* q, const uint8_t* s, const float* g,
                        uint16_t* y, int64_t N, int64_t K, cudaStream_t stream) {
  if (K % 32 == 0) return launch<4, 16>(x, q, s, g, y, (int)N, (int)K, stream);
  return launch<4, 8>(x, q, s, g, y, (int)N, (int)K, stream);
}

}  // namespace nvfp4

// nvfp4_quant.cuh -- the round-to-nearest NVFP4 block rule shared by the
// weight quantizer (quantize.cu) and the W4A4 activation quantizer
// (gemm_w4a4.cu), and two reductions they both use.
//
// imp docs/quantization.md, "imp-quantize" section: per 16-element block,
// scale = E4M3_rne_satfinite(amax_b / 6 / g), then every element
// E2M1_rne_satfinite(w / (scale * g)); g = tensor amax / 2688.
#pragma once

#include "nvfp4_device.cuh"

namespace nvfp4 {
namespace {

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

__device__ __forceinline__ float absmax8(uint4 v, float m) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m = fmaxf(m, fabsf(bf16lo_to_float(w[i])));
    m = fmaxf(m, fabsf(bf16hi_to_float(w[i])));
  }
  return m;
}

// One 16-element block: scale byte and 8 code bytes.
__device__ __forceinline__ void quantize_block(const float (&f)[16], float g, uint32_t& scale,
                                               uint2& codes) {
  float amax_b = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax_b = fmaxf(amax_b, fabsf(f[i]));
  uint32_t sc = 0;
  if (g != 0.0f) sc = float_to_e4m3_satfinite(__fdiv_rn(__fdiv_rn(amax_b, 6.0f), g));
  const float d = __fmul_rn(e4m3_to_float(sc), g);
  uint32_t c[8];
  if (d == 0.0f) {
#pragma unroll
    for (int i = 0; i < 8; ++i) c[i] = 0;
  } else {
    const float r = __frcp_rn(d);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      // +-0 keeps its sign even when r overflowed to infinity
      const float lo = (f[2 * i] == 0.0f) ? f[2 * i] : __fmul_rn(f[2 * i], r);
      const float hi = (f[2 * i + 1] == 0.0f) ? f[2 * i + 1] : __fmul_rn(f[2 * i + 1], r);
      c[i] = float2_to_e2m1x2_satfinite(lo, hi);
    }
  }
  scale = sc;
  codes.x = c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24);
  codes.y = c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24);
}

// Quantize the 16 BF16 values of (v0, v1): scale byte and 8 code bytes.
__device__ __forceinline__ void quantize_store_regs(uint4 v0, uint4 v1, float g, uint32_t& sc, uint2& codes) {
  const uint32_t wv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
  float f[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    f[2 * i] = bf16lo_to_float(wv[i]);
    f[2 * i + 1] = bf16hi_to_float(wv[i]);
  }
  quantize_block(f, g, sc, codes);
}

}  // namespace
}  // namespace nvfp4

// nvfp4_device.cuh -- device-side helpers shared by the NVFP4 kernels:
// format conversions through the sm_100a cvt instructions and streaming loads.
//
// Format (web pages, by title and section): "Raphael Friedmann" home page,
// NVFP4 bit-level graphic (E2M1 elements, FP8 scale per 16, FP32 per tensor);
// imp docs/quantization.md, NVFP4 KV paragraph (the PTX cvt.rn.f16x2.e2m1x2
// conversion used to decode packed FP4 on Blackwell).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace nvfp4 {

// Two E2M1 codes (low nibble -> low half) to an f16x2 pair; exact, sign kept.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte_in_low8) {
  uint32_t out;
  asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}"
      : "=r"(out)
      : "r"(byte_in_low8));
  return out;
}

// Byte `i` (0..3) of a 32-bit word as two E2M1 codes -> f16x2.
template <int I>
__device__ __forceinline__ uint32_t e2m1x2_byte_to_f16x2(uint32_t word) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b" "%2" ";\n\t}"
      : "=r"(out)
      : "r"(word), "n"(I));
  return out;
}

// Two E4M3 bytes (low byte -> low half) to an f16x2 pair; exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_bytes) {
  uint32_t out;
  const uint16_t v = static_cast<uint16_t>(two_bytes);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(out) : "h"(v));
  return out;
}

__device__ __forceinline__ float2 f16x2_to_float2(uint32_t h2) {
  __half2 h = *reinterpret_cast<__half2*>(&h2);
  return __half22float2(h);
}

__device__ __forceinline__ float e4m3_to_float(uint32_t byte) {
  return f16x2_to_float2(e4m3x2_to_f16x2(byte & 0xFFu)).x;
}

// fp32 -> E4M3 byte, round to nearest even, saturating at +-448.
__device__ __forceinline__ uint32_t float_to_e4m3_satfinite(float v) {
  uint16_t out;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(0.0f), "f"(v));
  return out & 0xFFu;
}

// (lo, hi) fp32 -> one byte of two E2M1 codes (lo in the low nibble), round to
// nearest even, saturating at +-6.  The instruction places its first source in
// the high nibble.
__device__ __forceinline__ uint32_t float2_to_e2m1x2_satfinite(float lo, float hi) {
  uint32_t out;
  asm("{\n\t.reg .b8 b;\n\tcvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\tcvt.u32.u8 %0, b;\n\t}"
      : "=r"(out)
      : "f"(hi), "f"(lo));
  return out;
}

// BF16 bit patterns of a 32-bit word -> two fp32 (exact).
__device__ __forceinline__ float bf16lo_to_float(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi_to_float(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// 16-byte global load that bypasses L1 (weights are streamed once per call).
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint2 ld_stream_v2(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];"
               : "=r"(v.x), "=r"(v.y)
               : "l"(p));
  return v;
}

// c + lo(a)*lo(b) + hi(a)*hi(b) with a, b f16x2 pairs, in fp32: one
// mixed-precision fma.rn.f32.f16 per product (products exact).
__device__ __forceinline__ float fma2_f16_f32(uint32_t a2, uint32_t b2, float c) {
  float d;
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t.reg .f32 t;\n\t"
      "mov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.f16 t, al, bl, %3;\n\tfma.rn.f32.f16 %0, ah, bh, t;\n\t}"
      : "=f"(d)
      : "r"(a2), "r"(b2), "f"(c));
  return d;
}

// floor(log2(v)) of a non-zero, finite BF16 magnitude given by its 15 low bits.
__device__ __forceinline__ int bf16_ilogb(uint32_t a) {
  return a >= 0x80u ? (int)(a >> 7) - 127 : (31 - __clz((int)a)) - 133;
}

// 2^k as fp32 for k in [-126, 127].
__device__ __forceinline__ float exp2i(int k) { return __uint_as_float((uint32_t)(k + 127) << 23); }

}  // namespace nvfp4

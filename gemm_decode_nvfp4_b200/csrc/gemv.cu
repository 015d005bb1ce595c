// gemv.cu -- batch-1 decode GEMV over packed NVFP4 weights (W4A16).
//
// The decode path of imp docs/quantization.md ("Dense layers" pipeline: an
// NVFP4 GEMV reading the packed nibbles, E4M3 micro-scales and FP32 tensor
// scale directly) with BF16 activations (model card "Qwen3.8-27B-NVFP4",
// "What is quantized": weight-only).  The pages' kernel targets sm_120 with a
// prmt register LUT; on sm_100a the weight decode is one
// cvt.rn.f16x2.e2m1x2 per two codes (exact, sign included) and each product
// is one mixed-precision fma.rn.f32.f16 (f16 x f16 -> fp32 accumulator),
// which issues at the full FFMA rate.
//
// x is staged once per CTA in shared memory.  For the f16 operand it is
// scaled by a power of two 2^e chosen from max|x| so that every element is
// exactly representable in f16 (BF16 has 8 significant bits, f16 11): this
// holds when all non-zero |x| lie within 2^32 of max|x| and x is finite, which
// the CTA checks while staging.  Otherwise the CTA takes the exact fp32 path
// (x in fp32, codes -> f16 -> fp32, packed fp32x2 FMAs).  Either way every
// product is exact and the accumulation is fp32; the result is
// y = bf16_rn(2^-e * (g * acc)).
//
// Work split: a warp owns R = 8 consecutive rows; lane l reads the 16-byte
// chunks l, l+32, ... of each row (512 contiguous bytes per warp-load, one
// 16-bit scale load per chunk).  Two register buffers alternate (the step
// loop is unrolled by two, so no buffer is copied): the next step's 8 x 16
// bytes per lane are in flight while the current step is computed.  Launched
// with programmatic dependent launch; with static weights the first loads are
// issued before the previous kernel has finished.  The weight stream (0.5625
// B/weight) is the roofline: HBM bandwidth.
#include "nvfp4_kernels.h"
#include "nvfp4_device.cuh"

namespace nvfp4 {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;




// Exact fp32 path for x outside the f16 window (not finite, or non-zero
// magnitudes spanning more than 2^32): rows row0 .. row0 + nrows - 1, one warp,
// x read as BF16 from global memory.  Kept out of line so that the common
// path's register allocation does not carry it.
__device__ __noinline__ void gemv_rows_exact(const uint16_t* __restrict__ x, const uint8_t* __restrict__ q,
                                             const uint8_t* __restrict__ s, float gv, uint16_t* __restrict__ y,
                                             int N, int K, int row0, int nrows) {
  const int lane = threadIdx.x & 31;
  for (int r = 0; r < nrows; ++r) {
    const int row = row0 + r;
    if (row >= N) break;
    const uint8_t* qr = q + (int64_t)row * (K / 2);
    const uint8_t* sr = s + (int64_t)row * (K / 16);
    float acc = 0.0f;
    for (int b = lane; b < K / 16; b += 32) {  // 16-element blocks
      const uint2 w = *reinterpret_cast<const uint2*>(qr + 8 * b);
      const uint4 xa = *reinterpret_cast<const uint4*>(x + 16 * b);
      const uint4 xb = *reinterpret_cast<const uint4*>(x + 16 * b + 8);
      const uint32_t wd[2] = {w.x, w.y};
      const uint32_t xw[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
      float2 p = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        p = __ffma2_rn(f16x2_to_float2(e2m1x2_byte_to_f16x2<0>(wd[i])),
                       make_float2(bf16lo_to_float(xw[4 * i]), bf16hi_to_float(xw[4 * i])), p);
        p = __ffma2_rn(f16x2_to_float2(e2m1x2_byte_to_f16x2<1>(wd[i])),
                       make_float2(bf16lo_to_float(xw[4 * i + 1]), bf16hi_to_float(xw[4 * i + 1])), p);
        p = __ffma2_rn(f16x2_to_float2(e2m1x2_byte_to_f16x2<2>(wd[i])),
                       make_float2(bf16lo_to_float(xw[4 * i + 2]), bf16hi_to_float(xw[4 * i + 2])), p);
        p = __ffma2_rn(f16x2_to_float2(e2m1x2_byte_to_f16x2<3>(wd[i])),
                       make_float2(bf16lo_to_float(xw[4 * i + 3]), bf16hi_to_float(xw[4 * i + 3])), p);
      }
      acc = fmaf(p.x + p.y, e4m3_to_float(sr[b]), acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
    if (lane == 0) {
      const __nv_bfloat16 o = __float2bfloat16_rn(acc * gv);
      y[row] = *reinterpret_cast<const uint16_t*>(&o);
    }
  }
}

template <int R, int CB, int MINB>
__global__ void __launch_bounds__(kThreads, MINB) gemv_kernel(const uint16_t* __restrict__ x,
                                                              const uint8_t* __restrict__ q,
                                                              const uint8_t* __restrict__ s,
                                                              const float* __restrict__ g,
                                                              uint16_t* __restrict__ y, int N, int K,
                                                              int static_weights) {
  extern __shared__ __align__(16) uint8_t xsm[];  // K f16
  __shared__ uint32_t red_max[kWarps], red_min[kWarps];
  constexpr int kBlocks = (2 * CB) / 16;  // scales per lane-chunk (2 or 1)
  constexpr int kWords = CB / 4;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = (blockIdx.x * kWarps + warp) * R;
  const int row_bytes = K >> 1;
  const int row_scales = K >> 4;
  const int steps = (row_bytes + 32 * CB - 1) / (32 * CB);

  auto load = [&](int step, uint32_t (&wq)[R][kWords], uint32_t (&ws)[R]) {
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
        for (int i = 0; i < kWords; ++i) wq[r][i] = 0;
        ws[r] = 0;
      }
    }
  };

  // Programmatic dependent launch: let the next kernel on the stream start
  // its prologue; read the weights before the previous kernel has finished
  // only when the caller declared them static, x and y only after it has.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (!static_weights) asm volatile("griddepcontrol.wait;" ::: "memory");
  uint32_t wq[R][kWords], ws[R];
  load(0, wq, ws);  // first weights in flight before x is staged
  if (static_weights) asm volatile("griddepcontrol.wait;" ::: "memory");

  // ---- range of |x| (bit patterns of non-negative BF16 order like values)
  uint32_t mx = 0, mn = 0xFFFFu;
  // (the raw BF16 vectors go to shared memory on the way; each thread later
  // converts the vectors it wrote, so x is read from global memory once)
  for (int i = threadIdx.x; i < (K >> 3); i += kThreads) {
    const uint4 v = *reinterpret_cast<const uint4*>(x + 8 * i);
    reinterpret_cast<uint4*>(xsm)[i] = v;
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t lo = w4[j] & 0x7FFFu, hi = (w4[j] >> 16) & 0x7FFFu;
      mx = max(mx, max(lo, hi));
      mn = min(mn, min(lo ? lo : 0xFFFFu, hi ? hi : 0xFFFFu));
    }
  }
  mx = __reduce_max_sync(0xFFFFFFFFu, mx);
  mn = __reduce_min_sync(0xFFFFFFFFu, mn);
  if (lane == 0) { red_max[warp] = mx; red_min[warp] = mn; }
  __syncthreads();
  mx = red_max[0]; mn = red_min[0];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) { mx = max(mx, red_max[w]); mn = min(mn, red_min[w]); }
  bool fast = true;
  int e = 0;
  if (mx >= 0x7F80u) {
    fast = false;                       // inf or NaN in x
  } else if (mx != 0) {
    const int hi_exp = bf16_ilogb(mx), lo_exp = bf16_ilogb(mn);
    e = 15 - hi_exp;                    // max |x| * 2^e in [2^15, 2^16)
    fast = hi_exp - lo_exp <= 32;       // smallest non-zero |x| * 2^e >= 2^-17
  }

  if (!fast) {  // x outside the f16 window: every warp takes its rows exactly
    gemv_rows_exact(x, q, s, *g, y, N, K, row0, R);
    return;
  }

  // ---- stage x (f16, scaled by 2^e)
  {
    const int e1 = e / 2, e2 = e - e1;  // two exact power-of-two steps
    const float m1 = exp2i(e1), m2 = exp2i(e2);
    for (int i = threadIdx.x; i < (K >> 3); i += kThreads) {
      const uint4 v = reinterpret_cast<const uint4*>(xsm)[i];  // written by this thread above
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __half2 h = __floats2half2_rn(bf16lo_to_float(w4[j]) * m1 * m2, bf16hi_to_float(w4[j]) * m1 * m2);
        o[j] = *reinterpret_cast<const uint32_t*>(&h);
      }
      reinterpret_cast<uint4*>(xsm)[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  __syncthreads();

  float acc[R];
#pragma unroll
  for (int r = 0; r < R; ++r) acc[r] = 0.0f;

  // One step of the dot products on the register buffer (cq, cs).
  auto compute = [&](int step, const uint32_t (&cq)[R][kWords], const uint32_t (&cs)[R]) {
    const int off = step * 32 * CB + lane * CB;
    if (off >= row_bytes) return;
    float part[R][kBlocks];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int b = 0; b < kBlocks; ++b) part[r][b] = 0.0f;
    const uint4* xp = reinterpret_cast<const uint4*>(xsm) + (2 * off) / 8;
#pragma unroll
    for (int wi = 0; wi < kWords; ++wi) {  // 8 weights per 32-bit word
      const uint4 xv = xp[wi];
      const int b = wi / 2;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const uint32_t word = cq[r][wi];
        float p = part[r][b];
        p = fma2_f16_f32(e2m1x2_byte_to_f16x2<0>(word), xv.x, p);
        p = fma2_f16_f32(e2m1x2_byte_to_f16x2<1>(word), xv.y, p);
        p = fma2_f16_f32(e2m1x2_byte_to_f16x2<2>(word), xv.z, p);
        p = fma2_f16_f32(e2m1x2_byte_to_f16x2<3>(word), xv.w, p);
        part[r][b] = p;
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float2 sc = f16x2_to_float2(e4m3x2_to_f16x2(cs[r]));
      acc[r] = fmaf(part[r][0], sc.x, acc[r]);
      if constexpr (kBlocks == 2) acc[r] = fmaf(part[r][1], sc.y, acc[r]);
    }
  };
  // Two register buffers in turn (the loop is unrolled by two so that no
  // buffer is ever copied): the next step's weights are always in flight
  // while the current step is computed.
  uint32_t bq[R][kWords], bs[R];
  int step = 0;
  for (; step + 1 < steps; step += 2) {
    load(step + 1, bq, bs);
    compute(step, wq, ws);
    if (step + 2 < steps) load(step + 2, wq, ws);
    compute(step + 1, bq, bs);
  }
  if (step < steps) compute(step, wq, ws);

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
      const float out = ldexpf(v * gv, -e);
      const __nv_bfloat16 o = __float2bfloat16_rn(out);
      y[row] = *reinterpret_cast<const uint16_t*>(&o);
    }
  }
}

template <int R, int CB, int MINB>
cudaError_t launch(const uint16_t* x, const uint8_t* q, const uint8_t* s, const float* g, uint16_t* y, int N,
                   int K, bool static_weights, cudaStream_t stream) {
  const size_t smem = (size_t)K * sizeof(uint16_t);
  auto kern = gemv_kernel<R, CB, MINB>;
  static int smem_set[64] = {};  // per device: largest dynamic shared memory enabled so far
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || smem_set[dev] < (int)smem) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) smem_set[dev] = (int)smem;
  }
  const int rows_per_cta = kWarps * R;
  const int grid = (N + rows_per_cta - 1) / rows_per_cta;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, x, q, s, g, y, N, K, static_weights ? 1 : 0);
}

}  // namespace

cudaError_t launch_gemv(const uint16_t* x, const uint8_t* q, const uint8_t* s, const float* g,
                        uint16_t* y, int64_t N, int64_t K, int sms, bool static_weights, cudaStream_t stream) {
  (void)sms;
  if (K % 32 == 0) return launch<8, 16, 2>(x, q, s, g, y, (int)N, (int)K, static_weights, stream);
  return launch<8, 8, 2>(x, q, s, g, y, (int)N, (int)K, static_weights, stream);
}

}  // namespace nvfp4

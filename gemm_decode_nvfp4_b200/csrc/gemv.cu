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
// y = bf16_rn(2^-e * (g * acc)).  The weight stream (0.5625 B/weight) is the
// roofline: HBM bandwidth.
//
// Two kernels:
//
// * Ring kernel (K a multiple of 256): CTAs of half an SM's registers and
//   shared memory, so that the next kernel on the stream can be resident
//   beside them.  K may be split over the C in {1, 2, 4, 8} CTAs of a thread-
//   block cluster ("K-parallel"; each CTA holds at most 11520 elements of x):
//   each cluster owns a contiguous range of about N / (#SMs / C) rows and rank
//   r takes its share of the 512-element columns of K.  A producer thread
//   streams the CTA's range through a ring of shared-memory stages with 2-D
//   TMA copies (up to 120 rows x 256 code bytes + their scales per stage;
//   rows past the end read as zero); 15 consumer warps own up to 4 rows x one
//   16-byte chunk per lane, release a stage as soon as its bytes are in
//   registers, and reduce each row over its 16 lanes once.  With C > 1 the
//   CTAs leave fp32 partials in shared memory and the cluster adds them in
//   rank order through distributed shared memory.  After the previous kernel
//   has finished, x arrives first (one bulk copy), then the ring, so x is
//   never queued behind weight traffic.  The next kernel on the stream may
//   start (programmatic dependent launch) once every CTA of this one has
//   issued its last stage; its CTAs then wait in the other half of each SM
//   while this kernel drains.  The static-weights flag does not change this
//   kernel: weight requests issued before x, into shared memory or into L2,
//   by it or by the kernel after it, were measured to delay x and the first
//   stages more than they saved.  One unsplit problem with full row blocks
//   (90-120 rows) runs a specialised copy with a fixed stage layout and four
//   consecutive rows per lane, which was measured faster on those shapes; it
//   requests its first stage before the dependency wait when the weights are
//   static (one stage gained, more lost).
//
// * Register kernel (every other K): a warp owns R = 8 consecutive rows; lane l
//   reads the 16-byte chunks l, l+32, ... of each row into two register buffers
//   that alternate, the next step's loads in flight while the current step is
//   computed.
#include "nvfp4_kernels.h"
#include "nvfp4_device.cuh"
#include "sm100_ptx.cuh"
#include "tc_host.h"

#include <algorithm>

namespace nvfp4 {

// CTAs of the ring kernel whose bounded pipeline wait gave up since the last read.
__device__ unsigned int g_gemv_wait_timeouts = 0;
// Grouped calls: problems whose expert or token id was out of range (their
// output rows are written as zeros).
__device__ unsigned int g_gemv_bad_ids = 0;

namespace {

// The problems of one launch: with expert_ids == nullptr a single GEMV (expert
// 0, token 0); otherwise problem p = blockIdx.y multiplies expert
// expert_ids[p] of the stacked [E, N, K/2] weights (and its tensor scale
// g[e]) by row token_ids[p] of X into row p of Y (grouped MoE decode).
struct Problems {
  const int* expert_ids;
  const int* token_ids;
  int E, T;
  int64_t x_stride, y_stride;  // elements between rows of X / of Y
};

// This CTA's expert and token; read only after griddepcontrol.wait (the ids
// may come from the previous kernel).  False when an id is out of range.
template <bool GROUPED>
__device__ __forceinline__ bool resolve_problem(const Problems& P, int& e, int& tok) {
  if (!GROUPED || P.expert_ids == nullptr) {
    e = 0;
    tok = 0;
    return true;
  }
  e = P.expert_ids[blockIdx.y];
  tok = P.token_ids[blockIdx.y];
  return e >= 0 && e < P.E && tok >= 0 && tok < P.T;
}

// Rows row0 .. row0 + nrows - 1 of an invalid problem become zeros (lane
// first_thread, then every 32nd row); the problem is counted once, by thread 0
// of its first CTA.
__device__ __forceinline__ void zero_rows(uint16_t* y, int N, int row0, int nrows, int first_thread) {
  for (int r = first_thread; r < nrows; r += 32)
    if (row0 + r < N) y[row0 + r] = 0;
}

__device__ __forceinline__ void count_bad_problem() {
  if (blockIdx.x == 0 && threadIdx.x == 0) atomicAdd(&g_gemv_bad_ids, 1u);
}

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

// UE8M0 micro-scale (MXFP4) -> fp32: 2^(b - 127); 0 is the subnormal 2^-127,
// 255 is NaN.
__device__ __forceinline__ float e8m0_to_float(uint32_t b) {
  return __uint_as_float(b == 0u ? 0x00400000u : (b == 255u ? 0x7FFFFFFFu : b << 23));
}

// MXFP4 counterpart of gemv_rows_exact: 32-element blocks with a UE8M0 scale,
// no tensor scale.
__device__ __noinline__ void gemv_rows_exact_mx(const uint16_t* __restrict__ x, const uint8_t* __restrict__ q,
                                                const uint8_t* __restrict__ s, uint16_t* __restrict__ y, int N,
                                                int K, int row0, int nrows) {
  const int lane = threadIdx.x & 31;
  for (int r = 0; r < nrows; ++r) {
    const int row = row0 + r;
    if (row >= N) break;
    const uint8_t* qr = q + (int64_t)row * (K / 2);
    const uint8_t* sr = s + (int64_t)row * (K / 32);
    float acc = 0.0f;
    for (int b = lane; b < K / 32; b += 32) {  // 32-element blocks
      const uint4 w = *reinterpret_cast<const uint4*>(qr + 16 * b);
      const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
      float2 p = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 xa = *reinterpret_cast<const uint4*>(x + 32 * b + 8 * i);
        const uint32_t xw[4] = {xa.x, xa.y, xa.z, xa.w};
        p = __ffma2_rn(f16x2_to_float2(e2m1x2_byte_to_f16x2<0>(wd[i])), make_float2(bf16lo_to_float(xw[0]), bf16hi_to_float(xw[0])), p);
        p = __ffma2_rn(f16x2_to_float2(e2m1x2_byte_to_f16x2<1>(wd[i])), make_float2(bf16lo_to_float(xw[1]), bf16hi_to_float(xw[1])), p);
        p = __ffma2_rn(f16x2_to_float2(e2m1x2_byte_to_f16x2<2>(wd[i])), make_float2(bf16lo_to_float(xw[2]), bf16hi_to_float(xw[2])), p);
        p = __ffma2_rn(f16x2_to_float2(e2m1x2_byte_to_f16x2<3>(wd[i])), make_float2(bf16lo_to_float(xw[3]), bf16hi_to_float(xw[3])), p);
      }
      acc = fmaf(p.x + p.y, e8m0_to_float(sr[b]), acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
    if (lane == 0) {
      const __nv_bfloat16 o = __float2bfloat16_rn(acc);
      y[row] = *reinterpret_cast<const uint16_t*>(&o);
    }
  }
}

// Rows row0 .. row0 + nrows - 1 exactly, in either format.
template <bool MX>
__device__ __forceinline__ void rows_exact(const uint16_t* x, const uint8_t* q, const uint8_t* s, const float* g,
                                           uint16_t* y, int N, int K, int row0, int nrows) {
  if constexpr (MX)
    gemv_rows_exact_mx(x, q, s, y, N, K, row0, nrows);
  else
    gemv_rows_exact(x, q, s, *g, y, N, K, row0, nrows);
}

template <int R, int CB, int MINB, bool MX, bool GROUPED>
__global__ void __launch_bounds__(kThreads, MINB) gemv_kernel(const uint16_t* __restrict__ x,
                                                              const uint8_t* __restrict__ q,
                                                              const uint8_t* __restrict__ s,
                                                              const float* __restrict__ g,
                                                              uint16_t* __restrict__ y, int N, int K,
                                                              int static_weights, Problems P) {
  extern __shared__ __align__(16) uint8_t xsm[];  // K f16
  __shared__ uint32_t red_max[kWarps], red_min[kWarps];
  constexpr int kBlocks = (2 * CB) / 16;  // scales per lane-chunk (2 or 1)
  constexpr int kWords = CB / 4;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = (blockIdx.x * kWarps + warp) * R;
  static_assert(!MX || CB == 16, "MXFP4: one 32-element block per 16-byte chunk");
  const int row_bytes = K >> 1;
  const int row_scales = MX ? K >> 5 : K >> 4;
  const int steps = (row_bytes + 32 * CB - 1) / (32 * CB);

  auto load = [&](int step, uint32_t (&wq)[R][kWords], uint32_t (&ws)[R]) {
    const int off = step * 32 * CB + lane * CB;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int row = row0 + r;
      if (row < N && off < row_bytes) {
        const uint8_t* pq = q + (int64_t)row * row_bytes + off;
        const uint8_t* ps = s + (int64_t)row * row_scales + (MX ? off / 16 : off / 8);
        if constexpr (CB == 16) {
          const uint4 v = ld_stream_v4(pq);
          wq[r][0] = v.x; wq[r][1] = v.y; wq[r][2] = v.z; wq[r][3] = v.w;
          ws[r] = MX ? (uint32_t)*ps : (uint32_t)*reinterpret_cast<const uint16_t*>(ps);
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
  // grouped calls learn their expert only after the previous kernel
  const bool early = static_weights && !GROUPED;
  if (!early) asm volatile("griddepcontrol.wait;" ::: "memory");
  int e_id = 0, tok = 0;
  if (!resolve_problem<GROUPED>(P, e_id, tok)) {  // the warp's rows of this problem become zeros
    zero_rows(y + (int64_t)blockIdx.y * P.y_stride, N, row0, R, lane);
    count_bad_problem();
    return;
  }
  q += (int64_t)e_id * N * (K / 2);
  s += (int64_t)e_id * N * (MX ? K / 32 : K / 16);
  if (!MX) g += e_id;
  x += (int64_t)tok * P.x_stride;
  y += (int64_t)blockIdx.y * P.y_stride;
  uint32_t wq[R][kWords], ws[R];
  load(0, wq, ws);  // first weights in flight before x is staged
  if (early) asm volatile("griddepcontrol.wait;" ::: "memory");

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
    rows_exact<MX>(x, q, s, g, y, N, K, row0, R);
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
      if constexpr (MX) {
        acc[r] = fmaf(part[r][0] + part[r][1], e8m0_to_float(cs[r]), acc[r]);
      } else {
        const float2 sc = f16x2_to_float2(e4m3x2_to_f16x2(cs[r]));
        acc[r] = fmaf(part[r][0], sc.x, acc[r]);
        if constexpr (kBlocks == 2) acc[r] = fmaf(part[r][1], sc.y, acc[r]);
      }
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

  const float gv = MX ? 1.0f : *g;
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

template <int R, int CB, int MINB, bool MX, bool GROUPED>
cudaError_t launch(const uint16_t* x, const uint8_t* q, const uint8_t* s, const float* g, uint16_t* y, int N,
                   int K, bool static_weights, cudaStream_t stream, const Problems& P, int num_problems) {
  const size_t smem = (size_t)K * sizeof(uint16_t);
  auto kern = gemv_kernel<R, CB, MINB, MX, GROUPED>;
  static tc::SmemOptIn opt_in;
  const cudaError_t e = opt_in.ensure((const void*)kern, (int)smem);
  if (e != cudaSuccess) return e;
  const int rows_per_cta = kWarps * R;
  const int grid = (N + rows_per_cta - 1) / rows_per_cta;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, num_problems);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, x, q, s, g, y, N, K, static_weights ? 1 : 0, P);
}


// ------------------------------------------------------------------------------------------ ring kernel

constexpr int kRingConsumerWarps = 15;                    // warp 15 is the producer
constexpr int kRingConsumers = kRingConsumerWarps * 32;   // 480 threads
constexpr int kRingThreads = kRingConsumers + 32;         // 512 threads x 64 registers: half an SM
constexpr int kRingBK = 256;                              // code bytes of a row per stage (512 weights)
constexpr int kRingChunks = kRingBK / 16;                 // 16 lanes share a row
constexpr int kRingSlots = kRingConsumers / kRingChunks;  // 30 row slots: a lane owns rows slot + 30 i
constexpr int kRingRows = 4;                              // rows per lane at most
constexpr int kRingMaxBR = kRingSlots * kRingRows;        // 120 rows per stage
constexpr int kRingMaxSlice = kRingConsumers * 24;        // x elements per CTA: at most 3 uint4 per consumer
constexpr int kRingMaxStages = 8;
constexpr int64_t kRingMinInFlight = 64 * 1024;  // ring bytes below which a split of 2 is preferred
constexpr uint64_t kRingWaitNs = 2000000000ull;

__device__ __forceinline__ void ring_sync(int n) { asm volatile("bar.sync 1, %0;" ::"r"(n) : "memory"); }

__device__ __forceinline__ void tma_load_3d_evict_first(void* dst, const void* tmap, uint64_t* bar, int c0, int c1,
                                                        int c2, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(ptx::smem_u32(dst)),
      "l"(tmap), "r"(ptx::smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
      : "memory");
}

// Exact fp32 dot product of weight row `row` with x over k in [k0, k1) (block
// boundaries), one warp, x read as BF16 from global memory: the path for x
// outside the f16 window.  Every lane returns the sum.
template <bool MX>
__device__ __noinline__ float dot_exact_range(const uint16_t* __restrict__ x, const uint8_t* __restrict__ q,
                                              const uint8_t* __restrict__ s, int K, int row, int k0, int k1) {
  constexpr int BS = MX ? 32 : 16;  // elements per scale
  const int lane = threadIdx.x & 31;
  const uint8_t* qr = q + (int64_t)row * (K / 2);
  const uint8_t* sr = s + (int64_t)row * (K / BS);
  float acc = 0.0f;
  for (int b = k0 / BS + lane; b < k1 / BS; b += 32) {
    float2 p = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int i = 0; i < BS / 8; ++i) {  // 8 weights (4 code bytes) at a time
      const uint32_t wd = *reinterpret_cast<const uint32_t*>(qr + (BS / 2) * b + 4 * i);
      const uint4 xa = *reinterpret_cast<const uint4*>(x + BS * b + 8 * i);
      p = __ffma2_rn(f16x2_to_float2(e2m1x2_byte_to_f16x2<0>(wd)), make_float2(bf16lo_to_float(xa.x), bf16hi_to_float(xa.x)), p);
      p = __ffma2_rn(f16x2_to_float2(e2m1x2_byte_to_f16x2<1>(wd)), make_float2(bf16lo_to_float(xa.y), bf16hi_to_float(xa.y)), p);
      p = __ffma2_rn(f16x2_to_float2(e2m1x2_byte_to_f16x2<2>(wd)), make_float2(bf16lo_to_float(xa.z), bf16hi_to_float(xa.z)), p);
      p = __ffma2_rn(f16x2_to_float2(e2m1x2_byte_to_f16x2<3>(wd)), make_float2(bf16lo_to_float(xa.w), bf16hi_to_float(xa.w)), p);
    }
    acc = fmaf(p.x + p.y, MX ? e8m0_to_float(sr[b]) : e4m3_to_float(sr[b]), acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
  return acc;
}

// The consumer loop of one warp of the ring kernel: NR rows per lane (a
// compile-time count, so that the loads, the decode and the FMAs of a stage
// are straight-line code), rows slot0 + 30 i of each stage, 16-byte chunk c.
// A warp with NR == 0 only keeps the ring's phases (waits and releases each
// stage).  emit(rb, local_row, value) receives each row's dot product times
// g * 2^-e.  Returns false when a bounded wait gave up.
template <bool MX, int NR, typename Emit>
__device__ __forceinline__ bool ring_rows(const uint8_t* lane_codes, const uint8_t* lane_scales, const uint4* lane_x,
                                          uint64_t* full, uint64_t* empty, int S, int SB, int nb_here, int ncols,
                                          int c, int slot0, int BR, float scale, int e, Emit&& emit) {
  constexpr int kSB = MX ? kRingBK / 16 : kRingBK / 8;
  constexpr int R = NR > 0 ? NR : 1;
  const int lane = threadIdx.x & 31;
  int sl = 0;
  uint32_t phase = 0;
  for (int rb = 0; rb < nb_here; ++rb) {
    float acc[R];
#pragma unroll
    for (int i = 0; i < R; ++i) acc[i] = 0.0f;
    for (int t = 0; t < ncols; ++t) {
      if (!__all_sync(0xFFFFFFFFu, ptx::mbar_wait(&full[sl], phase, kRingWaitNs))) return false;
      uint4 cw[R];
      uint32_t sc[R];
      if constexpr (NR > 0) {
        const uint8_t* pc = lane_codes + sl * SB;
        const uint8_t* ps = lane_scales + sl * SB;
#pragma unroll
        for (int i = 0; i < NR; ++i) {  // (the odd slot of the last i may be row BR: stale bytes, never stored)
          cw[i] = *reinterpret_cast<const uint4*>(pc + i * kRingSlots * kRingBK);
          sc[i] = MX ? (uint32_t)ps[i * kRingSlots * kSB]
                     : (uint32_t)*reinterpret_cast<const uint16_t*>(ps + i * kRingSlots * kSB);
        }
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&empty[sl]);  // the stage's bytes are in registers
      if (++sl == S) { sl = 0; phase ^= 1; }
      if constexpr (NR > 0) {
        const uint4* xp = lane_x + t * 64;
        float pt[NR][2];
#pragma unroll
        for (int i = 0; i < NR; ++i) pt[i][0] = pt[i][1] = 0.0f;
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {  // 8 weights per 32-bit word; words 0-1 block 0, words 2-3 block 1
          const uint4 xv = xp[wi * 16];
#pragma unroll
          for (int i = 0; i < NR; ++i) {
            const uint32_t word = wi == 0 ? cw[i].x : wi == 1 ? cw[i].y : wi == 2 ? cw[i].z : cw[i].w;
            float p = pt[i][wi >> 1];
            p = fma2_f16_f32(e2m1x2_byte_to_f16x2<0>(word), xv.x, p);
            p = fma2_f16_f32(e2m1x2_byte_to_f16x2<1>(word), xv.y, p);
            p = fma2_f16_f32(e2m1x2_byte_to_f16x2<2>(word), xv.z, p);
            p = fma2_f16_f32(e2m1x2_byte_to_f16x2<3>(word), xv.w, p);
            pt[i][wi >> 1] = p;
          }
        }
#pragma unroll
        for (int i = 0; i < NR; ++i) {
          if constexpr (MX) {  // one 32-element block per chunk
            acc[i] = fmaf(pt[i][0] + pt[i][1], e8m0_to_float(sc[i]), acc[i]);
          } else {
            const float2 sf = f16x2_to_float2(e4m3x2_to_f16x2(sc[i]));
            acc[i] = fmaf(pt[i][0], sf.x, acc[i]);
            acc[i] = fmaf(pt[i][1], sf.y, acc[i]);
          }
        }
      }
    }
    if constexpr (NR > 0) {
#pragma unroll
      for (int i = 0; i < NR; ++i) {
        float v = acc[i];
#pragma unroll
        for (int o = kRingChunks / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
        acc[i] = v;
      }
      if (c < NR) {
        float v = acc[0];
#pragma unroll
        for (int i = 1; i < NR; ++i)
          if (c == i) v = acc[i];
        const int rl = slot0 + kRingSlots * c;
        if (rl < BR) emit(rb, rl, ldexpf(v * scale, -e));
      }
    }
  }
  return true;
}

// Shared memory: S stages of SB bytes (a stage: BR rows x 256 code bytes, then
// their BR x 32 (NVFP4) or 16 (MXFP4) scale bytes), then x (ncx x 1 KB: f16,
// each stage column's 512 values laid out [word i][chunk c] so that a
// quarter-warp reads 128 contiguous bytes), then the barriers, the reduction
// scratch and (K split over a cluster) the fp32 partial of each row.
// Rows of a CTA: [cl * nblk * BR, + nblk * BR) for cluster cl = blockIdx.x / C,
// in nblk blocks of BR rows (BR <= 120) that go through the ring one 256-byte
// column at a time.  K: the nks = ceil(K / 512) columns are split over the C
// CTAs of a cluster (rank r takes columns [r nks / C, (r + 1) nks / C)); with
// C > 1 each CTA leaves its rows' partial sums in shared memory and the
// cluster adds them in rank order (fixed order: deterministic).
template <bool MX, bool GROUPED>
__global__ void __launch_bounds__(kRingThreads, 2)
    gemv_ring_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap ts,
                     const uint16_t* __restrict__ x, const uint8_t* __restrict__ q, const uint8_t* __restrict__ s,
                     const float* __restrict__ g, uint16_t* __restrict__ y, int N, int K, int BR, int nblk,
                     int S, int SB, int C, Problems P) {
  extern __shared__ __align__(1024) uint8_t sm[];
  constexpr int kSB = MX ? kRingBK / 16 : kRingBK / 8;  // scale bytes of a row per stage
  const int nks = (K / 2 + kRingBK - 1) / kRingBK;      // stage columns of a row
  const int ncx = (nks + C - 1) / C;                    // most columns a CTA takes
  const int rank = C > 1 ? (int)ptx::cluster_ctarank() : 0;
  const int t0 = (int)((int64_t)rank * nks / C), t1 = (int)((int64_t)(rank + 1) * nks / C);
  const int ncols = t1 - t0;
  const int k0 = t0 * 2 * kRingBK, k1 = min(t1 * 2 * kRingBK, K);  // this CTA's x elements
  uint8_t* ring = sm;
  uint4* xs = reinterpret_cast<uint4*>(sm + S * SB);
  uint64_t* full = reinterpret_cast<uint64_t*>(xs + ncx * 64);
  uint64_t* empty = full + S;
  uint64_t* xfull = empty + S;
  uint32_t* red = reinterpret_cast<uint32_t*>(xfull + 1);        // [2][16], then two flags
  volatile int* abort_flag = reinterpret_cast<volatile int*>(red + 32);
  float* part = reinterpret_cast<float*>(red + 36);               // [nblk * BR], used when C > 1

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row_base = (blockIdx.x / C) * nblk * BR;
  const int nb_here = min(nblk, (N - row_base + BR - 1) / BR);
  const int total = nb_here * ncols;

  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], kRingConsumerWarps);
    }
    ptx::mbar_init(xfull, 1);
    *abort_flag = 0;
    red[33] = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();

  if (warp == kRingConsumerWarps) {  // ------------------------------------------------- producer
    if (lane != 0) return;
    ptx::prefetch_tmap(&tq);
    ptx::prefetch_tmap(&ts);
    uint64_t policy;  // each weight byte is read once: do not keep it in L2
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(policy));
    int n = 0, slot = 0, t = 0, rb = 0, e_id = 0;
    uint32_t phase = 0;
    auto issue = [&]() {
      uint8_t* dst = ring + slot * SB;
      const int row0 = row_base + rb * BR;
      ptx::mbar_arrive_expect_tx(&full[slot], (uint32_t)BR * (kRingBK + kSB));
      tma_load_3d_evict_first(dst, &tq, &full[slot], (t0 + t) * kRingBK, row0, e_id, policy);
      tma_load_3d_evict_first(dst + BR * kRingBK, &ts, &full[slot], (t0 + t) * kSB, row0, e_id, policy);
      if (++slot == S) { slot = 0; phase ^= 1; }
      if (++t == ncols) { t = 0; ++rb; }
    };
    asm volatile("griddepcontrol.wait;" ::: "memory");  // x, ids and the weights only after this
    int tok = 0;
    if (!resolve_problem<GROUPED>(P, e_id, tok)) return;  // nothing issued: the consumers write zeros
    ptx::mbar_arrive_expect_tx(xfull, (uint32_t)(k1 - k0) * 2);
    ptx::bulk_load(xs, x + (int64_t)tok * P.x_stride + k0, (uint32_t)(k1 - k0) * 2, xfull);
    for (; n < total; ++n) {
      if (n >= S) {  // wait until the consumers have released this slot (or have given up on the ring)
        bool ok = ptx::mbar_try_wait(&empty[slot], phase ^ 1);
        const uint64_t tw = ok ? 0 : ptx::globaltimer_ns();
        while (!ok && !*abort_flag) {
          if (ptx::globaltimer_ns() - tw > kRingWaitNs) {
            atomicAdd(&g_gemv_wait_timeouts, 1u);
            break;
          }
          ok = ptx::mbar_try_wait(&empty[slot], phase ^ 1);
        }
        if (!ok) break;
      }
      if (*abort_flag) break;
      issue();
      if (n == total - 3) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // two stages left
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // short rings and early exits
    // nothing may still be landing in shared memory when the CTA exits
    for (int m = max(0, n - S); m < n; ++m) ptx::mbar_wait(&full[m % S], (m / S) & 1, kRingWaitNs);
    ptx::mbar_wait(xfull, 0, kRingWaitNs);
    return;
  }

  // ------------------------------------------------------------------------------- consumers
  asm volatile("griddepcontrol.wait;" ::: "memory");  // y is written only after the previous kernel
  {
    int e_id = 0, tok = 0;
    if (!resolve_problem<GROUPED>(P, e_id, tok)) {  // this CTA's rows of the problem become zeros
      if (warp == 0)
        for (int b = 0; b < nb_here; ++b) zero_rows(y + (int64_t)blockIdx.y * P.y_stride, N, row_base + b * BR, BR, lane);
      count_bad_problem();
      return;
    }
    q += (int64_t)e_id * N * (K / 2);
    s += (int64_t)e_id * N * (MX ? K / 32 : K / 16);
    if (!MX) g += e_id;
    x += (int64_t)tok * P.x_stride;
    y += (int64_t)blockIdx.y * P.y_stride;
  }
  const float gv = MX ? 1.0f : *g;
  // Row (block rb, local row rl) gets its value: stored (C == 1) or left as a
  // partial for the cluster.
  auto emit = [&](int rb, int rl, float v) {
    const int row = row_base + rb * BR + rl;
    if (C > 1) {
      part[rb * BR + rl] = v;
    } else if (row < N) {
      const __nv_bfloat16 o = __float2bfloat16_rn(v);
      y[row] = *reinterpret_cast<const uint16_t*>(&o);
    }
  };
  // x: a warp whose bounded wait gave up marks the CTA failed; every consumer
  // thread then learns it at the barrier below (no warp leaves before it, so
  // the barrier always completes)
  volatile int* x_failed = reinterpret_cast<volatile int*>(red + 33);
  if (!__all_sync(0xFFFFFFFFu, ptx::mbar_wait(xfull, 0, kRingWaitNs))) {
    if (lane == 0) {
      atomicAdd(&g_gemv_wait_timeouts, 1u);
      *x_failed = 1;
    }
    *abort_flag = 1;
  }
  bool failed;  // a bounded wait gave up: the partials are NaN, nothing else runs
  int e = 0;
  bool fast = true;
  const int nx = (k1 - k0) >> 3;  // x vectors of this CTA
  uint4 raw[3];
  {
    // range of |x| over the raw BF16 bit patterns, which stay in registers
    uint32_t mx = 0, mn = 0xFFFFu;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      const int u = tid + k * kRingConsumers;
      raw[k] = u < nx ? xs[u] : make_uint4(0, 0, 0, 0);
      const uint32_t w4[4] = {raw[k].x, raw[k].y, raw[k].z, raw[k].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t lo = w4[j] & 0x7FFFu, hi = (w4[j] >> 16) & 0x7FFFu;
        mx = max(mx, max(lo, hi));
        mn = min(mn, min(lo ? lo : 0xFFFFu, hi ? hi : 0xFFFFu));
      }
    }
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    mn = __reduce_min_sync(0xFFFFFFFFu, mn);
    if (lane == 0) { red[warp] = mx; red[16 + warp] = mn; }
    ring_sync(kRingConsumers);  // every raw value is in registers: the buffer may be overwritten
    failed = *x_failed != 0;
    mx = red[0]; mn = red[16];
#pragma unroll
    for (int w = 1; w < kRingConsumerWarps; ++w) { mx = max(mx, red[w]); mn = min(mn, red[16 + w]); }
    if (mx >= 0x7F80u) {
      fast = false;
    } else if (mx != 0) {
      const int hi_exp = bf16_ilogb(mx), lo_exp = bf16_ilogb(mn);
      e = 15 - hi_exp;
      fast = hi_exp - lo_exp <= 32;
    }
  }
  if (!failed && !fast) {  // x outside the f16 window: the producer stops, every warp takes rows exactly
    *abort_flag = 1;
    const int nrows = min(N - row_base, nb_here * BR);
    for (int r = warp; r < nrows; r += kRingConsumerWarps) {
      const float v = dot_exact_range<MX>(x, q, s, K, row_base + r, k0, k1) * gv;
      if (lane == 0) emit(r / BR, r % BR, v);
    }
  } else if (!failed) {
    const int e1 = e / 2, e2 = e - e1;  // two exact power-of-two steps
    const float m1 = exp2i(e1), m2 = exp2i(e2);
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      const int u = tid + k * kRingConsumers;  // x[8u .. 8u+8): column u/64, chunk (u%64)/4, word u%4
      if (u < nx) {
        const uint32_t w4[4] = {raw[k].x, raw[k].y, raw[k].z, raw[k].w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const __half2 h = __floats2half2_rn(bf16lo_to_float(w4[j]) * m1 * m2, bf16hi_to_float(w4[j]) * m1 * m2);
          o[j] = *reinterpret_cast<const uint32_t*>(&h);
        }
        xs[(u >> 6) * 64 + (u & 3) * 16 + ((u & 63) >> 2)] = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
    // the last column's elements past K meet zero codes: their x must be finite
    for (int u = nx + tid; u < ncols * 64; u += kRingConsumers)
      xs[(u >> 6) * 64 + (u & 3) * 16 + ((u & 63) >> 2)] = make_uint4(0, 0, 0, 0);
    ring_sync(kRingConsumers);
    // (the next launch is triggered by the producer when two stages are left
    // to request: its CTAs then take the other half of each SM while this
    // kernel drains its last stages, instead of waiting there for most of
    // its run)

    // lane: rows slot0 + 30 i (i < NR) of each stage, 16-byte chunk c of each;
    // the warp's two slots are 2w and 2w + 1, so NR counts the i whose even
    // row is below BR (warp-uniform; one compiled loop per count)
    const int c = tid & (kRingChunks - 1);
    const int slot0 = tid / kRingChunks;
    const int nrow_i = min(kRingRows, (BR - 2 * warp + kRingSlots - 1) / kRingSlots);
    const uint8_t* lane_codes = ring + slot0 * kRingBK + c * 16;
    const uint8_t* lane_scales = ring + BR * kRingBK + slot0 * kSB + (MX ? c : 2 * c);
    const uint4* lane_x = xs + c;
    bool ok;
    switch (nrow_i) {
      case 4: ok = ring_rows<MX, 4>(lane_codes, lane_scales, lane_x, full, empty, S, SB, nb_here, ncols, c, slot0, BR, gv, e, emit); break;
      case 3: ok = ring_rows<MX, 3>(lane_codes, lane_scales, lane_x, full, empty, S, SB, nb_here, ncols, c, slot0, BR, gv, e, emit); break;
      case 2: ok = ring_rows<MX, 2>(lane_codes, lane_scales, lane_x, full, empty, S, SB, nb_here, ncols, c, slot0, BR, gv, e, emit); break;
      case 1: ok = ring_rows<MX, 1>(lane_codes, lane_scales, lane_x, full, empty, S, SB, nb_here, ncols, c, slot0, BR, gv, e, emit); break;
      default: ok = ring_rows<MX, 0>(lane_codes, lane_scales, lane_x, full, empty, S, SB, nb_here, ncols, c, slot0, BR, gv, e, emit); break;
    }
    if (!ok) {
      if (lane == 0) atomicAdd(&g_gemv_wait_timeouts, 1u);
      *abort_flag = 1;
      failed = true;
    }
  }
  if (C == 1) return;

  // ---- K split over the cluster: every CTA's partials are in its shared
  // memory; rank r adds rows [r R / C, (r + 1) R / C) of the R rows over the
  // ranks in order and stores them.  Every consumer thread passes both
  // cluster barriers (also after a failed wait: its partials are then NaN),
  // so no CTA exits while another reads its shared memory.
  if (failed)
    for (int i = tid; i < nb_here * BR; i += kRingConsumers) part[i] = __int_as_float(0x7FC00000);
  ptx::cluster_sync();
  {
    const int R = nb_here * BR;
    const int lo = (int)((int64_t)rank * R / C), hi = (int)((int64_t)(rank + 1) * R / C);
    for (int r = lo + tid; r < hi; r += kRingConsumers) {
      float v = ptx::ld_cluster_f32(part + r, 0);
      for (int j = 1; j < C; ++j) v += ptx::ld_cluster_f32(part + r, (uint32_t)j);
      const int row = row_base + r;
      if (row < N) {
        const __nv_bfloat16 o = __float2bfloat16_rn(v);
        y[row] = *reinterpret_cast<const uint16_t*>(&o);
      }
    }
  }
  ptx::cluster_sync();
}

// The same ring for one unsplit problem with rows of at least 90 per block:
// a fixed 120-row stage layout and 4 consecutive rows per lane (every lane's
// rows are valid, so no per-warp row counts).  Measured faster on the
// 17408-row decode layer than the general kernel above (10.4 against
// 10.9 µs per launch in one process on one B200); the general kernel serves
// split-K, grouped and short-row launches.  With static weights the first
// stage is requested before the dependency wait, and the next launch is
// triggered when two stages are left to request (9.9 µs per launch).
constexpr int kRing1ScOff = kRingMaxBR * kRingBK;                      // scales after a fixed 120-row code block
constexpr int kRing1Stage = kRing1ScOff + kRingMaxBR * (kRingBK / 8);  // 34560 bytes
constexpr int kRing1MinBR = 90;                                        // rows per block the kernel is used from

template <bool MX>
__global__ void __launch_bounds__(kRingThreads, 2)
    gemv_ring1_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap ts,
                     const uint16_t* __restrict__ x, const uint8_t* __restrict__ q, const uint8_t* __restrict__ s,
                     const float* __restrict__ g, uint16_t* __restrict__ y, int N, int K, int BR, int nblk,
                     int S, int static_w) {
  extern __shared__ __align__(1024) uint8_t sm[];
  constexpr int kSB = MX ? kRingBK / 16 : kRingBK / 8;  // scale bytes of a row per stage
  const int nks = (K / 2 + kRingBK - 1) / kRingBK;  // stages per row block
  uint8_t* ring = sm;
  uint4* xs = reinterpret_cast<uint4*>(sm + S * kRing1Stage);
  uint64_t* full = reinterpret_cast<uint64_t*>(xs + nks * 64);
  uint64_t* empty = full + S;
  uint64_t* xfull = empty + S;
  uint32_t* red = reinterpret_cast<uint32_t*>(xfull + 1);        // [2][16]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(red + 32);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row_base = blockIdx.x * nblk * BR;
  const int nb_here = min(nblk, (N - row_base + BR - 1) / BR);
  const int total = nb_here * nks;

  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], kRingConsumerWarps);
    }
    ptx::mbar_init(xfull, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();

  if (warp == kRingConsumerWarps) {  // ------------------------------------------------- producer
    if (lane != 0) return;
    ptx::prefetch_tmap(&tq);
    ptx::prefetch_tmap(&ts);
    uint64_t policy;  // each weight byte is read once: do not keep it in L2
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(policy));
    int n = 0, slot = 0, t = 0, rb = 0, e_id = 0;
    uint32_t phase = 0;
    auto issue = [&]() {
      uint8_t* dst = ring + slot * kRing1Stage;
      const int row0 = row_base + rb * BR;
      ptx::mbar_arrive_expect_tx(&full[slot], (uint32_t)BR * (kRingBK + kSB));
      tma_load_3d_evict_first(dst, &tq, &full[slot], t * kRingBK, row0, e_id, policy);
      tma_load_3d_evict_first(dst + kRing1ScOff, &ts, &full[slot], t * kSB, row0, e_id, policy);
      if (++slot == S) { slot = 0; phase ^= 1; }
      if (++t == nks) { t = 0; ++rb; }
    };
    // static weights: the first stage is requested before the previous kernel
    // has finished (one stage: more delayed x and the running kernel's stream)
    if (static_w && total > 0) {
      issue();
      ++n;
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");  // x (and, without static weights, the weights) only after this
    ptx::mbar_arrive_expect_tx(xfull, (uint32_t)K * 2);
    ptx::bulk_load(xs, x, (uint32_t)K * 2, xfull);
    for (; n < total; ++n) {
      if (n >= S) {  // wait until the consumers have released this slot (or have given up on the ring)
        bool ok = ptx::mbar_try_wait(&empty[slot], phase ^ 1);
        const uint64_t t0 = ok ? 0 : ptx::globaltimer_ns();
        while (!ok && !*abort_flag) {
          if (ptx::globaltimer_ns() - t0 > kRingWaitNs) {
            atomicAdd(&g_gemv_wait_timeouts, 1u);
            break;
          }
          ok = ptx::mbar_try_wait(&empty[slot], phase ^ 1);
        }
        if (!ok) break;
      }
      if (*abort_flag) break;
      issue();
      // the next launch may start once this CTA has two stages left to request
      // (9.9 us per launch, steady; at the end of the loop the time split
      // between 9.9 and 10.4 us from launch to launch)
      if (n == total - 3) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // short rings and early exits
    // nothing may still be landing in shared memory when the CTA exits
    for (int m = max(0, n - S); m < n; ++m) ptx::mbar_wait(&full[m % S], (m / S) & 1, kRingWaitNs);
    ptx::mbar_wait(xfull, 0, kRingWaitNs);
    return;
  }

  // ------------------------------------------------------------------------------- consumers
  asm volatile("griddepcontrol.wait;" ::: "memory");  // y is written only after the previous kernel
  if (!__all_sync(0xFFFFFFFFu, ptx::mbar_wait(xfull, 0, kRingWaitNs))) {
    if (lane == 0) atomicAdd(&g_gemv_wait_timeouts, 1u);
    *abort_flag = 1;
    return;
  }
  // range of |x| over the raw BF16 bit patterns, which stay in registers
  const int nx = K >> 3;
  uint4 raw[3];
  uint32_t mx = 0, mn = 0xFFFFu;
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const int u = tid + k * kRingConsumers;
    raw[k] = u < nx ? xs[u] : make_uint4(0, 0, 0, 0);
    const uint32_t w4[4] = {raw[k].x, raw[k].y, raw[k].z, raw[k].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t lo = w4[j] & 0x7FFFu, hi = (w4[j] >> 16) & 0x7FFFu;
      mx = max(mx, max(lo, hi));
      mn = min(mn, min(lo ? lo : 0xFFFFu, hi ? hi : 0xFFFFu));
    }
  }
  mx = __reduce_max_sync(0xFFFFFFFFu, mx);
  mn = __reduce_min_sync(0xFFFFFFFFu, mn);
  if (lane == 0) { red[warp] = mx; red[16 + warp] = mn; }
  ring_sync(kRingConsumers);  // every raw value is in registers: the buffer may be overwritten
  mx = red[0]; mn = red[16];
#pragma unroll
  for (int w = 1; w < kRingConsumerWarps; ++w) { mx = max(mx, red[w]); mn = min(mn, red[16 + w]); }
  bool fast = true;
  int e = 0;
  if (mx >= 0x7F80u) {
    fast = false;
  } else if (mx != 0) {
    const int hi_exp = bf16_ilogb(mx), lo_exp = bf16_ilogb(mn);
    e = 15 - hi_exp;
    fast = hi_exp - lo_exp <= 32;
  }
  const float gv = MX ? 1.0f : *g;
  if (!fast) {  // x outside the f16 window: the producer stops, every warp takes rows exactly
    *abort_flag = 1;
    const int nrows = min(N - row_base, nblk * BR);
    for (int r = warp; r < nrows; r += kRingConsumerWarps) rows_exact<MX>(x, q, s, g, y, N, K, row_base + r, 1);
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    return;
  }
  {
    const int e1 = e / 2, e2 = e - e1;  // two exact power-of-two steps
    const float m1 = exp2i(e1), m2 = exp2i(e2);
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      const int u = tid + k * kRingConsumers;  // x[8u .. 8u+8): stage u/64, chunk (u%64)/4, word u%4
      if (u < nx) {
        const uint32_t w4[4] = {raw[k].x, raw[k].y, raw[k].z, raw[k].w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const __half2 h = __floats2half2_rn(bf16lo_to_float(w4[j]) * m1 * m2, bf16hi_to_float(w4[j]) * m1 * m2);
          o[j] = *reinterpret_cast<const uint32_t*>(&h);
        }
        xs[(u >> 6) * 64 + (u & 3) * 16 + ((u & 63) >> 2)] = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
    // the last stage's columns past K meet zero codes: their x must be finite
    for (int u = nx + tid; u < nks * 64; u += kRingConsumers)
      xs[(u >> 6) * 64 + (u & 3) * 16 + ((u & 63) >> 2)] = make_uint4(0, 0, 0, 0);
  }
  ring_sync(kRingConsumers);
  // (the next launch is triggered by the producer when two stages are left to
  // request: 9.9 µs per launch, against 10.4 with the trigger here, after x is
  // staged)

  // lane: rows r0 .. r0+3 of the 120-row stage layout, 16-byte chunk c of each
  // (rows at or past BR hold stale bytes; their sums are never stored)
  const int c = tid & (kRingChunks - 1);
  const int r0 = (tid / kRingChunks) * kRingRows;
  const uint8_t* lane_codes = ring + r0 * kRingBK + c * 16;
  const uint8_t* lane_scales = ring + kRing1ScOff + r0 * kSB + (MX ? c : 2 * c);
  const uint4* lane_x = xs + c;
  int slot = 0;
  uint32_t phase = 0;
  for (int rb = 0; rb < nb_here; ++rb) {
    float acc[kRingRows] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (int t = 0; t < nks; ++t) {
      if (!__all_sync(0xFFFFFFFFu, ptx::mbar_wait(&full[slot], phase, kRingWaitNs))) {
        if (lane == 0) atomicAdd(&g_gemv_wait_timeouts, 1u);
        *abort_flag = 1;
        return;
      }
      const uint8_t* pc = lane_codes + slot * kRing1Stage;
      const uint8_t* ps = lane_scales + slot * kRing1Stage;
      uint4 cw[kRingRows];
      uint32_t sc[kRingRows];
#pragma unroll
      for (int i = 0; i < kRingRows; ++i) {
        cw[i] = *reinterpret_cast<const uint4*>(pc + i * kRingBK);
        sc[i] = MX ? (uint32_t)ps[i * kSB] : (uint32_t)*reinterpret_cast<const uint16_t*>(ps + i * kSB);
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&empty[slot]);  // the stage's bytes are in registers
      if (++slot == S) { slot = 0; phase ^= 1; }
      const uint4* xp = lane_x + t * 64;
      float part[kRingRows][2];
#pragma unroll
      for (int i = 0; i < kRingRows; ++i) part[i][0] = part[i][1] = 0.0f;
#pragma unroll
      for (int wi = 0; wi < 4; ++wi) {  // 8 weights per 32-bit word; words 0-1 block 0, words 2-3 block 1
        const uint4 xv = xp[wi * 16];
#pragma unroll
        for (int i = 0; i < kRingRows; ++i) {
          const uint32_t word = wi == 0 ? cw[i].x : wi == 1 ? cw[i].y : wi == 2 ? cw[i].z : cw[i].w;
          float p = part[i][wi >> 1];
          p = fma2_f16_f32(e2m1x2_byte_to_f16x2<0>(word), xv.x, p);
          p = fma2_f16_f32(e2m1x2_byte_to_f16x2<1>(word), xv.y, p);
          p = fma2_f16_f32(e2m1x2_byte_to_f16x2<2>(word), xv.z, p);
          p = fma2_f16_f32(e2m1x2_byte_to_f16x2<3>(word), xv.w, p);
          part[i][wi >> 1] = p;
        }
      }
#pragma unroll
      for (int i = 0; i < kRingRows; ++i) {
        if constexpr (MX) {  // one 32-element block per chunk
          acc[i] = fmaf(part[i][0] + part[i][1], e8m0_to_float(sc[i]), acc[i]);
        } else {
          const float2 sf = f16x2_to_float2(e4m3x2_to_f16x2(sc[i]));
          acc[i] = fmaf(part[i][0], sf.x, acc[i]);
          acc[i] = fmaf(part[i][1], sf.y, acc[i]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kRingRows; ++i) {
      float v = acc[i];
#pragma unroll
      for (int o = kRingChunks / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
      acc[i] = v;
    }
    if (c < kRingRows) {
      const float v = c == 0 ? acc[0] : c == 1 ? acc[1] : c == 2 ? acc[2] : acc[3];
      const int rl = r0 + c;
      const int row = row_base + rb * BR + rl;
      if (rl < BR && row < N) {
        const __nv_bfloat16 o = __float2bfloat16_rn(ldexpf(v * gv, -e));
        y[row] = *reinterpret_cast<const uint16_t*>(&o);
      }
    }
  }
}

struct RingPlan {
  int BR, nblk, grid, S, SB, C;
  size_t smem;
  int64_t budget;  // shared memory a CTA may take (half of the SM)
};

// The ring kernel's shape: split K over C in {1, 2, 4, 8} CTAs of a cluster
// (forced when force_c != 0), rows split evenly over the SMs' worth of
// clusters, shared memory for 2..8 stages within half of the SM.  Without a
// forced C: no split when it fits and keeps at least 64 KB of weights in
// flight per CTA, else a split of 2, else the smallest split that fits.  (A
// sweep of six 5120..17408-row layers on B200: C = 1 is fastest whenever its
// ring holds 64 KB or more; a short ring (a few rows per CTA) loses to C = 2;
// C = 4 and 8 were 30-70% slower than C = 2 at equal work per CTA, so they
// are used only when one CTA's x slice would be too long otherwise.)  False
// when no split fits.
bool ring_plan(int64_t N, int64_t K, int sms, bool mx, int num_problems, int force_c, RingPlan& p) {
  // TMA row strides are multiples of 16 bytes: K/16 (NVFP4) or K/32 (MXFP4) scale bytes
  if (K % (mx ? 512 : 256) != 0 || N < 1 || sms < 1 || N > (int64_t)1 << 30) return false;
  int dev = 0, per_sm = 0, reserved = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess)
    return false;
  const int kSB = mx ? kRingBK / 16 : kRingBK / 8;
  const int64_t nks = (K / 2 + kRingBK - 1) / kRingBK;
  const int64_t budget = per_sm / 2 - reserved;  // two such CTAs per SM
  bool fallback_c1 = false;  // (p holds the C = 1 plan when its ring was short)
  bool found = false;
  for (int C = 1; C <= 8 && !found; C *= 2) {
    if (force_c && C != force_c) continue;
    if ((num_problems > 1 && C > 1) || C > nks) continue;  // grouped calls split rows only
    const int64_t ncx = (nks + C - 1) / C;
    if (ncx * 2 * kRingBK > kRingMaxSlice) continue;       // x slice of a CTA
    const int64_t clusters = std::max<int64_t>(1, sms / C);
    const int64_t rpc = ((int64_t)num_problems * N + clusters - 1) / clusters;  // rows of all problems over the clusters
    RingPlan c;
    c.C = C;
    c.budget = budget;
    c.nblk = (int)((rpc + kRingMaxBR - 1) / kRingMaxBR);
    c.BR = (int)((rpc + c.nblk - 1) / c.nblk);
    c.grid = (int)((N + (int64_t)c.nblk * c.BR - 1) / ((int64_t)c.nblk * c.BR)) * C;
    c.SB = (c.BR * (kRingBK + kSB) + 127) / 128 * 128;
    const int64_t fixed = ncx * 1024 + 8 * (2 * kRingMaxStages + 1) + 36 * 4 + (int64_t)4 * c.nblk * c.BR + 64;
    c.S = (int)std::min<int64_t>(kRingMaxStages, (budget - fixed) / c.SB);
    if (c.S < 2) continue;
    c.smem = (size_t)(c.S * c.SB + fixed);
    const bool last_choice = force_c != 0 || C == 8 || (num_problems > 1);
    if (C == 1 && !last_choice && (int64_t)c.S * c.SB < kRingMinInFlight) {
      // a short ring: keep it only if no split fits
      if (!found) p = c;
      found = false;
      fallback_c1 = true;
      continue;
    }
    p = c;
    found = true;
  }
  return found || fallback_c1;
}

template <bool MX, bool GROUPED>
cudaError_t launch_ring(const uint16_t* x, const uint8_t* q, const uint8_t* s, const float* g, uint16_t* y,
                        int64_t N, int64_t K, cudaStream_t stream, const RingPlan& p, const Problems& P,
                        int num_problems, bool static_weights, bool* encoded) {
  CUtensorMap tq, ts;  // [E, N, K/2] codes and [E, N, scale bytes]: the expert is the third coordinate
  const int64_t sbytes = MX ? K / 32 : K / 16;  // scale bytes per row
  const int64_t E = P.expert_ids ? P.E : 1;
  *encoded = tc::make_tmap_3d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, K / 2, N, E, K / 2, N * (K / 2), kRingBK,
                              p.BR, CU_TENSOR_MAP_SWIZZLE_NONE) &&
             tc::make_tmap_3d(&ts, CU_TENSOR_MAP_DATA_TYPE_UINT8, s, sbytes, N, E, sbytes, N * sbytes,
                              MX ? kRingBK / 16 : kRingBK / 8, p.BR, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!*encoded) return cudaSuccess;
  int Ni = (int)N, Ki = (int)K, BR = p.BR, nblk = p.nblk, S = p.S, SB = p.SB, C = p.C;
  if (!GROUPED && p.C == 1 && p.BR >= kRing1MinBR) {  // one unsplit problem with full row blocks
    const int64_t nks = (K / 2 + kRingBK - 1) / kRingBK;
    const int64_t fixed = nks * 1024 + 256;
    const int S1 = (int)std::min<int64_t>(4, (p.budget - fixed) / kRing1Stage);
    if (S1 >= 2) {
      const size_t smem1 = (size_t)(S1 * kRing1Stage + fixed);
      static tc::SmemOptIn opt_in1;
      cudaError_t e = opt_in1.ensure((const void*)gemv_ring1_kernel<MX>, (int)smem1);
      if (e != cudaSuccess) return e;
      int S1v = S1, sw = static_weights ? 1 : 0;
      void* args1[] = {&tq, &ts, &x, &q, &s, &g, &y, &Ni, &Ki, &BR, &nblk, &S1v, &sw};
      return tc::launch_pdl((const void*)gemv_ring1_kernel<MX>, dim3(p.grid), dim3(kRingThreads), smem1, stream, args1);
    }
  }
  static tc::SmemOptIn opt_in;
  cudaError_t e = opt_in.ensure((const void*)gemv_ring_kernel<MX, GROUPED>, (int)p.smem);
  if (e != cudaSuccess) return e;
  Problems Pc = P;
  void* args[] = {&tq, &ts, &x, &q, &s, &g, &y, &Ni, &Ki, &BR, &nblk, &S, &SB, &C, &Pc};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.grid, num_problems);
  cfg.blockDim = dim3(kRingThreads);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;  // the CTAs that split one row block's K
  attr[1].val.clusterDim.x = (unsigned)p.C;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.C > 1 ? 2 : 1;
  return cudaLaunchKernelExC(&cfg, (const void*)gemv_ring_kernel<MX, GROUPED>, args);
}

}  // namespace

namespace {

template <bool MX, bool GROUPED>
cudaError_t launch_any(const uint16_t* x, const uint8_t* q, const uint8_t* s, const float* g, uint16_t* y,
                       int64_t N, int64_t K, int sms, bool static_weights, cudaStream_t stream, const Problems& P,
                       int num_problems, int force_splits = 0) {
  RingPlan plan;
  if (ring_plan(N, K, sms, MX, num_problems, force_splits > 1 ? force_splits : (force_splits == 1 ? 1 : 0), plan)) {
    bool encoded = false;
    const cudaError_t e =
        launch_ring<MX, GROUPED>(x, q, s, g, y, N, K, stream, plan, P, num_problems, static_weights, &encoded);
    if (encoded || e != cudaSuccess) return e;
  }
  if (force_splits > 1) return cudaErrorInvalidConfiguration;  // the forced split does not fit this shape
  if (MX || K % 32 == 0)
    return launch<8, 16, 2, MX, GROUPED>(x, q, s, g, y, (int)N, (int)K, static_weights, stream, P, num_problems);
  return launch<8, 8, 2, false, GROUPED>(x, q, s, g, y, (int)N, (int)K, static_weights, stream, P, num_problems);
}

const Problems kSingle = {nullptr, nullptr, 1, 1, 0, 0};

}  // namespace

cudaError_t launch_gemv(const uint16_t* x, const uint8_t* q, const uint8_t* s, const float* g,
                        uint16_t* y, int64_t N, int64_t K, int sms, bool static_weights, cudaStream_t stream,
                        int splits) {
  return launch_any<false, false>(x, q, s, g, y, N, K, sms, static_weights, stream, kSingle, 1, splits);
}

cudaError_t launch_gemv_mx(const uint16_t* x, const uint8_t* q, const uint8_t* s, uint16_t* y, int64_t N,
                           int64_t K, int sms, bool static_weights, cudaStream_t stream, int splits) {
  return launch_any<true, false>(x, q, s, nullptr, y, N, K, sms, static_weights, stream, kSingle, 1, splits);
}

bool gemv_split_fits(int64_t N, int64_t K, int sms, bool mx, int splits) {
  RingPlan plan;
  return ring_plan(N, K, sms, mx, 1, splits, plan);
}

cudaError_t launch_gemv_grouped(const uint16_t* X, int64_t ldx, const uint8_t* q, const uint8_t* s,
                                const float* g, const int* expert_ids, const int* token_ids, uint16_t* Y,
                                int64_t ldy, int64_t P, int64_t E, int64_t T, int64_t N, int64_t K, int sms,
                                cudaStream_t stream) {
  const Problems pr = {expert_ids, token_ids, (int)E, (int)T, ldx, ldy};
  return launch_any<false, true>(X, q, s, g, Y, N, K, sms, false, stream, pr, (int)P);
}

cudaError_t read_and_clear_gemv_bad_ids(unsigned int* count) {
  cudaError_t e = cudaMemcpyFromSymbol(count, g_gemv_bad_ids, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  const unsigned int zero = 0;
  return cudaMemcpyToSymbol(g_gemv_bad_ids, &zero, sizeof(unsigned int));
}

cudaError_t read_and_clear_gemv_timeouts(unsigned int* count) {
  cudaError_t e = cudaMemcpyFromSymbol(count, g_gemv_wait_timeouts, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  const unsigned int zero = 0;
  return cudaMemcpyToSymbol(g_gemv_wait_timeouts, &zero, sizeof(unsigned int));
}

}  // namespace nvfp4

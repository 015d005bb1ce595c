// gemv_stream.cu -- persistent, TMA-fed batch-1 decode GEMV for K a multiple
// of 1024 (the 27B-class shapes: K = 5120 and K = 17408).
//
// Same arithmetic as gemv.cu (decode GEMV of imp docs/quantization.md, "Dense
// layers" pipeline; weight-only per the model card "Qwen3.8-27B-NVFP4"): every
// product e2m1 * x is exact and accumulated in fp32, the 16-block sums are
// scaled by their E4M3 scale, and y = bf16_rn(2^-e * (g * acc)).
//
// Structure (one CTA per SM, rows split evenly into contiguous ranges):
//   - a producer warp streams the CTA's rows with 1-D bulk copies
//     (cp.async.bulk) into a ring of shared-memory stages of RS rows each:
//     the codes of a run of rows are one contiguous block of global memory,
//     and so are their scales, so each stage is two copies;
//   - compute warp w owns the K slice [1024 (w % WK), +1024) of every row
//     (WK = K / 1024), so each lane keeps its 32 x values in registers for the
//     whole kernel; RG groups of WK warps take alternate rows of a stage;
//   - each warp reduces its RPW rows across lanes with a transposed butterfly
//     (one shuffle per row and lane instead of five) and leaves one partial
//     per row and K slice in shared memory;
//   - when a stage is released, the producer warp sums the WK partials of
//     each row in a fixed order (deterministic), applies g and 2^-e, and
//     stores y before refilling the stage.
// Each compute warp scales its own K slice of x by a power of two into f16
// (exact when the slice's range allows, else an exact fp32 path); the
// producer undoes each slice's scale before summing the slices.
#include "nvfp4_device.cuh"
#include "nvfp4_kernels.h"
#include "sm100_ptx.cuh"

#include <type_traits>

namespace nvfp4 {

__device__ unsigned int g_gemv_wait_timeouts = 0;

namespace {

constexpr uint64_t kWaitLimitNs = 2000000000ull;

// mbarrier wait with a suspend-time hint (the warp sleeps until the phase
// completes instead of spinning), bounded by wall-clock time.
__device__ __forceinline__ bool try_wait_sleep(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(ptx::smem_u32(bar)), "r"(parity), "r"(1000000u)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool wait_sleep(uint64_t* bar, uint32_t parity) {
  if (try_wait_sleep(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  while (!try_wait_sleep(bar, parity))
    if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) return false;
  return true;
}




__device__ __forceinline__ uint4 lds128(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }

// Dot product of one 16-byte code chunk (32 weights, two 16-blocks) with this
// lane's x slice: f16 fast path.
__device__ __forceinline__ float chunk_dot_f16(uint4 w, uint32_t sc2, const uint32_t (&xh)[16]) {
  float a0 = 0.0f, a1 = 0.0f, b0 = 0.0f, b1 = 0.0f;  // four short chains
  a0 = fma2_f16_f32(e2m1x2_byte_to_f16x2<0>(w.x), xh[0], a0);
  a1 = fma2_f16_f32(e2m1x2_byte_to_f16x2<1>(w.x), xh[1], a1);
  b0 = fma2_f16_f32(e2m1x2_byte_to_f16x2<0>(w.z), xh[8], b0);
  b1 = fma2_f16_f32(e2m1x2_byte_to_f16x2<1>(w.z), xh[9], b1);
  a0 = fma2_f16_f32(e2m1x2_byte_to_f16x2<2>(w.x), xh[2], a0);
  a1 = fma2_f16_f32(e2m1x2_byte_to_f16x2<3>(w.x), xh[3], a1);
  b0 = fma2_f16_f32(e2m1x2_byte_to_f16x2<2>(w.z), xh[10], b0);
  b1 = fma2_f16_f32(e2m1x2_byte_to_f16x2<3>(w.z), xh[11], b1);
  a0 = fma2_f16_f32(e2m1x2_byte_to_f16x2<0>(w.y), xh[4], a0);
  a1 = fma2_f16_f32(e2m1x2_byte_to_f16x2<1>(w.y), xh[5], a1);
  b0 = fma2_f16_f32(e2m1x2_byte_to_f16x2<0>(w.w), xh[12], b0);
  b1 = fma2_f16_f32(e2m1x2_byte_to_f16x2<1>(w.w), xh[13], b1);
  a0 = fma2_f16_f32(e2m1x2_byte_to_f16x2<2>(w.y), xh[6], a0);
  a1 = fma2_f16_f32(e2m1x2_byte_to_f16x2<3>(w.y), xh[7], a1);
  b0 = fma2_f16_f32(e2m1x2_byte_to_f16x2<2>(w.w), xh[14], b0);
  b1 = fma2_f16_f32(e2m1x2_byte_to_f16x2<3>(w.w), xh[15], b1);
  const float2 sc = f16x2_to_float2(e4m3x2_to_f16x2(sc2));
  return fmaf(b0 + b1, sc.y, (a0 + a1) * sc.x);
}

// Same with x read as BF16 from global memory (L1-cached) and widened to fp32:
// the exact path for x of extreme dynamic range, kept out of registers.
__device__ __forceinline__ float chunk_dot_f32(uint4 w, uint32_t sc2, const uint16_t* __restrict__ xg) {
  const uint32_t words[4] = {w.x, w.y, w.z, w.w};
  float2 p[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll
  for (int wi = 0; wi < 4; ++wi) {
    const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xg) + wi);  // 8 BF16
    float2& a = p[wi >> 1];
    a = __ffma2_rn(f16x2_to_float2(e2m1x2_byte_to_f16x2<0>(words[wi])),
                   make_float2(bf16lo_to_float(xv.x), bf16hi_to_float(xv.x)), a);
    a = __ffma2_rn(f16x2_to_float2(e2m1x2_byte_to_f16x2<1>(words[wi])),
                   make_float2(bf16lo_to_float(xv.y), bf16hi_to_float(xv.y)), a);
    a = __ffma2_rn(f16x2_to_float2(e2m1x2_byte_to_f16x2<2>(words[wi])),
                   make_float2(bf16lo_to_float(xv.z), bf16hi_to_float(xv.z)), a);
    a = __ffma2_rn(f16x2_to_float2(e2m1x2_byte_to_f16x2<3>(words[wi])),
                   make_float2(bf16lo_to_float(xv.w), bf16hi_to_float(xv.w)), a);
  }
  const float2 sc = f16x2_to_float2(e4m3x2_to_f16x2(sc2));
  return fmaf(p[1].x + p[1].y, sc.y, (p[0].x + p[0].y) * sc.x);
}

// Reduce RPW per-lane values over the 32 lanes; afterwards lane l holds the
// full sum of value j(l) = sum over the top log2(RPW) bits of l.
template <int RPW>
__device__ __forceinline__ float transpose_reduce(float (&v)[RPW], int lane) {
  int count = RPW;
  int off = 16;
#pragma unroll
  for (int step = 0; (1 << step) < RPW; ++step) {
    const int half = count / 2;
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < RPW / 2; ++i) {
      if (i < half) {
        const float send = upper ? v[i] : v[i + half];
        const float keep = upper ? v[i + half] : v[i];
        v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, off);
      }
    }
    count = half;
    off >>= 1;
  }
  float r = v[0];
  for (; off > 0; off >>= 1) r += __shfl_xor_sync(0xFFFFFFFFu, r, off);
  return r;
}

template <int RPW>
__device__ __forceinline__ int transposed_index(int lane) {
  int j = 0, off = 16, span = RPW;
#pragma unroll
  for (int step = 0; (1 << step) < RPW; ++step) {
    span >>= 1;
    if (lane & off) j += span;
    off >>= 1;
  }
  return j;
}

struct StreamShape {
  int wk, rg, rs, ns;
};

template <int RPW, int MAXT>
__global__ void __launch_bounds__(MAXT, 1)
    gemv_stream_kernel(const uint16_t* __restrict__ x, const uint8_t* __restrict__ q, const uint8_t* __restrict__ s,
                       const float* __restrict__ g, uint16_t* __restrict__ y, int N, int K, StreamShape sh,
                       int static_weights) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float slice_scale[32];  // per K slice: 2^-e, e the power of two its x was scaled by
  __shared__ int s_err;
  const int wk = sh.wk, rg = sh.rg, rs = sh.rs, ns = sh.ns;
  const int n_compute = wk * rg;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row_bytes = K >> 1, row_sc = K >> 4;
  const int stage_q = rs * row_bytes, stage_bytes = rs * (row_bytes + row_sc);
  float* red = reinterpret_cast<float*>(smem + (size_t)ns * stage_bytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(red + ns * rs * wk + ((ns * rs * wk) & 1));
  uint64_t* empty = full + ns;

  const int row_begin = (int)((int64_t)N * blockIdx.x / gridDim.x);
  const int row_end = (int)((int64_t)N * (blockIdx.x + 1) / gridDim.x);
  const int nrows = row_end - row_begin;
  const int nstages = (nrows + rs - 1) / rs;
  const bool producer = warp == n_compute;

  if (threadIdx.x == 0) {
    for (int i = 0; i < ns; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], n_compute);
    }
    s_err = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();

  auto issue = [&](int i, int st) {
    const int r0 = row_begin + i * rs;
    const int cnt = min(rs, nrows - i * rs);
    uint8_t* dq = smem + (size_t)st * stage_bytes;
    uint8_t* ds = dq + stage_q;
    const uint32_t bq = (uint32_t)cnt * row_bytes, bs = (uint32_t)cnt * row_sc;
    ptx::mbar_arrive_expect_tx(&full[st], bq + bs);
    ptx::bulk_load(dq, q + (int64_t)r0 * row_bytes, bq, &full[st]);
    ptx::bulk_load(ds, s + (int64_t)r0 * row_sc, bs, &full[st]);
  };
  // Programmatic dependent launch: let the next kernel on the stream start its
  // prologue now; read q and s before the previous kernel has finished only
  // when the caller declared them static, and x, g, y only after it has.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (!static_weights) asm volatile("griddepcontrol.wait;" ::: "memory");
  if (producer && lane == 0)
    for (int i = 0; i < min(ns, nstages); ++i) issue(i, i);
  if (static_weights) asm volatile("griddepcontrol.wait;" ::: "memory");

  if (!producer && warp < n_compute) {
    // ------------------------------------------------------------ compute
    const int kw = warp % wk, rgi = warp / wk;
    const int kbase = kw * 1024 + lane * 32;  // this lane's 32 x elements
    // This warp's K slice of x as f16 scaled by 2^e, e chosen from the
    // slice's own range (exact when its non-zero magnitudes lie within 2^32
    // of each other and it is finite; else the exact fp32 path).  The
    // producer scales each slice's partial sums back by 2^-e before the
    // fixed-order sum, so no block-wide pass over x is needed.
    uint4 xv[4];
    {
      const uint4* xp = reinterpret_cast<const uint4*>(x + kbase);
#pragma unroll
      for (int c = 0; c < 4; ++c) xv[c] = xp[c];
    }
    uint32_t mx = 0, mn = 0xFFFFu;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t w4[4] = {xv[c].x, xv[c].y, xv[c].z, xv[c].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t lo = w4[j] & 0x7FFFu, hi = (w4[j] >> 16) & 0x7FFFu;
        mx = max(mx, max(lo, hi));
        mn = min(mn, min(lo ? lo : 0xFFFFu, hi ? hi : 0xFFFFu));
      }
    }
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    mn = __reduce_min_sync(0xFFFFFFFFu, mn);
    bool fast = true;
    int e = 0;
    if (mx >= 0x7F80u) {
      fast = false;
    } else if (mx != 0) {
      const int hi_exp = bf16_ilogb(mx), lo_exp = bf16_ilogb(mn);
      e = 15 - hi_exp;
      fast = hi_exp - lo_exp <= 32;
    }
    if (!fast) e = 0;
    // read by the producer after the first stage: 2^-e (subnormal below 2^-126)
    if (rgi == 0 && lane == 0)
      slice_scale[kw] = e <= 126 ? exp2i(-e) : __uint_as_float(1u << (149 - e));
    uint32_t xh[16];
    {
      const int e1 = e / 2, e2 = e - e1;
      const float m1 = exp2i(e1), m2 = exp2i(e2);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t w4[4] = {xv[c].x, xv[c].y, xv[c].z, xv[c].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const __half2 h = __floats2half2_rn(bf16lo_to_float(w4[j]) * m1 * m2, bf16hi_to_float(w4[j]) * m1 * m2);
          xh[4 * c + j] = *reinterpret_cast<const uint32_t*>(&h);
        }
      }
    }
    const int jrow = transposed_index<RPW>(lane);
    const bool writer = (lane & ((32 / RPW) - 1)) == 0;
    const int q_off = rgi * row_bytes + kw * 512 + lane * 16;   // row rgi of a stage, this lane's chunk
    const int s_off = stage_q + rgi * row_sc + kw * 64 + lane * 2;
    const int q_step = rg * row_bytes, s_step = rg * row_sc;    // next row of this row group
    const int red_off = (rgi + jrow * rg) * wk + kw;
    const uint16_t* xg = x + kbase;
    auto consume = [&](auto fast_tag) {
      constexpr bool kFast = decltype(fast_tag)::value;
      int st = 0;
      uint32_t phase = 0;
      for (int i = 0; i < nstages; ++i) {
        if (!wait_sleep(&full[st], phase)) {
          if (lane == 0 && atomicExch(&s_err, 1) == 0) atomicAdd(&g_gemv_wait_timeouts, 1u);
          break;
        }
        const int rows_here = min(rs, nrows - i * rs);
        const uint8_t* base = smem + (size_t)st * stage_bytes;
        float part[RPW];
#pragma unroll
        for (int j = 0; j < RPW; ++j) {
          part[j] = 0.0f;
          if (rgi + j * rg < rows_here) {
            const uint4 w = lds128(base + q_off + j * q_step);
            const uint32_t sc2 = *reinterpret_cast<const uint16_t*>(base + s_off + j * s_step);
            if constexpr (kFast)
              part[j] = chunk_dot_f16(w, sc2, xh);
            else
              part[j] = chunk_dot_f32(w, sc2, xg);
          }
        }
        const float tot = transpose_reduce<RPW>(part, lane);
        if (writer) red[st * rs * wk + red_off] = tot;
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&empty[st]);
        if (++st == ns) {
          st = 0;
          phase ^= 1u;
        }
      }
    };
    if (fast)
      consume(std::true_type{});
    else
      consume(std::false_type{});
  } else if (producer) {
    // ------------------------------------------- finish rows, refill stages
    const float gv = *g;
    int st = 0;
    uint32_t phase = 0;
    for (int i = 0; i < nstages; ++i) {
      // spin (no suspend): the refill below is on the critical path
      if (!ptx::mbar_wait(&empty[st], phase, kWaitLimitNs)) {
        if (lane == 0 && atomicExch(&s_err, 1) == 0) atomicAdd(&g_gemv_wait_timeouts, 1u);
        break;
      }
      // refill the stage first (its partial sums live in a separate buffer
      // that is rewritten only after this refill has landed and been read)
      if (lane == 0 && i + ns < nstages) issue(i + ns, st);
      const int rows_here = min(rs, nrows - i * rs);
      for (int r = lane; r < rows_here; r += 32) {
        const float* rp = red + (st * rs + r) * wk;
        float acc = 0.0f;
        for (int k = 0; k < wk; ++k) acc = fmaf(rp[k], slice_scale[k], acc);
        const float out = acc * gv;
        const __nv_bfloat16 o = __float2bfloat16_rn(out);
        y[row_begin + i * rs + r] = *reinterpret_cast<const uint16_t*>(&o);
      }
      __syncwarp();
      if (++st == ns) {
        st = 0;
        phase ^= 1u;
      }
    }
    if (s_err && lane == 0) {
      // let copies already in flight land before the CTA exits
      for (int i = 0; i < min(ns, nstages); ++i) ptx::mbar_wait(&full[i], 0, kWaitLimitNs);
    }
  }
}

template <int RPW, int MAXT>
cudaError_t launch_rpw(const uint16_t* x, const uint8_t* q, const uint8_t* s, const float* g, uint16_t* y, int N,
                       int K, StreamShape sh, int sms, int static_weights, cudaStream_t stream) {
  const int stage_bytes = sh.rs * (K / 2 + K / 16);
  const size_t smem = (size_t)sh.ns * stage_bytes + (size_t)sh.ns * sh.rs * sh.wk * 4 + 8 + 16 * sh.ns;
  static int smem_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || smem_set[dev] < (int)smem) {
    e = cudaFuncSetAttribute(gemv_stream_kernel<RPW, MAXT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) smem_set[dev] = (int)smem;
  }
  int grid = sms;
  const int max_ctas = (N + sh.rs - 1) / sh.rs;
  if (grid > max_ctas) grid = max_ctas;
  const int threads = (sh.wk * sh.rg + 1) * 32;
  if (threads > MAXT) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_stream_kernel<RPW, MAXT>, x, q, s, g, y, N, K, sh, static_weights);
}

}  // namespace

bool gemv_stream_supported(int64_t N, int64_t K) { return K % 1024 == 0 && K / 1024 <= 31 && N >= 1; }

cudaError_t launch_gemv_stream(const uint16_t* x, const uint8_t* q, const uint8_t* s, const float* g, uint16_t* y,
                               int64_t N, int64_t K, int sms, bool static_weights, cudaStream_t stream) {
  // About 20 compute warps per SM: WK warps cover one row, RG row groups.
  StreamShape sh;
  sh.wk = (int)(K / 1024);
  sh.rg = sh.wk >= 20 ? 1 : 20 / sh.wk;
  constexpr int kRpw = 4;
  sh.rs = sh.rg * kRpw;
  const int stage_bytes = sh.rs * (int)(K / 2 + K / 16);
  sh.ns = (200 * 1024) / stage_bytes;
  if (sh.ns > 8) sh.ns = 8;
  if (sh.ns < 2) {  // very large rows: fewer row groups per stage
    sh.rg = 1;
    sh.rs = kRpw;
    sh.ns = (200 * 1024) / (sh.rs * (int)(K / 2 + K / 16));
    if (sh.ns < 2) sh.ns = 2;
  }
  return launch_rpw<kRpw, 1024>(x, q, s, g, y, (int)N, (int)K, sh, sms, static_weights ? 1 : 0, stream);
}

cudaError_t read_and_clear_gemv_timeouts(unsigned int* count) {
  cudaError_t e = cudaMemcpyFromSymbol(count, g_gemv_wait_timeouts, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  const unsigned int zero = 0;
  return cudaMemcpyToSymbol(g_gemv_wait_timeouts, &zero, sizeof(unsigned int));
}

}  // namespace nvfp4

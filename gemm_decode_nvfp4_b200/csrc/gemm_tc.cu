// gemm_tc.cu -- W4A16 NVFP4 GEMM on the sm_100a tensor cores (tcgen05).
//
// Y[m, n] = bf16(g * sum_k W_deq[n, k] * X[m, k]) for the 32-user batched
// decode and the 512-token prefill of a 27B-class layer (model card
// "Qwen3.8-27B-NVFP4", "Measurements"; imp docs/quantization.md, "Dense layers"
// pipeline: the prefill GEMM reads the packed NVFP4 weights).  The pages'
// prefill runs a CUTLASS block-scaled FP4 x FP4 GEMM on sm_120; here the
// activations stay 16-bit (weight-only quantization, "What is quantized"), so
// the weights are dequantized on chip and the contraction runs as a 16-bit
// tcgen05 MMA with fp32 accumulation in tensor memory.
//
// Both MMA operands are f16 and every product is exact:
//   - a weight e2m1 * e4m3 has at most 6 significant bits and lies in
//     [2^-10, 2688], so it is an exact normal f16 (one cvt.rn.f16x2.e2m1x2 per
//     two codes and one f16x2 multiply by the block scale);
//   - prep_x_kernel writes X' = f16(X * 2^e_m) per row m with e_m chosen from
//     the row's max |x|; this is exact when the row is finite and its non-zero
//     magnitudes lie within 2^32 of each other (BF16 has 8 significant bits,
//     f16 keeps 11 down to 2^-24).  The epilogue undoes 2^e_m exactly.
// Rows outside that window ("wide" rows, a flag next to e_m) are recomputed
// after the epilogue by the CTA's dequant warps with an exact fp32 CUDA-core
// dot product over the original BF16 X, so the result never depends on the
// f16 window.
//
// Tile: 128 weight rows (MMA M, weights are operand A) x BNT = BN * NSUB
// activation rows (NSUB MMAs of N = BN per k-step), 64 k per MMA stage.
//   - warp 0, one thread: TMA loads of the f16 X' tile [BNT, 64] per MMA stage
//     (128-byte swizzle, the UMMA K-major layout) and, every 256 k, of the
//     packed W tile [128 rows, 128 B] (one full 128-byte line per row, so the
//     weight stream reaches DRAM as whole lines) with its scales [128, 16 B];
//   - warps 2..9 (two threads per weight row, 32 codes each): e2m1 x e4m3 ->
//     f16 into the swizzled A tile of each MMA stage;
//   - warp 1, one thread: tcgen05.mma into the TMEM accumulator [128, BNT],
//     committing each stage to its "empty" barrier;
//   - warps 2..17 (the dequant warps and eight that wait for the last MMA in
//     a named barrier) then read TMEM, apply g * 2^-e_m and store BF16 Y.
// Kernels are launched with programmatic dependent launch: with static
// weights the W tiles start streaming while the previous kernel (the X prep)
// is still running; X', e_m and Y are touched only after it completes.
// Every mbarrier wait is bounded.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "nvfp4_device.cuh"
#include "nvfp4_kernels.h"
#include "sm100_ptx.cuh"
#include "tc_host.h"

namespace nvfp4 {

// Number of CTAs whose pipeline wait ran past its time limit (diagnostic).
__device__ unsigned int g_gemm_wait_timeouts = 0;

namespace {

constexpr int kBM = 128;        // weight rows per tile (MMA M)
constexpr int kBK = 64;         // k per stage: one 128-byte swizzle row of f16
constexpr int kDeqWarp0 = 2;    // warps 2..9 dequantize, then run the epilogue
constexpr int kDeqWarps = 8;
constexpr int kEpiWarps = 16;   // warps 2..17 run the epilogue (10..17 only that)
constexpr int kThreads = (kDeqWarp0 + kEpiWarps) * 32;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr int kWideRow = -(1 << 30);  // row-info marker: recompute this row exactly

struct Bars {
  uint64_t deq[8];    // f16 A tile of the MMA stage written (256 arrivals)
  uint64_t empty[8];  // MMAs reading the A tile finished
  uint64_t xfull[8];  // X' slot landed
  uint64_t xempty[8]; // MMAs reading the X' slot finished
  uint64_t wfull[8];  // packed W and scales of the weight stage landed
  uint64_t wempty[8]; // dequant threads done with the weight stage (8 warp arrivals)
  uint64_t tmem_full; // last MMA finished
  uint32_t tmem_addr;
  volatile int err;
  int info[512];      // the tile's row exponents (or kWideRow), staged for the epilogue
  float colpow[512];  // 2^-e of each row (1 for wide rows)
};

template <int BN, int NSUB>
struct Cfg {
  static constexpr int kBNT = BN * NSUB;
  static constexpr int kXG = kBNT <= 64 ? 4 : 1;      // MMA stages per X' slot (small tiles: one per 256 k)
  static constexpr int kXSub = kBNT * 128;            // f16 X' tile of one MMA stage
  static constexpr int kXBytes = kXG * kXSub;         // one X' slot
  static constexpr int kABytes = kBM * 128;           // f16 A tile of one MMA stage
  static constexpr int kWBytes = kBM * 128;           // packed W of one weight stage (256 k)
  static constexpr int kSBytes = kBM * 16;            // its E4M3 scales
  // A tiles are produced on chip and X' comes from L2; the weights come from
  // HBM with microseconds of latency under load, so the shared memory left
  // after the A and X' rings goes to a deep weight ring.
  static constexpr int kBudget = 218 * 1024;
  static constexpr int kStages = kBNT >= 512 ? 3 : (kBNT >= 256 ? 2 : 3);  // A ring
  static constexpr int kXStages = kXG == 4 ? 3 : (kBNT >= 256 ? 2 : 3);  // X' ring
  static constexpr int kFixed = kStages * kABytes + kXStages * kXBytes;
  static constexpr int kWFit = (kBudget - kFixed) / (kWBytes + kSBytes);
  static constexpr int kWStages = kWFit > 8 ? 8 : kWFit;
  static constexpr int kWRing = kWStages * (kWBytes + kSBytes);
  static constexpr int kSmemBytes = kFixed + kWRing + (int)sizeof(Bars) + 1024;
  static constexpr uint32_t kTmemCols = kBNT < 32 ? 32 : kBNT;
  static constexpr uint32_t kIdesc = ptx::idesc_f16_f32(kBM, BN);
  static_assert(kWStages >= 2, "weight ring needs two stages");
  static_assert(BN % 16 == 0 && BN <= 256, "MMA N");
  static_assert(kBNT <= 512, "TMEM has 512 columns");
  static_assert(kEpiWarps * 2048 <= kStages * kABytes, "epilogue staging blocks fit in the A ring");
};

__device__ __forceinline__ bool wait_or_fail(uint64_t* bar, uint32_t parity, Bars* bars) {
  if (bars->err) return false;
  if (ptx::mbar_wait(bar, parity, kWaitLimitNs)) return true;
  if (!bars->err) {
    bars->err = 1;
    atomicAdd(&g_gemm_wait_timeouts, 1u);
  }
  return false;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ void st_shared_u16(uint32_t addr, uint16_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Eight E2M1 codes (one 32-bit word, low nibble first) times the block scale
// (f16x2 pair (s, s)) -> eight f16, exact.
__device__ __forceinline__ uint4 dequant8_f16(uint32_t word, uint32_t s2) {
  return make_uint4(hmul2(e2m1x2_byte_to_f16x2<0>(word), s2), hmul2(e2m1x2_byte_to_f16x2<1>(word), s2),
                    hmul2(e2m1x2_byte_to_f16x2<2>(word), s2), hmul2(e2m1x2_byte_to_f16x2<3>(word), s2));
}

// OR of `v` over the `count` threads that meet at named barrier `id` (a
// barrier: shared-memory writes before it are visible to all after it).
__device__ __forceinline__ bool group_any(int id, int count, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// 2^k as fp32 for k in [-149, 127] (subnormal below -126).
__device__ __forceinline__ float pow2f(int k) {
  return k >= -126 ? __uint_as_float((uint32_t)(k + 127) << 23) : __uint_as_float(1u << (k + 149));
}

// Exact fp32 dot product of weight row n (all K) with BF16 activation row xr,
// over the k range [k0, k1) (multiples of 32).
__device__ float exact_row_dot(const uint8_t* __restrict__ q, const uint8_t* __restrict__ s, int64_t n, int K,
                               const uint16_t* __restrict__ xr, int k0, int k1) {
  const uint8_t* qr = q + n * (K / 2);
  const uint8_t* sr = s + n * (K / 16);
  float acc = 0.0f;
  for (int k = k0; k < k1; k += 32) {
    const uint4 w = *reinterpret_cast<const uint4*>(qr + k / 2);
    const uint32_t words[4] = {w.x, w.y, w.z, w.w};
    const float2 sc = f16x2_to_float2(e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(sr + k / 16)));
    float2 p[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
      const uint4 xv = *reinterpret_cast<const uint4*>(xr + k + 8 * wi);
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
    acc = fmaf(p[0].x + p[0].y, sc.x, acc);
    acc = fmaf(p[1].x + p[1].y, sc.y, acc);
  }
  return acc;
}

// ----------------------------------------------------------------- X prep

// One CTA of 128 threads per row m: range of |X[m, :]|, exponent e_m with
// max |x| * 2^e_m in [2^15, 2^16), and X'[m, :] = f16(X[m, :] * 2^e_m).
// info[m] = e_m, or kWideRow when the row is not finite or its non-zero
// magnitudes span more than 2^32 (then X' is not exact and the GEMM recomputes
// the row on CUDA cores).
constexpr int kPrepThreads = 256;
constexpr int kPrepPer = 8;  // 16-byte vectors per thread held in registers (K <= 256 * 8 * 8 = 16384)

// Row m of X: range of |x| and X'[m, :] = f16(X[m, :] * 2^e_m).  For K <= 16384
// every thread issues all of its loads at once and keeps the values in
// registers for the conversion (one memory round trip); longer rows read X
// twice.
__global__ void __launch_bounds__(kPrepThreads) prep_x_kernel(const uint16_t* __restrict__ X, int64_t ldx, int K,
                                                              int* __restrict__ info, uint16_t* __restrict__ Xh) {
  __shared__ uint32_t red_max[kPrepThreads / 32], red_min[kPrepThreads / 32];
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int m = blockIdx.x;
  const uint16_t* xr = X + (int64_t)m * ldx;
  uint16_t* hr = Xh + (int64_t)m * K;
  const int nv = K / 8;
  const bool in_regs = nv <= kPrepThreads * kPrepPer;
  uint4 v[kPrepPer];
  uint32_t mx = 0, mn = 0xFFFFu;
  auto scan = [&](const uint4& x4) {
    const uint32_t w4[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t lo = w4[j] & 0x7FFFu, hi = (w4[j] >> 16) & 0x7FFFu;
      mx = max(mx, max(lo, hi));
      mn = min(mn, min(lo ? lo : 0xFFFFu, hi ? hi : 0xFFFFu));
    }
  };
  if (in_regs) {
#pragma unroll
    for (int k = 0; k < kPrepPer; ++k) {
      const int i = threadIdx.x + k * kPrepThreads;
      v[k] = i < nv ? *reinterpret_cast<const uint4*>(xr + 8 * i) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int k = 0; k < kPrepPer; ++k) scan(v[k]);
  } else {
    for (int i = threadIdx.x; i < nv; i += kPrepThreads) scan(*reinterpret_cast<const uint4*>(xr + 8 * i));
  }
  mx = __reduce_max_sync(0xFFFFFFFFu, mx);
  mn = __reduce_min_sync(0xFFFFFFFFu, mn);
  if ((threadIdx.x & 31) == 0) {
    red_max[threadIdx.x >> 5] = mx;
    red_min[threadIdx.x >> 5] = mn;
  }
  __syncthreads();
  mx = red_max[0];
  mn = red_min[0];
#pragma unroll
  for (int w = 1; w < kPrepThreads / 32; ++w) {
    mx = max(mx, red_max[w]);
    mn = min(mn, red_min[w]);
  }
  int e = 0;
  bool wide = false;
  if (mx >= 0x7F80u) {
    wide = true;
  } else if (mx != 0) {
    const int hi_exp = bf16_ilogb(mx), lo_exp = bf16_ilogb(mn);
    e = 15 - hi_exp;
    wide = hi_exp - lo_exp > 32;
  }
  const int e1 = e / 2, e2 = e - e1;
  const float m1 = exp2i(e1), m2 = exp2i(e2);
  auto convert = [&](const uint4& x4) {
    const uint32_t w4[4] = {x4.x, x4.y, x4.z, x4.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __half2 h = __floats2half2_rn(bf16lo_to_float(w4[j]) * m1 * m2, bf16hi_to_float(w4[j]) * m1 * m2);
      o[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
  };
  if (in_regs) {
#pragma unroll
    for (int k = 0; k < kPrepPer; ++k) {
      const int i = threadIdx.x + k * kPrepThreads;
      if (i < nv) *reinterpret_cast<uint4*>(hr + 8 * i) = convert(v[k]);
    }
  } else {
    for (int i = threadIdx.x; i < nv; i += kPrepThreads)
      *reinterpret_cast<uint4*>(hr + 8 * i) = convert(*reinterpret_cast<const uint4*>(xr + 8 * i));
  }
  if (threadIdx.x == 0) info[m] = wide ? kWideRow : e;
}

// ----------------------------------------------------------------- GEMM

template <int BN, int NSUB>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                   const __grid_constant__ CUtensorMap tmap_s, const uint8_t* __restrict__ q,
                   const uint8_t* __restrict__ s, const float* __restrict__ g, const int* __restrict__ info,
                   const uint16_t* __restrict__ X, int64_t ldx, uint16_t* __restrict__ Y, int64_t ldy, int M, int N,
                   int K, int static_weights) {
  using C = Cfg<BN, NSUB>;
  constexpr int NS = C::kStages;
  constexpr int NX = C::kXStages;
  constexpr int XG = C::kXG;
  constexpr int NW = C::kWStages;
  constexpr int BNT = C::kBNT;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  // layout: [NS A tiles] [NX X' slots] [NW W tiles] [NW scale tiles] [barriers]
  auto a_tile = [&](int st) { return smem + st * C::kABytes; };
  auto x_slot = [&](int xs) { return smem + NS * C::kABytes + xs * C::kXBytes; };
  auto w_tile = [&](int ws) { return smem + C::kFixed + ws * C::kWBytes; };
  auto s_tile = [&](int ws) { return smem + C::kFixed + NW * C::kWBytes + ws * C::kSBytes; };
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kFixed + C::kWRing);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kBM, m0 = blockIdx.y * BNT;
  const int num_kb = K / kBK;        // MMA stages (64 k)
  const int num_wb = num_kb / 4;     // weight stages (256 k)
  const int num_xb = num_kb / XG;    // X' slots

  if (threadIdx.x == 0) {
    for (int st = 0; st < NS; ++st) {
      ptx::mbar_init(&bars->deq[st], kDeqWarps * 32);
      ptx::mbar_init(&bars->empty[st], 1);
    }
    for (int xs = 0; xs < NX; ++xs) {
      ptx::mbar_init(&bars->xfull[xs], 1);
      ptx::mbar_init(&bars->xempty[xs], 1);
    }
    for (int ws = 0; ws < NW; ++ws) {
      ptx::mbar_init(&bars->wfull[ws], 1);
      ptx::mbar_init(&bars->wempty[ws], kDeqWarps);
    }
    ptx::mbar_init(&bars->tmem_full, 1);
    bars->err = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tmap_x);
    ptx::prefetch_tmap(&tmap_w);
    ptx::prefetch_tmap(&tmap_s);
  }
  if (warp == 1) {
    ptx::tmem_alloc(&bars->tmem_addr, C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_addr;

  // Programmatic dependent launch: the next kernel may start its prologue; the
  // weights may be read before the previous kernel finishes only if static.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (!static_weights) asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      auto issue_w = [&](int wb) {
        const int ws = wb % NW;
        ptx::mbar_arrive_expect_tx(&bars->wfull[ws], C::kWBytes + C::kSBytes);
        ptx::tma_load_2d(w_tile(ws), &tmap_w, &bars->wfull[ws], wb * 128, n0);
        ptx::tma_load_2d(s_tile(ws), &tmap_s, &bars->wfull[ws], wb * 16, n0);
      };
      auto issue_x = [&](int xb) {
        const int xs = xb % NX;
        ptx::mbar_arrive_expect_tx(&bars->xfull[xs], C::kXBytes);
#pragma unroll
        for (int i = 0; i < XG; ++i)
#pragma unroll
          for (int h = 0; h < (BNT + 255) / 256; ++h)
            ptx::tma_load_2d(x_slot(xs) + i * C::kXSub + h * 256 * 128, &tmap_x, &bars->xfull[xs],
                             (xb * XG + i) * kBK, m0 + h * 256);
      };
      // weight stages that need no slot release go out before the X prep ends
      const int w_first = num_wb < NW ? num_wb : NW;
      for (int wb = 0; wb < w_first; ++wb) issue_w(wb);
      if (static_weights) asm volatile("griddepcontrol.wait;" ::: "memory");
      int next_wb = w_first, next_xb = 0;
      for (int kb = 0; kb < num_kb && !bars->err; ++kb) {
        // weights: keep the ring NW - 1 weight stages ahead of this MMA stage
        while (next_wb < num_wb && next_wb <= kb / 4 + NW - 1) {
          if (!wait_or_fail(&bars->wempty[next_wb % NW], ((next_wb / NW) - 1) & 1, bars)) break;
          issue_w(next_wb);
          ++next_wb;
        }
        // X': the slot holding this MMA stage, and up to NX - 1 slots ahead
        while (!bars->err && next_xb < num_xb && next_xb <= kb / XG + NX - 1) {
          if (next_xb >= NX && !wait_or_fail(&bars->xempty[next_xb % NX], ((next_xb / NX) - 1) & 1, bars)) break;
          issue_x(next_xb);
          ++next_xb;
        }
      }
      if (bars->err) {
        // let copies already issued land before the CTA exits
        for (int xb = next_xb > NX ? next_xb - NX : 0; xb < next_xb; ++xb)
          ptx::mbar_wait(&bars->xfull[xb % NX], (xb / NX) & 1, kWaitLimitNs);
        for (int wb = next_wb > NW ? next_wb - NW : 0; wb < next_wb; ++wb)
          ptx::mbar_wait(&bars->wfull[wb % NW], (wb / NW) & 1, kWaitLimitNs);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      for (int kb = 0; kb < num_kb; ++kb) {
        const int st = kb % NS, round = kb / NS;
        const int xb = kb / XG, xs = xb % NX, xi = kb % XG;
        if (!wait_or_fail(&bars->deq[st], round & 1, bars)) break;
        if (xi == 0 && !wait_or_fail(&bars->xfull[xs], (xb / NX) & 1, bars)) break;
        ptx::tc_fence_after();
        const uint32_t a0 = ptx::smem_u32(a_tile(st));
        const uint32_t b0 = ptx::smem_u32(x_slot(xs)) + (uint32_t)(xi * C::kXSub);
#pragma unroll
        for (int j = 0; j < kBK / 16; ++j) {
#pragma unroll
          for (int sub = 0; sub < NSUB; ++sub)
            ptx::mma_f16(tmem + (uint32_t)(sub * BN), ptx::sw128_kmajor_desc(a0 + 32 * j),
                         ptx::sw128_kmajor_desc(b0 + sub * BN * 128 + 32 * j), C::kIdesc, (kb | j) != 0);
        }
        ptx::mma_commit(&bars->empty[st]);
        if (xi == XG - 1) ptx::mma_commit(&bars->xempty[xs]);
      }
      // arrives when every MMA above is done (also on the error path, so that
      // TMEM is never freed under a running MMA)
      ptx::mma_commit(&bars->tmem_full);
      if (bars->err) ptx::mbar_wait(&bars->tmem_full, 0, kWaitLimitNs);
    }
  } else {
    // Epilogue of warp `warp` (any of the kEpiWarps): TMEM lane
    // (32 * (warp % 4) + lane) holds weight row n; columns are m.  The warps
    // of a lane quarter split the columns (when there are enough); each
    // 32 x 32 block goes through 2 KB of the (now idle) A ring, so that Y is
    // written as 64-byte row segments with 16-byte stores.
    auto epilogue = [&]() {
      if (!__all_sync(0xFFFFFFFFu, wait_or_fail(&bars->tmem_full, 0, bars))) return;
      ptx::tc_fence_after();
      const int quarter = warp & 3;
      const float gv = *g;
      constexpr int kParts = BNT >= 128 ? kEpiWarps / 4 : (BNT >= 64 ? 2 : 1);
      constexpr int kColsPerWarp = BNT / kParts;
      const int part = (warp - kDeqWarp0) >> 2;
      if (part >= kParts) return;
      const int c_begin = part * kColsPerWarp;
      const uint32_t stage = ptx::smem_u32(a_tile(0)) + (uint32_t)(warp - kDeqWarp0) * 2048u;
      const bool vec_ok = ((reinterpret_cast<uintptr_t>(Y) & 15u) == 0) && (ldy % 8 == 0);
#pragma unroll 1
      for (int c0 = c_begin; c0 < c_begin + kColsPerWarp; c0 += 32) {
        uint32_t rr[32];
        ptx::tmem_ld_32cols(tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)c0, rr);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const __nv_bfloat16 o = __float2bfloat16_rn((__uint_as_float(rr[j]) * gv) * bars->colpow[c0 + j]);
          st_shared_u16(stage + (uint32_t)(j * 32 + lane) * 2u, *reinterpret_cast<const uint16_t*>(&o));
        }
        __syncwarp();
        // row j of the block: 32 consecutive n = 64 bytes, four lanes per row
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int p = 32 * k + lane, j = p >> 2, piece = p & 3;
          const int m = m0 + c0 + j;
          const int nb = n0 + 32 * quarter + 8 * piece;
          if (c0 + j < c_begin + kColsPerWarp && m < M && bars->info[c0 + j] != kWideRow && nb < N) {
            const uint4 v = ld_shared_v4(stage + (uint32_t)(j * 32 + 8 * piece) * 2u);
            uint16_t* dst = Y + (int64_t)m * ldy + nb;
            if (vec_ok && nb + 8 <= N) {
              *reinterpret_cast<uint4*>(dst) = v;
            } else {
              const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
              for (int i = 0; i < 8 && nb + i < N; ++i) dst[i] = (uint16_t)(w4[i >> 1] >> (16 * (i & 1)));
            }
          }
        }
        __syncwarp();
      }
    };
    if (warp >= kDeqWarp0 + kDeqWarps) {
      // ------------------------------------------------ epilogue only
      if (static_weights) asm volatile("griddepcontrol.wait;" ::: "memory");  // Y
      // wait (in the barrier, not polling) until the dequantization warps have
      // staged the tile's row info, after their last stage
      group_any(1, kEpiWarps * 32, false);
      epilogue();
    } else {
    // ------------------------------------------------ dequantize, then epilogue
    const int t = threadIdx.x - kDeqWarp0 * 32;  // 0..255
    const int r = t >> 1, h = t & 1;              // weight row in the tile, half of each 64 k
    const int row = n0 + r;
    const bool row_ok = row < N;
    const uint32_t swz = (uint32_t)(r & 7);
    bool ok = true;
    for (int wb = 0; wb < num_wb && ok; ++wb) {
      const int ws = wb % NW;
      if (!wait_or_fail(&bars->wfull[ws], (wb / NW) & 1, bars)) break;
      // this row's 128 packed bytes (16-byte chunks stored at chunk ^ (row % 8)) and 16 scale bytes
      const uint32_t wrow = ptx::smem_u32(w_tile(ws)) + r * 128;
      const uint4 sc16 = ld_shared_v4(ptx::smem_u32(s_tile(ws)) + r * 16);
      const uint32_t scw[4] = {sc16.x, sc16.y, sc16.z, sc16.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int kb = wb * 4 + i;
        const int st = kb % NS, round = kb / NS;
        // the A tile of this stage is free once the MMAs of its previous use finished
        if (round > 0 && !wait_or_fail(&bars->empty[st], (round - 1) & 1, bars)) {
          ok = false;
          break;
        }
        const uint4 c = ld_shared_v4(wrow + ((((uint32_t)(2 * i + h)) ^ swz) << 4));
        const uint32_t sc2 = (scw[i] >> (16 * h)) & 0xFFFFu;  // blocks 2h, 2h+1 of this stage
        const uint32_t s01 = e4m3x2_to_f16x2(sc2);             // (s0, s1) as f16
        const uint32_t s0 = __byte_perm(s01, 0, 0x1010);      // (s0, s0)
        const uint32_t s1 = __byte_perm(s01, 0, 0x3232);      // (s1, s1)
        const uint32_t dst = ptx::smem_u32(a_tile(st)) + r * 128;
        const uint32_t cb = (uint32_t)(4 * h);                 // first 16-byte chunk of this half
        st_shared_v4(dst + (((cb + 0) ^ swz) << 4), dequant8_f16(c.x, s0));
        st_shared_v4(dst + (((cb + 1) ^ swz) << 4), dequant8_f16(c.y, s0));
        st_shared_v4(dst + (((cb + 2) ^ swz) << 4), dequant8_f16(c.z, s1));
        st_shared_v4(dst + (((cb + 3) ^ swz) << 4), dequant8_f16(c.w, s1));
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(&bars->deq[st]);
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bars->wempty[ws]);
    }
    if (static_weights) asm volatile("griddepcontrol.wait;" ::: "memory");  // info and Y
    // stage the tile's row info once (the epilogue reads it per element) and
    // find out whether any row needs the exact recompute
    bool wide_here = false;
    for (int i = t; i < BNT; i += kDeqWarps * 32) {
      const int e = m0 + i < M ? __ldg(info + m0 + i) : 0;
      bars->info[i] = e;
      bars->colpow[i] = e == kWideRow ? 1.0f : pow2f(-e);
      wide_here |= e == kWideRow;
    }
    const bool any_wide = group_any(1, kEpiWarps * 32, wide_here);
    epilogue();
    // rows of X outside the exact f16 window: exact fp32 dot on CUDA cores,
    // two threads per weight row (halves of K), combined with one shuffle
    const float gv = *g;
    for (int mi = 0; mi < BNT && any_wide; ++mi) {
      const int m = m0 + mi;
      if (m >= M) break;
      if (bars->info[mi] != kWideRow) continue;
      float part = 0.0f;
      if (row_ok) part = exact_row_dot(q, s, row, K, X + (int64_t)m * ldx, h * (K / 2), (h + 1) * (K / 2));
      part += __shfl_xor_sync(0xFFFFFFFFu, part, 1);
      if (row_ok && h == 0) {
        const __nv_bfloat16 o = __float2bfloat16_rn(part * gv);
        Y[(int64_t)m * ldy + row] = *reinterpret_cast<const uint16_t*>(&o);
      }
    }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int BN, int NSUB>
cudaError_t launch_cfg(const uint16_t* X, int64_t ldx, const uint8_t* q, const uint8_t* s, const float* g,
                       uint16_t* Y, int64_t ldy, int M, int N, int K, const int* info, const uint16_t* Xh,
                       bool static_weights, cudaStream_t stream) {
  using C = Cfg<BN, NSUB>;
  auto enc = tc::encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap tx, tw, ts;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)(C::kBNT < 256 ? C::kBNT : 256)};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t*>(Xh), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)N};
    const cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    const cuuint32_t box[2] = {128u, (cuuint32_t)kBM};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(q), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)(K / 16), (cuuint64_t)N};
    const cuuint64_t strides[1] = {(cuuint64_t)(K / 16)};
    const cuuint32_t box[2] = {16u, (cuuint32_t)kBM};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&ts, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(s), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  static tc::SmemOptIn opt_in;
  const cudaError_t e = opt_in.ensure((const void*)gemm_tc_kernel<BN, NSUB>, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  int sw = static_weights ? 1 : 0;
  void* args[] = {&tx, &tw, &ts, (void*)&q, (void*)&s, (void*)&g, (void*)&info, (void*)&X, &ldx, &Y, &ldy,
                  &M, &N, &K, &sw};
  dim3 grid((N + kBM - 1) / kBM, (M + C::kBNT - 1) / C::kBNT);
  return tc::launch_pdl((const void*)gemm_tc_kernel<BN, NSUB>, grid, dim3(kThreads), C::kSmemBytes, stream, args);
}

size_t align16(size_t v) { return (v + 15) & ~(size_t)15; }

}  // namespace

bool gemm_tc_supported(int64_t M, int64_t N, int64_t K) {
  return M >= 2 && N >= 1 && K % 256 == 0 && K <= (int64_t)1 << 24 && N <= ((int64_t)1 << 31) - 128 &&
         M <= ((int64_t)1 << 31) - 512;
}

size_t gemm_prep_workspace_bytes(int64_t M, int64_t K) { return align16((size_t)M * 4) + (size_t)M * K * 2; }

size_t gemm_tc_workspace_bytes(int64_t M, int64_t K) { return gemm_prep_workspace_bytes(M, K); }

cudaError_t launch_gemm_prep(const uint16_t* X, int64_t ldx, int64_t M, int64_t K, void* workspace, int** info_out,
                             uint16_t** xh_out, cudaStream_t stream) {
  int* info = reinterpret_cast<int*>(workspace);
  uint16_t* Xh = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(workspace) + align16((size_t)M * 4));
  *info_out = info;
  *xh_out = Xh;
  const uint16_t* xp = X;
  int kk = (int)K;
  void* args[] = {(void*)&xp, &ldx, &kk, (void*)&info, (void*)&Xh};
  return tc::launch_pdl((const void*)prep_x_kernel, dim3((unsigned)M), dim3(kPrepThreads), 0, stream, args);
}

cudaError_t launch_gemm_tc(const uint16_t* X, int64_t ldx, const uint8_t* q, const uint8_t* s, const float* g,
                           uint16_t* Y, int64_t ldy, int64_t M, int64_t N, int64_t K, void* workspace,
                           bool static_weights, cudaStream_t stream) {
  int* info = nullptr;
  uint16_t* Xh = nullptr;
  {
    cudaError_t e = launch_gemm_prep(X, ldx, M, K, workspace, &info, &Xh, stream);
    if (e != cudaSuccess) return e;
  }
  const int m = (int)M, n = (int)N, k = (int)K;
  if (M <= 16) return launch_cfg<16, 1>(X, ldx, q, s, g, Y, ldy, m, n, k, info, Xh, static_weights, stream);
  if (M <= 32) return launch_cfg<32, 1>(X, ldx, q, s, g, Y, ldy, m, n, k, info, Xh, static_weights, stream);
  if (M <= 64) return launch_cfg<64, 1>(X, ldx, q, s, g, Y, ldy, m, n, k, info, Xh, static_weights, stream);
  if (M <= 128) return launch_cfg<128, 1>(X, ldx, q, s, g, Y, ldy, m, n, k, info, Xh, static_weights, stream);
  if (M <= 256) return launch_cfg<256, 1>(X, ldx, q, s, g, Y, ldy, m, n, k, info, Xh, static_weights, stream);
  return launch_cfg<256, 2>(X, ldx, q, s, g, Y, ldy, m, n, k, info, Xh, static_weights, stream);
}

cudaError_t read_and_clear_gemm_timeouts(unsigned int* count) {
  cudaError_t e = cudaMemcpyFromSymbol(count, g_gemm_wait_timeouts, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  const unsigned int zero = 0;
  return cudaMemcpyToSymbol(g_gemm_wait_timeouts, &zero, sizeof(unsigned int));
}

}  // namespace nvfp4

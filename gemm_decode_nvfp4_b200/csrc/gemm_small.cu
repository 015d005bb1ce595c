// gemm_small.cu -- NVFP4 W4A16 decode GEMV and small-M GEMM (M <= 64) on the
// sm_100a tensor cores, with the dequantized weights held in tensor memory.
//
// Y[m, n] = bf16(g * sum_k W_deq[n, k] * X[m, k]) for batch-1 decode (M = 1)
// and batched decode (the 32-user GEMM of the model card "Qwen3.8-27B-NVFP4",
// "Measurements"); imp docs/quantization.md, "Dense layers" pipeline: the
// decode path reads the packed NVFP4 weights directly.  Weight-only ("What is
// quantized"): X stays 16-bit.
//
// At these M the layer is a stream of weight bytes (about 0.56 byte per
// weight) and the work per weight is the dequantization, so the kernel is
// built to keep HBM busy and to spend as few instructions per weight as
// possible:
//   - one CTA per 128 weight rows (MMA M = 128; the weights are operand A, the
//     activations operand B with N = 16, 32 or 64 rows, "swap AB");
//   - warp 0 streams the packed weights and their scales with TMA in stages of
//     256 k (one 128-byte line per row, 128-byte swizzle) into a deep ring;
//   - 16 dequantization warps in four groups: group j takes the 128-k stages
//     j mod 4 (halves of weight stages) and turns them into exact f16 values e2m1 * e4m3 (one
//     cvt.rn.f16x2.e2m1x2 and one f16x2 multiply per two weights), stored with
//     tcgen05.st straight into a ring of A stages in tensor memory (no shared
//     memory traffic for the 2-byte weights), so four stages are dequantized
//     at once;
//   - four MMA warps, issuer j for the stages of group j: an MMA instruction
//     costs its issuing warp tens of cycles at these N, and every barrier
//     wait in that warp as much again, so each issuer handles whole 128-k
//     stages (8 MMAs per wait) with A read from tensor memory and B (f16
//     activations, K-major, 128-byte swizzle) from shared memory, into its own
//     fp32 accumulator in tensor memory; the epilogue sums the four;
//   - the activations reach shared memory as exact f16 values X * 2^e_m
//     (e_m per row, chosen from its max |x|): for M <= 8 each dequantization
//     group converts the activations of its own stages (no workspace, no extra
//     launch); for larger M a pre-pass kernel writes the f16 copy into the
//     workspace and TMA loads it;
//   - the epilogue reads the accumulator (tcgen05.ld), applies g * 2^-e_m and
//     stores BF16; rows of X whose non-zero magnitudes span more than 2^32
//     (where X * 2^e_m is not exact in f16) are recomputed exactly in fp32 on
//     CUDA cores.
// Every product is exact and sums are fp32, so the result equals the exact
// dot product up to fp32 summation order.  Every wait is bounded in time.
#include "nvfp4_device.cuh"
#include "nvfp4_kernels.h"
#include "sm100_ptx.cuh"
#include "tc_host.h"

namespace nvfp4 {

// CTAs of this kernel whose pipeline wait ran past its time limit (diagnostic).
__device__ unsigned int g_small_wait_timeouts = 0;

namespace {

constexpr int kBM = 128;        // weight rows per CTA (MMA M)
constexpr int kBK = 64;         // k per A tile (one 128-byte row of f16)
constexpr int kWK = 256;        // k per weight stage (one 128-byte line of codes per row)
// Warp roles: producer, four MMA issuers (a lone thread issues one MMA about
// every 56 cycles at these N, while the tensor pipe needs 16 for an N = 32
// MMA, so one issuer per dequantization group keeps it supplied), converter,
// 16 dequantizers.
constexpr int kProdWarp = 0, kMmaWarp0 = 1, kMmaWarps = 4, kConvWarp = 5, kDeqWarp0 = 6, kDeqWarps = 16;
// M > 8: one f16-activation producer warp per MMA issuer, so that each
// issuer's activation tiles are refilled as soon as its own MMAs release them
// (a single producer serving the four issuers in order made every issuer wait
// for the slowest one).
constexpr int kXWarp0 = kDeqWarp0 + kDeqWarps, kXWarps = kMmaWarps;
constexpr int kMmaWarp = kMmaWarp0;  // also allocates and frees tensor memory
constexpr int kThreads = (kXWarp0 + kXWarps) * 32;
constexpr int kScanThreads = (1 + kDeqWarps) * 32;  // converter + dequant warps (range scan)
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr int kWideRow = -(1 << 30);
constexpr uint32_t kTmemCols = 512;
constexpr int kConvMaxM = 8;
constexpr int kEpiBar = 2;       // named barrier of the 16 dequantization warps (1 is the range scan)

struct SmallBars {
  uint64_t wfull[16], wempty[16];  // weight stage landed / read by the 16 dequant warps
  uint64_t afull[16], aempty[16];  // A sub-slot (group g, slot i at 3g+i) written (128 threads) / read
  uint64_t xfull[16], xempty[16];  // f16 B tile ready / read by its MMAs (xempty: M <= 8 path)
  // M > 8: the MMAs of group g's k-th 128-k half stage finished (at 4g + k % 4);
  // frees its two A sub-slots and its B slot with one commit
  uint64_t hdone[16];
  uint64_t tmem_full;              // every issuer's last MMA finished (4 arrivals)
  uint32_t tmem_addr;
  volatile int err;
  uint32_t xmax[kConvMaxM], xmin[kConvMaxM];  // per-row |x| range as BF16 bits (M <= 8 path)
  int info[64];                    // the tile's row exponents (or kWideRow), staged for the epilogue
};

template <int BNT, bool CONV>
struct SmallCfg {
  // f16 B stage: 128 k as two 64-k tiles of BNT rows x 128 B (8 rows, 1 KB,
  // on the M <= 8 path), each a K-major tile with the 128-byte swizzle.  Ring
  // sizes are multiples of 4 so that every slot is always used by the same
  // dequantization group / MMA issuer (the parity waits of a ring are only
  // exact for a consumer that sees every phase of its slot).
  // On the M <= 8 path each dequantization group converts its own B tiles,
  // one per A sub-slot (released together with it).
  // On the M > 8 path every issuer owns the slots h % kNX of its half
  // stages h (kNX / 4 of them): 4, 3 and 2 per issuer for N = 16, 32, 64,
  // enough that a slot's reload (MMA completion, then an L2 round trip) runs
  // behind the issuer's MMAs on its other slots.
  static constexpr int kXTile = CONV ? 1024 : BNT * 128;
  static constexpr int kXSlot = CONV ? kXTile : 2 * kXTile;
  static constexpr int kNX = CONV ? 4 * (BNT <= 32 ? 3 : 2) : (BNT <= 16 ? 16 : BNT <= 32 ? 12 : 8);
  // +1024: the MMA reads B rows 8..15 one 1024-byte atom past each 8-row tile
  // of the M <= 8 path (those output columns are discarded)
  static constexpr int kXRing = kNX * kXSlot + 1024;
  static constexpr int kWQ = kBM * 128, kWS = kBM * 16, kWStage = kWQ + kWS;
  static constexpr int kBudget = 218 * 1024;
  static constexpr int kWFit = (kBudget - kXRing) / kWStage;
  static constexpr int kNW = (kWFit > 12 ? 12 : kWFit) / 2 * 2;
  // one fp32 accumulator per MMA issuer (summed in the epilogue), then a ring
  // of kNS A sub-slots (64 k of f16 weights = 32 TMEM columns) per
  // dequantization group, so that a group dequantizes the next half stage
  // while the MMAs read the previous one
  static constexpr int kNAcc = kMmaWarps;
  static constexpr int kABase = kNAcc * BNT < 32 ? 32 : kNAcc * BNT;
  static constexpr int kNS = BNT <= 32 ? 3 : 2;
  static constexpr int kNA = 4 * kNS;
  static constexpr int kSmem = 1024 + kXRing + kNW * kWStage + (int)sizeof(SmallBars);
  static constexpr uint32_t kIdesc = ptx::idesc_f16_f32(kBM, BNT);
  static_assert(BNT % 16 == 0 && BNT >= 16 && BNT <= 64, "MMA N");
  static_assert(!CONV || BNT == 16, "the converted path covers M <= 8");
  static_assert(kNW >= 4 && kNW <= 16 && kNX <= 16, "rings");
  // a weight stage is read by the groups of its two halves ({0, 1} for even
  // stages, {2, 3} for odd ones): an even ring keeps each slot with one pair;
  // an activation slot h % kNX belongs to issuer h % 4
  static_assert(kNW % 2 == 0 && kNX % 4 == 0, "slots owned by one group");
  static_assert(kABase % 32 == 0 && kABase + 32 * kNA <= (int)kTmemCols, "TMEM columns");
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ bool wait_or_fail(uint64_t* bar, uint32_t parity, SmallBars* bars) {
  if (bars->err) return false;
  if (ptx::mbar_wait(bar, parity, kWaitLimitNs)) return true;
  if (!bars->err) {
    bars->err = 1;
    atomicAdd(&g_small_wait_timeouts, 1u);
  }
  return false;
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

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Eight codes of `word` (low nibble first) times the block scale pair (s, s):
// four f16x2 words in k order, exact.
__device__ __forceinline__ void dequant8(uint32_t word, uint32_t s2, uint32_t* o) {
  o[0] = hmul2(e2m1x2_byte_to_f16x2<0>(word), s2);
  o[1] = hmul2(e2m1x2_byte_to_f16x2<1>(word), s2);
  o[2] = hmul2(e2m1x2_byte_to_f16x2<2>(word), s2);
  o[3] = hmul2(e2m1x2_byte_to_f16x2<3>(word), s2);
}

// 2^k as fp32 for k in [-149, 127].
__device__ __forceinline__ float pow2f(int k) {
  return k >= -126 ? __uint_as_float((uint32_t)(k + 127) << 23) : __uint_as_float(1u << (k + 149));
}

// Row exponent from the |x| range (BF16 bit patterns without sign): e with
// max |x| * 2^e in [2^15, 2^16), or kWideRow when the row is not finite or its
// non-zero magnitudes span more than 2^32.
__device__ __forceinline__ int row_exponent(uint32_t mx, uint32_t mn) {
  if (mx >= 0x7F80u) return kWideRow;
  if (mx == 0) return 0;
  const int hi = bf16_ilogb(mx), lo = bf16_ilogb(mn);
  return hi - lo > 32 ? kWideRow : 15 - hi;
}

// Eight BF16 values times 2^e (split in two factors so that each stays a
// normal fp32) rounded to f16; exact when the row is not wide.
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 v, float m1, float m2) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __half2 h = __floats2half2_rn(bf16lo_to_float(w[j]) * m1 * m2, bf16hi_to_float(w[j]) * m1 * m2);
    o[j] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Exact fp32 dot product of weight row n with BF16 activations xr over
// k in [k0, k1) (multiples of 32).
__device__ float exact_dot(const uint8_t* __restrict__ q, const uint8_t* __restrict__ s, int64_t n, int K,
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

template <int BNT, bool CONV>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_small_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_s,
                      const __grid_constant__ CUtensorMap tmap_x, const uint8_t* __restrict__ q,
                      const uint8_t* __restrict__ s, const float* __restrict__ g, const int* __restrict__ info,
                      const uint16_t* __restrict__ X, int64_t ldx, uint16_t* __restrict__ Y, int64_t ldy, int M,
                      int N, int K, int static_weights) {
  using C = SmallCfg<BNT, CONV>;
  constexpr int NW = C::kNW, NA = C::kNA, NX = C::kNX;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  // layout: [f16 B ring + 1 KB] [NW code tiles] [NW scale tiles] [barriers]
  uint8_t* const xring = smem;
  uint8_t* const wq = smem + C::kXRing;
  uint8_t* const wsc = wq + NW * C::kWQ;
  SmallBars* bars = reinterpret_cast<SmallBars*>(wsc + NW * C::kWS);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kBM, m0 = blockIdx.y * BNT;
  const int num_kb = K / kBK, num_wb = K / kWK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NW; ++i) {
      ptx::mbar_init(&bars->wfull[i], 1);
      ptx::mbar_init(&bars->wempty[i], 8);  // the two groups that read halves of the stage
    }
    for (int i = 0; i < NA; ++i) {
      ptx::mbar_init(&bars->afull[i], 128);
      ptx::mbar_init(&bars->aempty[i], 1);
    }
    for (int i = 0; i < NX; ++i) {
      ptx::mbar_init(&bars->xfull[i], CONV ? 32 : 1);
      ptx::mbar_init(&bars->xempty[i], 1);
    }
    for (int i = 0; i < 16; ++i) ptx::mbar_init(&bars->hdone[i], 1);
    ptx::mbar_init(&bars->tmem_full, kMmaWarps);
    for (int i = 0; i < kConvMaxM; ++i) {
      bars->xmax[i] = 0;
      bars->xmin[i] = 0xFFFFu;
    }
    bars->err = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kProdWarp && lane == 0) {
    ptx::prefetch_tmap(&tmap_w);
    ptx::prefetch_tmap(&tmap_s);
    ptx::prefetch_tmap(&tmap_x);
  }
  if (warp == kMmaWarp) {
    ptx::tmem_alloc(&bars->tmem_addr, kTmemCols);
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

  if (warp == kProdWarp) {
    // ------------------------------------------------ weight producer (TMA)
    if (lane == 0) {
      int nw = 0;
      for (; nw < num_wb; ++nw) {
        const int st = nw % NW;
        if (nw >= NW && !wait_or_fail(&bars->wempty[st], ((nw / NW) - 1) & 1, bars)) break;
        ptx::mbar_arrive_expect_tx(&bars->wfull[st], C::kWStage);
        ptx::tma_load_2d(wq + st * C::kWQ, &tmap_w, &bars->wfull[st], nw * 128, n0);
        ptx::tma_load_2d(wsc + st * C::kWS, &tmap_s, &bars->wfull[st], nw * 16, n0);
      }
      if (bars->err) {
        // let the copies already issued land before the CTA exits
        for (int wb = nw > NW ? nw - NW : 0; wb < nw; ++wb)
          ptx::mbar_wait(&bars->wfull[wb % NW], (wb / NW) & 1, kWaitLimitNs);
      }
    }
  } else if (warp < kMmaWarp0 + kMmaWarps) {
    // ------------------------ MMA issuers: issuer g takes the 128-k stages h = g mod 4
    if (lane == 0) {
      const int gi = warp - kMmaWarp0;
      const uint32_t d_acc = tmem + (uint32_t)(gi * BNT);
      const int num_h = num_kb / 2;
      int sidx = 0;  // 64-k sub-stages of this group so far
      for (int h = gi; h < num_h && !bars->err; h += kMmaWarps) {
        const int xs = h % NX;
        if (!CONV) {
          // one wait for the B tile and one for the half stage's second A
          // sub-slot: the same 128 threads signal the first sub-slot before
          // the second, so its phase is complete too (fewer waits: with the
          // dequantization warps storing into tensor memory, this warp's
          // waits and MMAs take several times their cost in an idle CTA)
          if (!wait_or_fail(&bars->xfull[xs], (h / NX) & 1, bars)) break;
          const int s1 = sidx + 1;
          if (!wait_or_fail(&bars->afull[gi * C::kNS + s1 % C::kNS], (s1 / C::kNS) & 1, bars)) break;
        }
#pragma unroll
        for (int sub = 0; sub < 2; ++sub, ++sidx) {
          const int slot = gi * C::kNS + sidx % C::kNS;
          if (CONV && !wait_or_fail(&bars->afull[slot], (sidx / C::kNS) & 1, bars)) break;
          ptx::tc_fence_after();
          const uint32_t a_col = tmem + (uint32_t)(C::kABase + 32 * slot);
          const uint32_t b_tile = CONV ? ptx::smem_u32(xring + slot * C::kXSlot)
                                       : ptx::smem_u32(xring + xs * C::kXSlot + sub * C::kXTile);
#pragma unroll
          for (int j = 0; j < kBK / 16; ++j)  // the issuer's first MMA overwrites its accumulator
            ptx::mma_ts_f16(d_acc, a_col + 8 * j, ptx::sw128_kmajor_desc(b_tile + 32 * j), C::kIdesc,
                            h != gi || sub != 0 || j != 0);
          if (CONV) ptx::mma_commit(&bars->aempty[slot]);
        }
        // M > 8: one commit frees both A sub-slots and the B slot of the half stage
        if (!CONV) ptx::mma_commit(&bars->hdone[gi * 4 + ((h - gi) / kMmaWarps) % 4]);
      }
      // arrives when every MMA of this issuer is done (also on the error path,
      // so that TMEM is never freed under a running MMA)
      ptx::mma_commit(&bars->tmem_full);
      if (bars->err) ptx::mbar_wait(&bars->tmem_full, 0, kWaitLimitNs);
    }
  } else if (warp >= kXWarp0) {
    // ------------------ M > 8: f16 activation tiles from the pre-pass (TMA), one warp per issuer
    if constexpr (!CONV) {
      if (lane == 0) {
        asm volatile("griddepcontrol.wait;" ::: "memory");  // written by the pre-pass kernel
        const int gi = warp - kXWarp0;
        const int num_h = num_kb / 2;
        int h = gi;
        for (; h < num_h; h += kMmaWarps) {  // this issuer's half stages h = gi mod 4, slot h % NX
          const int xs = h % NX;
          // the slot was last read by this issuer's half stage kk - NX / 4 (kk = its index among them)
          const int kk = (h - gi) / kMmaWarps, kprev = kk - NX / kMmaWarps;
          if (kprev >= 0 && !wait_or_fail(&bars->hdone[gi * 4 + kprev % 4], (kprev / 4) & 1, bars)) break;
          ptx::mbar_arrive_expect_tx(&bars->xfull[xs], C::kXSlot);
#pragma unroll
          for (int sub = 0; sub < 2; ++sub)
            ptx::tma_load_2d(xring + xs * C::kXSlot + sub * C::kXTile, &tmap_x, &bars->xfull[xs],
                             (2 * h + sub) * kBK, m0);
        }
        if (bars->err)  // let the copies already issued land before the CTA exits
          for (int hh = h - NX > gi ? h - NX : gi; hh < h; hh += kMmaWarps)
            ptx::mbar_wait(&bars->xfull[hh % NX], (hh / NX) & 1, kWaitLimitNs);
      }
    }
  } else {
    // ------------------------------- M <= 8: |x| range of every row, all 17 warps
    if constexpr (CONV) {
      asm volatile("griddepcontrol.wait;" ::: "memory");  // X may come from the previous kernel
      const int t = threadIdx.x - kConvWarp * 32;
      // rows M..7 of every B tile (and the atom after the ring) stay zero
      for (int i = t; i < C::kXRing / 16; i += kScanThreads) sts128(ptx::smem_u32(xring) + 16 * i, make_uint4(0, 0, 0, 0));
      for (int m = 0; m < M; ++m) {
        const uint16_t* xr = X + (int64_t)m * ldx;
        uint32_t mx = 0, mn = 0xFFFFu;
        for (int i = t; i < K / 8; i += kScanThreads) {
          const uint4 v = *reinterpret_cast<const uint4*>(xr + 8 * i);
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
        if (lane == 0) {
          atomicMax(&bars->xmax[m], mx);
          atomicMin(&bars->xmin[m], mn);
        }
      }
      asm volatile("bar.sync 1, %0;" ::"r"(kScanThreads) : "memory");
    }

    if (warp == kConvWarp) {
      if constexpr (CONV) {
        // M <= 8: the dequantization groups convert X themselves
      } else {
        // M > 8: the activation tiles come from the producer warps kXWarp0.. (one per issuer)
      }
    } else {
      // ------------------------------------------------ dequantize into TMEM
      const int dw = warp - kDeqWarp0;         // 0..15
      const int grp = dw >> 2;                 // weight stages grp mod 4
      const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31
      const int r = 32 * quarter + lane;       // weight row in the tile
      const uint32_t swz = (uint32_t)(r & 7);
      const uint32_t lane_base = tmem + ((uint32_t)(32 * quarter) << 16);
      const int num_h = num_kb / 2;
      // M <= 8: warp j of the group converts rows 2j, 2j+1 of X for each of its
      // stages (lane l: row 2j + l / 16, 8 k at 8 * (l % 16), i.e. 64-k tile
      // (l % 16) / 8), prefetched one stage ahead from global memory
      const int xm = 2 * (dw & 3) + (lane >> 4), xc = lane & 15;
      const bool x_row = CONV && xm < M;
      float xf1 = 1.0f, xf2 = 1.0f;
      if (x_row) {
        const int e = row_exponent(bars->xmax[xm], bars->xmin[xm]);
        const int ee = e == kWideRow ? 0 : e;  // wide rows: these columns are recomputed
        xf1 = exp2i(ee / 2);
        xf2 = exp2i(ee - ee / 2);
      }
      const uint16_t* xsrc = X + (int64_t)(x_row ? xm : 0) * ldx + 8 * xc;
      const uint32_t xoff = (uint32_t)(xm * 128) + ((((uint32_t)xc & 7u) ^ (uint32_t)(xm & 7)) << 4);
      uint4 xnext = make_uint4(0, 0, 0, 0);
      if (x_row && grp < num_h) xnext = *reinterpret_cast<const uint4*>(xsrc + 128 * grp);
      int sidx = 0;  // 64-k sub-stages of this group so far
      bool ok = true;
      for (int h = grp; h < num_h && ok; h += 4) {  // 128-k stage h: half h % 2 of weight stage h / 2
        const int wb = h >> 1, half = h & 1;
        const int st = wb % NW;
        // warp-uniform outcome: the TMEM stores below are warp-wide instructions
        if (!__all_sync(0xFFFFFFFFu, wait_or_fail(&bars->wfull[st], (wb / NW) & 1, bars))) break;
        // this row's 64 code bytes of the half stage (16-byte chunks stored at
        // chunk ^ (row % 8)) and its 8 scale bytes
        const uint32_t wrow = ptx::smem_u32(wq + st * C::kWQ) + r * 128;
        const uint2 sc = lds64(ptx::smem_u32(wsc + st * C::kWS) + r * 16 + 8 * half);
        const uint32_t scw[2] = {sc.x, sc.y};
        const uint4 xv = xnext;
        if (x_row && h + 4 < num_h) xnext = *reinterpret_cast<const uint4*>(xsrc + 128 * (h + 4));
#pragma unroll
        for (int sub = 0; sub < 2; ++sub, ++sidx) {  // 64 k per A sub-slot of 32 TMEM columns
          const int slot = grp * C::kNS + sidx % C::kNS, round = sidx / C::kNS;
          const uint32_t ch = (uint32_t)(4 * half + 2 * sub);
          const uint4 c0 = lds128(wrow + ((ch ^ swz) << 4));
          const uint4 c1 = lds128(wrow + (((ch + 1) ^ swz) << 4));
          const uint32_t s01 = e4m3x2_to_f16x2(scw[sub] & 0xFFFFu), s23 = e4m3x2_to_f16x2(scw[sub] >> 16);
          uint32_t v[32];
          dequant8(c0.x, __byte_perm(s01, 0, 0x1010), v + 0);
          dequant8(c0.y, __byte_perm(s01, 0, 0x1010), v + 4);
          dequant8(c0.z, __byte_perm(s01, 0, 0x3232), v + 8);
          dequant8(c0.w, __byte_perm(s01, 0, 0x3232), v + 12);
          dequant8(c1.x, __byte_perm(s23, 0, 0x1010), v + 16);
          dequant8(c1.y, __byte_perm(s23, 0, 0x1010), v + 20);
          dequant8(c1.z, __byte_perm(s23, 0, 0x3232), v + 24);
          dequant8(c1.w, __byte_perm(s23, 0, 0x3232), v + 28);
          // the sub-slot is free once the MMAs of its previous use (sub-stage
          // sidx - kNS) finished: for M > 8 that is the group's half stage
          // (sidx - kNS) / 2, whose MMAs signal hdone with one commit
          const int kprev = (sidx - C::kNS) / 2;
          if (round > 0 && !__all_sync(0xFFFFFFFFu,
                                       CONV ? wait_or_fail(&bars->aempty[slot], (round - 1) & 1, bars)
                                            : wait_or_fail(&bars->hdone[grp * 4 + kprev % 4], (kprev / 4) & 1, bars))) {
            ok = false;
            break;
          }
          ptx::tmem_st_32cols(lane_base + (uint32_t)(C::kABase + 32 * slot), v);
          if (x_row && (xc >> 3) == sub) {
            sts128(ptx::smem_u32(xring + slot * C::kXSlot) + xoff, bf16x8_to_f16x8(xv, xf1, xf2));
            ptx::fence_proxy_async_smem();
          }
          ptx::tmem_st_wait();
          ptx::tc_fence_before();
          ptx::mbar_arrive(&bars->afull[slot]);
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bars->wempty[st]);
      }

      // ------------------------------------------------------------ epilogue
      if (static_weights) asm volatile("griddepcontrol.wait;" ::: "memory");  // row info and Y
      // stage the tile's row info once and find out whether any row needs the
      // exact recompute
      bool wide_here = false;
      for (int i = dw * 32 + lane; i < BNT; i += kDeqWarps * 32) {
        const int m = m0 + i;
        const int e = m >= M ? 0 : (CONV ? row_exponent(bars->xmax[m], bars->xmin[m]) : __ldg(info + m));
        bars->info[i] = e;
        wide_here |= e == kWideRow;
      }
      const bool any_wide = group_any(kEpiBar, kDeqWarps * 32, wide_here);
      const bool acc_ready = __all_sync(0xFFFFFFFFu, wait_or_fail(&bars->tmem_full, 0, bars));
      const float gv = *g;
      if (acc_ready) {
        ptx::tc_fence_after();
        if (16 * grp < BNT) {  // group j stores columns 16j .. 16j+15
          float acc[16];
          const int n_acc = num_kb / 2 < C::kNAcc ? num_kb / 2 : C::kNAcc;  // issuers that had work
#pragma unroll 1
          for (int a = 0; a < n_acc; ++a) {  // fixed order: deterministic
            uint32_t part[16];
            ptx::tmem_ld_16cols(lane_base + (uint32_t)(a * BNT + 16 * grp), part);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] = a == 0 ? __uint_as_float(part[j]) : acc[j] + __uint_as_float(part[j]);
          }
          const int n = n0 + r;
          if (n < N) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int m = m0 + 16 * grp + j;
              if (m < M) {
                const int e = bars->info[16 * grp + j];
                if (e != kWideRow) {
                  const __nv_bfloat16 o = __float2bfloat16_rn((acc[j] * gv) * pow2f(-e));
                  Y[(int64_t)m * ldy + n] = *reinterpret_cast<const uint16_t*>(&o);
                }
              }
            }
          }
        }
      }
      // wide rows of X: exact fp32 dot on CUDA cores, four threads per weight
      // row (quarters of K), combined with two shuffles
      const int t = dw * 32 + lane;
      const int row = n0 + (t >> 2), part = t & 3;
      for (int mi = 0; mi < BNT && any_wide; ++mi) {
        const int m = m0 + mi;
        if (m >= M) break;
        if (bars->info[mi] != kWideRow) continue;
        float p = 0.0f;
        if (row < N) p = exact_dot(q, s, row, K, X + (int64_t)m * ldx, part * (K / 4), (part + 1) * (K / 4));
        p += __shfl_xor_sync(0xFFFFFFFFu, p, 1);
        p += __shfl_xor_sync(0xFFFFFFFFu, p, 2);
        if (row < N && part == 0) {
          const __nv_bfloat16 o = __float2bfloat16_rn(p * gv);
          Y[(int64_t)m * ldy + row] = *reinterpret_cast<const uint16_t*>(&o);
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int BNT, bool CONV>
cudaError_t launch_small(const uint16_t* X, int64_t ldx, const uint16_t* Xh, const int* info, const uint8_t* q,
                         const uint8_t* s, const float* g, uint16_t* Y, int64_t ldy, int M, int N, int K,
                         bool static_weights, cudaStream_t stream) {
  using C = SmallCfg<BNT, CONV>;
  CUtensorMap tw, ts, tx;
  if (!tc::make_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2, 128u,
                        (uint32_t)kBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !tc::make_tmap_2d(&ts, CU_TENSOR_MAP_DATA_TYPE_UINT8, s, (uint64_t)K / 16, (uint64_t)N, (uint64_t)K / 16, 16u,
                        (uint32_t)kBM, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  if (CONV) {
    if (!tc::make_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, (uint64_t)K, (uint64_t)M, (uint64_t)ldx * 2,
                          (uint32_t)kBK, 8u, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  } else {
    if (!tc::make_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Xh, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2,
                          (uint32_t)kBK, (uint32_t)BNT, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  static tc::SmemOptIn opt_in;
  const cudaError_t e = opt_in.ensure((const void*)gemm_small_kernel<BNT, CONV>, C::kSmem);
  if (e != cudaSuccess) return e;
  int sw = static_weights ? 1 : 0;
  void* args[] = {&tw, &ts, &tx, (void*)&q, (void*)&s, (void*)&g, (void*)&info, (void*)&X, &ldx, &Y, &ldy,
                  &M, &N, &K, &sw};
  const dim3 grid((N + kBM - 1) / kBM, CONV ? 1 : (M + BNT - 1) / BNT);
  return tc::launch_pdl((const void*)gemm_small_kernel<BNT, CONV>, grid, dim3(kThreads), C::kSmem, stream, args);
}

}  // namespace

bool gemm_small_supported(int64_t M, int64_t N, int64_t K) {
  return M >= 1 && M <= 64 && N >= 1 && N <= ((int64_t)1 << 31) - 128 && K % 256 == 0 && K <= ((int64_t)1 << 24);
}

size_t gemm_small_workspace_bytes(int64_t M, int64_t K) {
  return M <= kConvMaxM ? 0 : gemm_prep_workspace_bytes(M, K);
}

cudaError_t launch_gemm_small(const uint16_t* X, int64_t ldx, const uint8_t* q, const uint8_t* s, const float* g,
                              uint16_t* Y, int64_t ldy, int64_t M, int64_t N, int64_t K, void* workspace,
                              bool static_weights, cudaStream_t stream) {
  const int m = (int)M, n = (int)N, k = (int)K;
  if (M <= kConvMaxM)
    return launch_small<16, true>(X, ldx, nullptr, nullptr, q, s, g, Y, ldy, m, n, k, static_weights, stream);
  int* info = nullptr;
  uint16_t* Xh = nullptr;
  cudaError_t e = launch_gemm_prep(X, ldx, M, K, workspace, &info, &Xh, stream);
  if (e != cudaSuccess) return e;
  if (M <= 16) return launch_small<16, false>(X, ldx, Xh, info, q, s, g, Y, ldy, m, n, k, static_weights, stream);
  if (M <= 32) return launch_small<32, false>(X, ldx, Xh, info, q, s, g, Y, ldy, m, n, k, static_weights, stream);
  return launch_small<64, false>(X, ldx, Xh, info, q, s, g, Y, ldy, m, n, k, static_weights, stream);
}

cudaError_t read_and_clear_small_timeouts(unsigned int* count) {
  cudaError_t e = cudaMemcpyFromSymbol(count, g_small_wait_timeouts, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  const unsigned int zero = 0;
  return cudaMemcpyToSymbol(g_small_wait_timeouts, &zero, sizeof(unsigned int));
}

}  // namespace nvfp4

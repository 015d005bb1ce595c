// gemm_w4a4.cu -- NVFP4 x NVFP4 (W4A4) prefill GEMM on the sm_100a block-scaled
// FP4 tensor cores (tcgen05.mma kind::mxf4nvf4).
//
// The pages' prefill runs weights and activations both in NVFP4 ("CUTLASS
// NVFP4 GEMM" of the dense-layer pipeline, imp docs/quantization.md; the
// Modelopt row's "NVFP4 x NVFP4 prefill"), with the weight micro-scales
// rearranged once into the tensor core's scale-factor layout ("Phase 3b").
// Here:
//   Y[m, n] = bf16(g * g_x * sum_k (sw[n, k/16] qw[n, k]) (sx[m, k/16] qx[m, k]))
// with g_x = x_amax / 2688 and X quantized by the weights' rule
// (x_amax_partial_kernel and quantize_x_mma_kernel below, with the block
// rule of nvfp4_quant.cuh).  Every product of two E2M1 codes and two E4M3
// scales is exact in fp32; the tensor core accumulates in fp32.
//
// Scale-factor layout (weights and activations alike): one 512-byte atom per
// 128 rows and 64 k; row r, 16-block j of the step at byte
// (r % 32) * 16 + (r / 32) * 4 + j.  One tcgen05.cp (32 rows x 16 bytes,
// replicated into the four lane quarters) moves an atom into 4 TMEM columns,
// where the MMA reads row r at lane r % 32, column r / 32, byte j.
//
// Tile: 128 weight rows (MMA M, operand A) x 256 tokens (MMA N, operand B),
// 256 k per pipeline stage (one 128-byte swizzled row of packed codes, four
// MMAs of K = 64):
//   - warp 0, one thread: TMA loads of the weight codes [128, 128 B] and the
//     token codes [256, 128 B] (out-of-range rows read as zero) and bulk
//     copies of the stage's scale atoms (2 KB of weights, 2 x 2 KB of tokens);
//   - warps 18..20, one thread each: warp 18 + j copies atom j of every MMA
//     (j = 0: weight scales, 1 and 2: the two halves of the token scales)
//     into the stage's own TMEM columns with tcgen05.cp, committed per stage
//     to "sf_full" (three arrivals);
//   - warp 1, one thread: the four MMAs of a stage into the [128 x 256] fp32
//     accumulator once its codes ("full") and scale factors ("sf_full") are
//     in; each stage is committed to its "empty" barrier;
//   - warps 2..17: the epilogue, TMEM -> g * g_x -> BF16 Y, four warps per
//     TMEM lane quarter, each with two of the tile's eight 32-column blocks.
// The copies have threads of their own because one thread issues a tcgen05
// instruction only every few tens of cycles: with the twelve copies and four
// MMAs of a stage in one thread, the issue took longer than the tensor pipe's
// work (35.0 µs on the 512 x 17408 x 5120 layer, 26.5 µs with the copies
// left out, 32.2 µs with them in one thread of their own).
// The kernel is persistent (one CTA per SM, tiles in a fixed stride), so
// the next tile's stages stream in while the epilogue drains the accumulator.
// A stage's TMEM scale columns are rewritten only after the MMAs that read
// them have completed: the copy warp rewrites them after the stage's next
// "full", which follows its "empty" (the MMAs' commit) and the reload.
// Every wait is bounded.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "nvfp4_device.cuh"
#include "nvfp4_kernels.h"
#include "nvfp4_quant.cuh"
#include "sm100_ptx.cuh"
#include "tc_host.h"

namespace nvfp4 {

// CTAs of the W4A4 GEMM whose pipeline wait ran past its time limit.
__device__ unsigned int g_w4a4_wait_timeouts = 0;

namespace {

constexpr int kBM = 128;                      // weight rows per tile (MMA M)
constexpr int kBN = 256;                      // tokens per tile (MMA N)
constexpr int kStageK = 256;                  // k per pipeline stage
constexpr int kStages = 4;
constexpr int kABytes = kBM * 128;            // packed weight codes of a stage
constexpr int kBBytes = kBN * 128;            // packed token codes of a stage
constexpr int kSFABytes = 4 * 512;            // weight scale atoms (4 MMAs)
constexpr int kSFBBytes = 2 * 4 * 512;        // token scale atoms (2 x 128 tokens, 4 MMAs)
constexpr int kStageBytes = kABytes + kBBytes + kSFABytes + kSFBBytes;
constexpr int kEpiWarp0 = 2, kEpiWarps = 16;  // epilogue: four warps per TMEM lane quarter
static_assert(kEpiWarps % 4 == 0, "every TMEM lane quarter has the same number of epilogue warps");
constexpr int kEpiBytes = kEpiWarps * 512;     // each epilogue warp's 8 tokens x 32 rows BF16 staging block
constexpr int kSfWarp0 = kEpiWarp0 + kEpiWarps, kSfWarps = 3;  // scale-factor copies, one warp per atom
constexpr int kThreads = (kSfWarp0 + kSfWarps) * 32;
constexpr uint32_t kTmemCols = 512;           // 256 accumulator + 4 stages x 4 MMAs x 12 scale columns
constexpr uint32_t kSfCol0 = 256;
constexpr uint32_t kSfColsPerMma = 12;        // 4 weight + 8 token columns
constexpr uint32_t kIdesc = ptx::idesc_nvf4(kBM, kBN);
constexpr uint64_t kWaitLimitNs = 2000000000ull;
static_assert(kStageBytes % 1024 == 0, "stages stay 1024-byte aligned (128-byte swizzle)");
static_assert(kSfCol0 + kStages * 4 * kSfColsPerMma <= kTmemCols, "TMEM columns");

struct Bars {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t sf_full[kStages];  // the stage's scale factors are in tensor memory (the copy warps' commits)
  uint64_t sf_done;           // every scale-factor copy of the CTA has finished (teardown)
  uint64_t acc_full;   // the accumulator of the current tile is complete (one phase per tile)
  uint64_t acc_empty;  // the epilogue has read it (kEpiWarps arrivals per tile)
  uint64_t mma_done;   // every MMA of the CTA has finished (teardown)
  uint32_t tmem_addr;
  volatile int err;
};

constexpr int kSmemBytes = kStages * kStageBytes + kEpiBytes + (int)sizeof(Bars) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

__device__ __forceinline__ bool wait_or_fail(uint64_t* bar, uint32_t parity, Bars* bars) {
  if (bars->err) return false;
  if (ptx::mbar_wait(bar, parity, kWaitLimitNs)) return true;
  if (!bars->err) {
    bars->err = 1;
    atomicAdd(&g_w4a4_wait_timeouts, 1u);
  }
  return false;
}

// A wait that spans a whole main loop (the epilogue's): the thread sleeps
// between polls instead of taking issue slots from the producer, copy and MMA
// threads.  Bounded like every other wait.
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  while (!ptx::mbar_try_wait_sleep(bar, parity))
    if (ptx::globaltimer_ns() - t0 > limit_ns) return false;
  return true;
}

// wait_or_fail with the sleeping wait
__device__ __forceinline__ bool wait_or_fail_sleep(uint64_t* bar, uint32_t parity, Bars* bars) {
  if (bars->err) return false;
  if (mbar_wait_sleep(bar, parity, kWaitLimitNs)) return true;
  if (!bars->err) {
    bars->err = 1;
    atomicAdd(&g_w4a4_wait_timeouts, 1u);
  }
  return false;
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

// Epilogue of a [128 weight rows x 256 tokens] fp32 accumulator tile: the
// warp reads the TMEM lane quarter its index fixes (warp % 4: a warp may only
// reach those 32 lanes, its weight rows) and the 32-column blocks p, p + 4
// (tokens) for its rank p = (warp - kEpiWarp0) / 4 among the epilogue warps
// of that quarter, scales by `scale` and stores BF16 Y[m, n], eight tokens
// at a time through its 512 bytes of shared memory at `stage` so that each
// lane stores 16 bytes (a quarter of a token's 32 rows).
__device__ __forceinline__ void store_tile(uint32_t tmem, int warp, int lane, float scale, uint32_t stage,
                                           uint16_t* __restrict__ Y, int64_t ldy, int M, int N, int m0, int n0) {
  const int quarter = warp & 3, part = (warp - kEpiWarp0) >> 2;
  const int jj = lane >> 2, piece = lane & 3;  // this lane's 16 bytes of a round: token jj, rows 8 piece ..
  const int nb = n0 + 32 * quarter + 8 * piece;
  const bool vec_ok = ((reinterpret_cast<uintptr_t>(Y) & 15u) == 0) && (ldy % 8 == 0);
#pragma unroll 1
  for (int c0 = 32 * part; c0 < kBN && m0 + c0 < M; c0 += 32 * (kEpiWarps / 4)) {
    uint32_t rr[32];
    ptx::tmem_ld_32cols(tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)c0, rr);
    ptx::tmem_ld_wait();
#pragma unroll
    for (int r = 0; r < 4; ++r) {  // tokens c0 + 8 r .. c0 + 8 r + 7
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const __nv_bfloat16 o = __float2bfloat16_rn(__uint_as_float(rr[8 * r + j]) * scale);
        st_shared_u16(stage + (uint32_t)(j * 32 + lane) * 2u, *reinterpret_cast<const uint16_t*>(&o));
      }
      __syncwarp();
      const int m = m0 + c0 + 8 * r + jj;
      if (m < M && nb < N) {
        const uint4 v = ld_shared_v4(stage + (uint32_t)(jj * 32 + 8 * piece) * 2u);
        uint16_t* dst = Y + (int64_t)m * ldy + nb;
        if (vec_ok && nb + 8 <= N) {
          *reinterpret_cast<uint4*>(dst) = v;
        } else {
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
          for (int i = 0; i < 8 && nb + i < N; ++i) dst[i] = (uint16_t)(w4[i >> 1] >> (16 * (i & 1)));
        }
      }
      __syncwarp();
    }
  }
}

// Rows of the weight scale rearrangement: thread t writes the 16 bytes of
// atom row r0 for (tile, step): the four scale words of rows
// tile*128 + 32*i + r0, i = 0..3 (zero beyond N).
__global__ void __launch_bounds__(256) scales_to_mma_kernel(const uint8_t* __restrict__ s, int64_t N, int64_t K,
                                                            uint8_t* __restrict__ s_mma) {
  const int64_t steps = K / 64, tiles = (N + 127) / 128;
  const int64_t total = tiles * steps * 32;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total; t += stride) {
    const int64_t r0 = t % 32, atom = t / 32;  // atom = tile * steps + step
    const int64_t tile = atom / steps, step = atom - tile * steps;
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t row = tile * 128 + 32 * i + r0;
      w[i] = row < N ? *reinterpret_cast<const uint32_t*>(s + row * (K / 16) + step * 4) : 0u;
    }
    *reinterpret_cast<uint4*>(s_mma + atom * 512 + r0 * 16) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// Persistent: gridDim.x CTAs (at most one per SM) take the tiles
// t = blockIdx.x, blockIdx.x + gridDim.x, ... (weight tile t % tiles_n, token
// tile t / tiles_n).  The ring's stage counter runs on across tiles, so the
// producer streams the next tile while the epilogue drains the accumulator;
// the next tile's first MMA waits for the epilogue (acc_empty).
__global__ void __launch_bounds__(kThreads, 1)
    gemm_w4a4_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                     const uint8_t* __restrict__ s_mma, const uint8_t* __restrict__ sx,
                     const float* __restrict__ g, const float* __restrict__ x_amax, uint16_t* __restrict__ Y,
                     int64_t ldy, int M, int N, int K, int static_weights) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  auto a_tile = [&](int st) { return smem + st * kStageBytes; };
  auto b_tile = [&](int st) { return smem + st * kStageBytes + kABytes; };
  auto sfa = [&](int st) { return smem + st * kStageBytes + kABytes + kBBytes; };
  auto sfb = [&](int st) { return smem + st * kStageBytes + kABytes + kBBytes + kSFABytes; };
  uint8_t* epi = smem + kStages * kStageBytes;
  Bars* bars = reinterpret_cast<Bars*>(epi + kEpiBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int steps64 = K / 64;
  const int num_ks = K / kStageK;
  const int tiles_n = (N + kBM - 1) / kBM;
  const int tiles = tiles_n * ((M + kBN - 1) / kBN);

  if (threadIdx.x == 0) {
    for (int st = 0; st < kStages; ++st) {
      ptx::mbar_init(&bars->full[st], 1);
      ptx::mbar_init(&bars->empty[st], 1);
      ptx::mbar_init(&bars->sf_full[st], kSfWarps);
    }
    ptx::mbar_init(&bars->sf_done, kSfWarps);
    ptx::mbar_init(&bars->acc_full, 1);
    ptx::mbar_init(&bars->acc_empty, kEpiWarps);
    ptx::mbar_init(&bars->mma_done, 1);
    bars->err = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tmap_w);
    ptx::prefetch_tmap(&tmap_x);
  }
  if (warp == 1) {
    ptx::tmem_alloc(&bars->tmem_addr, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_addr;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int gi = 0;  // stages issued so far (over all tiles of this CTA)
      bool first = true;
      for (int t = blockIdx.x; t < tiles && !bars->err; t += gridDim.x) {
        const int nt = t % tiles_n, mt = t / tiles_n;
        const int n0 = nt * kBM, m0 = mt * kBN;
        const uint8_t* sa_src = s_mma + (int64_t)nt * steps64 * 512;
        const uint8_t* sb_src0 = sx + (int64_t)(2 * mt) * steps64 * 512;
        const uint8_t* sb_src1 = sx + (int64_t)(2 * mt + 1) * steps64 * 512;
        auto issue_w = [&](int st, int ks) {
          ptx::tma_load_2d(a_tile(st), &tmap_w, &bars->full[st], ks * 128, n0);
          ptx::bulk_load(sfa(st), sa_src + ks * kSFABytes, kSFABytes, &bars->full[st]);
        };
        auto issue_x = [&](int st, int ks) {
          ptx::tma_load_2d(b_tile(st), &tmap_x, &bars->full[st], ks * 128, m0);
          ptx::bulk_load(sfb(st), sb_src0 + ks * 2048, 2048, &bars->full[st]);
          ptx::bulk_load(sfb(st) + 2048, sb_src1 + ks * 2048, 2048, &bars->full[st]);
        };
        int ks = 0;
        if (first) {
          // the ring starts empty; with static weights the first stages'
          // weights stream before the producer of X has finished
          const int f = num_ks < kStages ? num_ks : kStages;
          for (int k = 0; k < f; ++k) ptx::mbar_arrive_expect_tx(&bars->full[k], kStageBytes);
          if (static_weights)
            for (int k = 0; k < f; ++k) issue_w(k, k);
          asm volatile("griddepcontrol.wait;" ::: "memory");
          for (int k = 0; k < f; ++k) {
            if (!static_weights) issue_w(k, k);
            issue_x(k, k);
          }
          ks = f;
          gi = f;
          first = false;
        }
        for (; ks < num_ks; ++ks) {
          const int st = gi % kStages;
          if (gi >= kStages && !wait_or_fail(&bars->empty[st], ((gi / kStages) - 1) & 1, bars)) break;
          ptx::mbar_arrive_expect_tx(&bars->full[st], kStageBytes);
          issue_w(st, ks);
          issue_x(st, ks);
          ++gi;
        }
      }
      if (bars->err) {
        // let the copies already issued land before the CTA exits
        for (int j = gi > kStages ? gi - kStages : 0; j < gi; ++j)
          ptx::mbar_wait(&bars->full[j % kStages], (j / kStages) & 1, kWaitLimitNs);
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int gi = 0, it = 0;
      for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++it) {
        // the accumulator is free once the epilogue has read the previous tile
        if (it > 0) {
          if (!wait_or_fail(&bars->acc_empty, (it - 1) & 1, bars)) break;
          ptx::tc_fence_after();
        }
        bool ok = true;
        for (int ks = 0; ks < num_ks; ++ks, ++gi) {
          const int st = gi % kStages;
          // the stage's codes (TMA) and its scale factors (the copy warp)
          if (!wait_or_fail(&bars->full[st], (gi / kStages) & 1, bars) ||
              !wait_or_fail(&bars->sf_full[st], (gi / kStages) & 1, bars)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a0 = ptx::smem_u32(a_tile(st)), b0 = ptx::smem_u32(b_tile(st));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t col = tmem + kSfCol0 + (uint32_t)(st * 4 + kk) * kSfColsPerMma;
            ptx::mma_nvf4(tmem, ptx::sw128_kmajor_desc(a0 + 32 * kk), ptx::sw128_kmajor_desc(b0 + 32 * kk),
                          kIdesc, col, col + 4, (ks | kk) != 0);
          }
          ptx::mma_commit(&bars->empty[st]);
        }
        if (!ok) break;
        ptx::mma_commit(&bars->acc_full);
      }
      // arrives when every MMA above is done, so that TMEM is never freed
      // under a running MMA (also on the error path)
      ptx::mma_commit(&bars->mma_done);
      ptx::mbar_wait(&bars->mma_done, 0, kWaitLimitNs);
    }
  } else if (warp >= kSfWarp0) {
    // ------------------------------------------- scale factors into tensor memory
    // copy warp j: atom j of each MMA (weights, tokens 0-127, tokens 128-255),
    // four 512-byte copies per stage, ahead of the MMAs (a slot's columns are
    // rewritten only after its next `full`: after the MMAs that read them)
    const uint32_t j = (uint32_t)(warp - kSfWarp0);
    if (lane == 0) {
      int gi = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        for (int ks = 0; ks < num_ks; ++ks, ++gi) {
          const int st = gi % kStages;
          if (!wait_or_fail(&bars->full[st], (gi / kStages) & 1, bars)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          // atom j of MMA kk: weights at sfa + 512 kk, tokens at sfb + 2048 (j - 1) + 512 kk
          const uint32_t src = j == 0 ? ptx::smem_u32(sfa(st)) : ptx::smem_u32(sfb(st)) + 2048u * (j - 1);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t col = tmem + kSfCol0 + (uint32_t)(st * 4 + kk) * kSfColsPerMma + 4u * j;
            ptx::tmem_copy_sf(col, ptx::rows16_desc(src + kk * 512));
          }
          ptx::mma_commit(&bars->sf_full[st]);
        }
      }
      // arrives when every copy above is done, so that TMEM is never freed
      // under a running copy (also on the error path)
      ptx::mma_commit(&bars->sf_done);
      ptx::mbar_wait(&bars->sf_done, 0, kWaitLimitNs);
    }
  } else {
    // ----------------------------------------------------------------- epilogue
    asm volatile("griddepcontrol.wait;" ::: "memory");  // x_amax and Y
    const float scale = __fmul_rn(*g, __fdiv_rn(*x_amax, 2688.0f));
    const uint32_t stage = ptx::smem_u32(epi) + (uint32_t)(warp - kEpiWarp0) * 512u;
    int it = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++it) {
      const int nt = t % tiles_n, mt = t / tiles_n;
      if (!__all_sync(0xFFFFFFFFu, wait_or_fail_sleep(&bars->acc_full, it & 1, bars))) break;
      ptx::tc_fence_after();
      store_tile(tmem, warp, lane, scale, stage, Y, ldy, M, N, mt * kBN, nt * kBM);
      // every TMEM read of this tile has completed (tcgen05.wait::ld above)
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bars->acc_empty);
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------ pair-of-SMs tile
//
// The same GEMM on tiles of 256 weight rows x 256 tokens run by a cluster of
// two CTAs on two SMs (tcgen05 cta_group::2): each CTA holds its 128 weight
// rows (the pair's MMA has M = 256) and half of the tile's tokens (B rows
// 128 r .. 128 r + 127 of CTA rank r), so a token tile crosses from L2 into
// the SMs once per 256 weight rows instead of once per 128.  The even CTA
// issues the scale copies and the MMAs for both; each CTA's tensor memory
// holds its 128 accumulator rows x 256 tokens and the scale factors of its
// own weight rows and of all 256 tokens (each CTA loads the token scales in
// full).  A stage is 38 KB (16 KB of weight codes, 16 KB of token codes,
// 2 + 4 KB of scale atoms), so five stages fit beside the epilogue.
//   - warp 0 of each CTA: TMA of its own stage bytes (codes and scale atoms)
//     into its own shared memory, all counted on the even CTA's `full`
//     (the odd CTA's loads use the pair form of the tensor copy);
//   - warps 18..20 of the even CTA: the scale-factor copies (pair form), one
//     warp per atom as in the one-SM kernel, committed to "sf_full";
//   - warp 1 of the even CTA: the MMA issuer; its commits arrive on both
//     CTAs' barriers;
//   - warps 2..17: the epilogue of each CTA's accumulator rows; the even
//     CTA's issuer waits for both epilogues (acc_empty, 32 arrivals) before
//     it overwrites the accumulator.
constexpr int kPairStages = 5;
constexpr int kPairThreads = kThreads;                 // the same warp roles
constexpr int kPairBBytes = (kBN / 2) * 128;          // this CTA's 128 tokens of a stage
constexpr int kPairStageBytes = kABytes + kPairBBytes + kSFABytes + kSFBBytes;
constexpr uint32_t kPairIdesc = ptx::idesc_nvf4(2 * kBM, kBN);
static_assert(kPairStageBytes % 1024 == 0, "stages stay 1024-byte aligned (128-byte swizzle)");
static_assert(kSfCol0 + kPairStages * 4 * kSfColsPerMma <= kTmemCols, "TMEM columns");

struct PairBars {
  uint64_t full[kPairStages];       // (even CTA) both CTAs' bytes of the stage have landed
  uint64_t empty[kPairStages];      // the pair's MMAs that read the stage are done
  uint64_t sf_full[kPairStages];    // the stage's scale factors are in both CTAs' tensor memory
  uint64_t sf_done;                 // (even CTA) every scale-factor copy has finished (teardown)
  uint64_t acc_full;                // the tile's accumulator is complete
  uint64_t acc_empty;               // (even CTA) both CTAs' epilogues have read it
  uint64_t mma_done;                // every MMA of the pair has finished (teardown)
  uint32_t tmem_addr;
  volatile int err;
};

constexpr int kPairSmemBytes = kPairStages * kPairStageBytes + kEpiBytes + (int)sizeof(PairBars) + 1024;
static_assert(kPairSmemBytes <= 232448, "shared memory per CTA");

__device__ __forceinline__ bool pair_wait(uint64_t* bar, uint32_t parity, PairBars* bars) {
  if (bars->err) return false;
  if (ptx::mbar_wait_cluster(bar, parity, kWaitLimitNs)) return true;
  if (!bars->err) {
    bars->err = 1;
    atomicAdd(&g_w4a4_wait_timeouts, 1u);
  }
  return false;
}

// Persistent pairs: cluster c = blockIdx.x / 2 takes the pair tiles
// t = c, c + gridDim.x / 2, ... (weight rows 256 (t % tiles_n), tokens
// 256 (t / tiles_n)); both CTAs walk the same tiles and stages.
__global__ void __launch_bounds__(kPairThreads, 1)
    gemm_w4a4_pair_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                          const __grid_constant__ CUtensorMap tmap_sa, const __grid_constant__ CUtensorMap tmap_sb,
                          const float* __restrict__ g, const float* __restrict__ x_amax, uint16_t* __restrict__ Y,
                          int64_t ldy, int M, int N, int K, int static_weights) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  auto a_tile = [&](int st) { return smem + st * kPairStageBytes; };
  auto b_tile = [&](int st) { return smem + st * kPairStageBytes + kABytes; };
  auto sfa = [&](int st) { return smem + st * kPairStageBytes + kABytes + kPairBBytes; };
  auto sfb = [&](int st) { return smem + st * kPairStageBytes + kABytes + kPairBBytes + kSFABytes; };
  uint8_t* epi = smem + kPairStages * kPairStageBytes;
  PairBars* bars = reinterpret_cast<PairBars*>(epi + kEpiBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();  // 0: issues the pair's MMAs
  const int cluster = blockIdx.x >> 1, clusters = gridDim.x >> 1;
  const int steps64 = K / 64;
  const int num_ks = K / kStageK;
  const int tiles_n = (N + 2 * kBM - 1) / (2 * kBM);
  const int tiles = tiles_n * ((M + kBN - 1) / kBN);
  const int scale_tiles = (N + kBM - 1) / kBM;  // 128-row tiles of s_mma

  if (threadIdx.x == 0) {
    for (int st = 0; st < kPairStages; ++st) {
      ptx::mbar_init(&bars->full[st], 1);
      ptx::mbar_init(&bars->empty[st], 1);
      ptx::mbar_init(&bars->sf_full[st], kSfWarps);
    }
    ptx::mbar_init(&bars->sf_done, kSfWarps);
    ptx::mbar_init(&bars->acc_full, 1);
    ptx::mbar_init(&bars->acc_empty, 2 * kEpiWarps);
    ptx::mbar_init(&bars->mma_done, 1);
    bars->err = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tmap_w);
    ptx::prefetch_tmap(&tmap_x);
    ptx::prefetch_tmap(&tmap_sa);
    ptx::prefetch_tmap(&tmap_sb);
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(&bars->tmem_addr, kTmemCols);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // both CTAs' barriers exist before either signals the other
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_addr;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int gi = 0;  // stages issued so far (over all tiles of this pair)
      bool first = true;
      for (int t = cluster; t < tiles && !bars->err; t += clusters) {
        const int nt = t % tiles_n, mt = t / tiles_n;
        const int n0 = nt * 2 * kBM + (int)rank * kBM, m0 = mt * kBN;
        // the odd CTA's rows may lie past N: its scale atoms then come from
        // the last tile (its codes read as zero; its outputs are not stored)
        const int sa_tile = n0 / kBM < scale_tiles ? n0 / kBM : scale_tiles - 1;
        // scale maps: rows of 256 bytes, a stage's four 512-byte atoms are 8 rows
        const int sa_row = sa_tile * steps64 * 2, sb_row0 = 2 * mt * steps64 * 2, sb_row1 = (2 * mt + 1) * steps64 * 2;
        auto issue = [&](int st, int ks, bool weights, bool tokens) {
          if (rank == 0) {
            if (weights) {
              ptx::tma_load_2d(a_tile(st), &tmap_w, &bars->full[st], ks * 128, n0);
              ptx::tma_load_2d(sfa(st), &tmap_sa, &bars->full[st], 0, sa_row + ks * 8);
            }
            if (tokens) {
              ptx::tma_load_2d(b_tile(st), &tmap_x, &bars->full[st], ks * 128, m0);
              ptx::tma_load_2d(sfb(st), &tmap_sb, &bars->full[st], 0, sb_row0 + ks * 8);
              ptx::tma_load_2d(sfb(st) + 2048, &tmap_sb, &bars->full[st], 0, sb_row1 + ks * 8);
            }
          } else {
            const uint32_t fb = ptx::cluster_addr(&bars->full[st], 0);
            if (weights) {
              ptx::tma_load_2d_pair(a_tile(st), &tmap_w, fb, ks * 128, n0);
              ptx::tma_load_2d_pair(sfa(st), &tmap_sa, fb, 0, sa_row + ks * 8);
            }
            if (tokens) {
              ptx::tma_load_2d_pair(b_tile(st), &tmap_x, fb, ks * 128, m0 + kBN / 2);
              ptx::tma_load_2d_pair(sfb(st), &tmap_sb, fb, 0, sb_row0 + ks * 8);
              ptx::tma_load_2d_pair(sfb(st) + 2048, &tmap_sb, fb, 0, sb_row1 + ks * 8);
            }
          }
        };
        int ks = 0;
        if (first) {
          const int f = num_ks < kPairStages ? num_ks : kPairStages;
          // the even CTA's barrier counts both CTAs' bytes of each stage
          if (rank == 0)
            for (int k = 0; k < f; ++k) ptx::mbar_arrive_expect_tx(&bars->full[k], 2 * kPairStageBytes);
          if (static_weights)
            for (int k = 0; k < f; ++k) issue(k, k, true, false);
          asm volatile("griddepcontrol.wait;" ::: "memory");
          for (int k = 0; k < f; ++k) issue(k, k, !static_weights, true);
          ks = f;
          gi = f;
          first = false;
        }
        for (; ks < num_ks; ++ks) {
          const int st = gi % kPairStages;
          if (gi >= kPairStages && !pair_wait(&bars->empty[st], ((gi / kPairStages) - 1) & 1, bars)) break;
          if (rank == 0) ptx::mbar_arrive_expect_tx(&bars->full[st], 2 * kPairStageBytes);
          issue(st, ks, true, true);
          ++gi;
        }
      }
      if (bars->err && rank == 0) {
        // let copies already issued land before the CTA exits (the odd CTA's
        // land on the even CTA's barriers, which this waits for too)
        for (int j = gi > kPairStages ? gi - kPairStages : 0; j < gi; ++j)
          ptx::mbar_wait_cluster(&bars->full[j % kPairStages], (j / kPairStages) & 1, kWaitLimitNs);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      if (rank == 0) {
        // ------------------------------------------- MMA issuer for the pair
        int gi = 0, it = 0;
        for (int t = cluster; t < tiles; t += clusters, ++it) {
          // the accumulator is free once both epilogues have read the previous tile
          if (it > 0) {
            if (!pair_wait(&bars->acc_empty, (it - 1) & 1, bars)) break;
            ptx::tc_fence_after();
          }
          bool ok = true;
          for (int ks = 0; ks < num_ks; ++ks, ++gi) {
            const int st = gi % kPairStages;
            const uint32_t par = (uint32_t)(gi / kPairStages) & 1u;
            if (!pair_wait(&bars->full[st], par, bars) || !pair_wait(&bars->sf_full[st], par, bars)) {
              ok = false;
              break;
            }
            ptx::tc_fence_after();
            const uint32_t a0 = ptx::smem_u32(a_tile(st)), b0 = ptx::smem_u32(b_tile(st));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t col = tmem + kSfCol0 + (uint32_t)(st * 4 + kk) * kSfColsPerMma;
              ptx::mma_nvf4_pair(tmem, ptx::sw128_kmajor_desc(a0 + 32 * kk), ptx::sw128_kmajor_desc(b0 + 32 * kk),
                                 kPairIdesc, col, col + 4, (ks | kk) != 0);
            }
            ptx::mma_commit_pair(&bars->empty[st]);
          }
          if (!ok) break;
          ptx::mma_commit_pair(&bars->acc_full);
        }
        // arrives in both CTAs when every MMA above is done (also on the
        // error path), so that neither frees its tensor memory under an MMA
        ptx::mma_commit_pair(&bars->mma_done);
      }
      ptx::mbar_wait_cluster(&bars->mma_done, 0, kWaitLimitNs);
    }
  } else if (warp >= kSfWarp0) {
    // ------------------ scale factors into both CTAs' tensor memory (even CTA)
    // copy warp j: atom j of each MMA, as in the one-SM kernel, with the pair
    // form of tcgen05.cp (each CTA's atom from its own shared memory)
    const uint32_t j = (uint32_t)(warp - kSfWarp0);
    if (lane == 0 && rank == 0) {
      int gi = 0;
      bool ok = true;
      for (int t = cluster; t < tiles && ok; t += clusters) {
        for (int ks = 0; ks < num_ks; ++ks, ++gi) {
          const int st = gi % kPairStages;
          if (!pair_wait(&bars->full[st], (uint32_t)(gi / kPairStages) & 1u, bars)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t src = j == 0 ? ptx::smem_u32(sfa(st)) : ptx::smem_u32(sfb(st)) + 2048u * (j - 1);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t col = tmem + kSfCol0 + (uint32_t)(st * 4 + kk) * kSfColsPerMma + 4u * j;
            ptx::tmem_copy_sf_pair(col, ptx::rows16_desc(src + kk * 512));
          }
          ptx::mma_commit_pair(&bars->sf_full[st]);
        }
      }
      // every copy done before the cluster's teardown (also on the error path)
      ptx::mma_commit_pair(&bars->sf_done);
      ptx::mbar_wait_cluster(&bars->sf_done, 0, kWaitLimitNs);
    }
  } else {
    // ----------------------------------------------------------------- epilogue
    asm volatile("griddepcontrol.wait;" ::: "memory");  // x_amax and Y
    const float scale = __fmul_rn(*g, __fdiv_rn(*x_amax, 2688.0f));
    const uint32_t stage = ptx::smem_u32(epi) + (uint32_t)(warp - kEpiWarp0) * 512u;
    int it = 0;
    for (int t = cluster; t < tiles; t += clusters, ++it) {
      const int nt = t % tiles_n, mt = t / tiles_n;
      if (!__all_sync(0xFFFFFFFFu, pair_wait(&bars->acc_full, it & 1, bars))) break;
      ptx::tc_fence_after();
      // this CTA's accumulator rows are weight rows nt * 256 + 128 * rank + lane
      store_tile(tmem, warp, lane, scale, stage, Y, ldy, M, N, mt * kBN, nt * 2 * kBM + (int)rank * kBM);
      // every TMEM read of this tile has completed (tcgen05.wait::ld above)
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0)
          ptx::mbar_arrive(&bars->acc_empty);
        else
          ptx::mbar_arrive_remote(&bars->acc_empty, 0);
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // neither CTA leaves while the other may still signal it or read its shared memory
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// ------------------------------------------------- activations for W4A4 GEMMs
//
// X [M, K] quantized by the weights' rule with g_x = x_amax / 2688: codes
// row-major [M, K/2] and the E4M3 scales in the tensor core's scale-factor
// layout: the scale of row m, 16-block b sits at byte
//   ((m / 128) * (K / 64) + b / 4) * 512 + (m % 32) * 16 + ((m % 128) / 32) * 4 + b % 4,
// i.e. one 512-byte atom per 128 rows and 64 k.  Rows M .. Mpad-1 get zero
// scales (Mpad = M rounded up to 256, the GEMM's token tile).
//
// The dynamic amax takes two launches and no memset: x_amax_partial_kernel
// writes one maximum per CTA into amax[1 ..], and every CTA of the quantizer
// reduces those before it starts (CTA 0 also stores the total in amax[0]).
constexpr int kXAmaxParts = 256;

__global__ void __launch_bounds__(256) x_amax_partial_kernel(const uint16_t* __restrict__ X, int64_t ldx, int64_t M,
                                                             int64_t K, float* __restrict__ amax) {
  __shared__ float red[8];
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t vpr = K / 8, total = M * vpr;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  float m = 0.0f;
  // eight 16-byte loads in flight per thread (one memory round trip for
  // tensors up to 8 x the grid's threads)
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total; t += 8 * stride) {
    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t u = t + i * stride;
      const int64_t r = u / vpr, c = (u - r * vpr) * 8;
      v[i] = u < total ? ld_stream_v4(X + r * ldx + c) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) m = absmax8(v[i], m);
  }
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w]);
    amax[1 + blockIdx.x] = m;
  }
}

// One thread per (row, 16-block) of the padded rows.  parts > 0: reduce
// amax[1 .. parts] first (dynamic); parts == 0: amax[0] is given.
__global__ void __launch_bounds__(256) quantize_x_mma_kernel(const uint16_t* __restrict__ X, int64_t ldx,
                                                             int64_t M, int64_t K, int64_t Mpad,
                                                             float* __restrict__ amax, int parts,
                                                             uint8_t* __restrict__ qx, uint8_t* __restrict__ sx) {
  __shared__ float s_amax;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (threadIdx.x < 32) {
    float m = 0.0f;
    if (parts > 0) {
      for (int i = threadIdx.x; i < parts; i += 32) m = fmaxf(m, amax[1 + i]);
      m = warp_max(m);
    } else {
      m = amax[0];
    }
    if (threadIdx.x == 0) {
      s_amax = m;
      if (parts > 0 && blockIdx.x == 0) amax[0] = m;
    }
  }
  __syncthreads();
  const float g = __fdiv_rn(s_amax, 2688.0f);
  const int64_t nb = K / 16, steps = K / 64;
  const int64_t total = Mpad * nb;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total; t += stride) {
    const int64_t m = t / nb, b = t - m * nb;
    uint32_t sc = 0;
    if (m < M) {
      const uint16_t* src = X + m * ldx + b * 16;
      uint2 codes;
      quantize_store_regs(ld_stream_v4(src), ld_stream_v4(src + 8), g, sc, codes);
      *reinterpret_cast<uint2*>(qx + m * (K / 2) + b * 8) = codes;
    }
    const int64_t r = m % 128;
    sx[((m / 128) * steps + b / 4) * 512 + (r % 32) * 16 + (r / 32) * 4 + (b % 4)] = (uint8_t)sc;
  }
}

int grid_for(int64_t work_items, int sms) {
  const int64_t blocks = (work_items + 255) / 256;
  const int64_t cap = (int64_t)sms * 8;
  return (int)(blocks < 1 ? 1 : (blocks < cap ? blocks : cap));
}

}  // namespace

cudaError_t launch_quantize_x_mma(const uint16_t* X, int64_t ldx, int64_t M, int64_t K, float* amax, bool given,
                                  uint8_t* qx, uint8_t* sx, cudaStream_t stream, int sms) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int64_t ldx_ = ldx, M_ = M, K_ = K;
  int parts = 0;
  if (!given) {
    const int64_t blocks = (M * (K / 8) + 255) / 256;
    parts = (int)(blocks < kXAmaxParts ? blocks : kXAmaxParts);
    cfg.gridDim = dim3(parts);
    void* args[] = {(void*)&X, (void*)&ldx_, (void*)&M_, (void*)&K_, (void*)&amax};
    cudaError_t e = cudaLaunchKernelExC(&cfg, (const void*)x_amax_partial_kernel, args);
    if (e != cudaSuccess) return e;
  }
  int64_t Mpad = (M + 255) / 256 * 256;
  const int64_t blocks = (Mpad * (K / 16) + 255) / 256;
  const int64_t cap = (int64_t)sms * 16;
  cfg.gridDim = dim3((unsigned)(blocks < cap ? blocks : cap));
  void* args[] = {(void*)&X, (void*)&ldx_, (void*)&M_, (void*)&K_, (void*)&Mpad, (void*)&amax, (void*)&parts,
                  (void*)&qx, (void*)&sx};
  return cudaLaunchKernelExC(&cfg, (const void*)quantize_x_mma_kernel, args);
}

cudaError_t launch_scales_to_mma(const uint8_t* s, int64_t N, int64_t K, uint8_t* s_mma, cudaStream_t stream,
                                 int sms) {
  const int64_t total = (N + 127) / 128 * (K / 64) * 32;
  scales_to_mma_kernel<<<grid_for(total, sms), 256, 0, stream>>>(s, N, K, s_mma);
  return cudaGetLastError();
}

cudaError_t launch_gemm_w4a4(const uint8_t* qx, const uint8_t* sx, const float* x_amax, const uint8_t* q,
                             const uint8_t* s_mma, const float* g, uint16_t* Y, int64_t ldy, int64_t M, int64_t N,
                             int64_t K, bool static_weights, bool pair, cudaStream_t stream, int sms) {
  CUtensorMap tw, tx;
  if (!tc::make_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, (uint64_t)(K / 2), (uint64_t)N, (uint64_t)(K / 2),
                        128u, (uint32_t)kBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !tc::make_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, qx, (uint64_t)(K / 2), (uint64_t)M, (uint64_t)(K / 2),
                        128u, (uint32_t)kBN, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  int m = (int)M, n = (int)N, k = (int)K, sw = static_weights ? 1 : 0;
  if (pair && sms >= 2) {
    // pairs of SMs: the token map's box is the 128 tokens one CTA of a pair loads
    // and the scale atoms as rows of 256 bytes (a stage's four atoms: 8 rows)
    CUtensorMap txh, tsa, tsb;
    const uint64_t sa_rows = (uint64_t)((N + kBM - 1) / kBM) * (uint64_t)(K / 64) * 2;
    const uint64_t sb_rows = (uint64_t)((M + kBN - 1) / kBN * 2) * (uint64_t)(K / 64) * 2;
    if (!tc::make_tmap_2d(&txh, CU_TENSOR_MAP_DATA_TYPE_UINT8, qx, (uint64_t)(K / 2), (uint64_t)M, (uint64_t)(K / 2),
                          128u, (uint32_t)(kBN / 2), CU_TENSOR_MAP_SWIZZLE_128B) ||
        !tc::make_tmap_2d(&tsa, CU_TENSOR_MAP_DATA_TYPE_UINT8, s_mma, 256u, sa_rows, 256u, 256u, 8u,
                          CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !tc::make_tmap_2d(&tsb, CU_TENSOR_MAP_DATA_TYPE_UINT8, sx, 256u, sb_rows, 256u, 256u, 8u,
                          CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
    static tc::SmemOptIn opt_in_pair;
    const cudaError_t e = opt_in_pair.ensure((const void*)gemm_w4a4_pair_kernel, kPairSmemBytes);
    if (e != cudaSuccess) return e;
    void* args[] = {&tw, &txh, &tsa, &tsb, (void*)&g, (void*)&x_amax, &Y, &ldy, &m, &n, &k, &sw};
    const int64_t tiles = (N + 2 * kBM - 1) / (2 * kBM) * ((M + kBN - 1) / kBN);
    const int64_t clusters = tiles < sms / 2 ? tiles : sms / 2;  // one persistent pair per two SMs at most
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * clusters));
    cfg.blockDim = dim3(kPairThreads);
    cfg.dynamicSmemBytes = kPairSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelExC(&cfg, (const void*)gemm_w4a4_pair_kernel, args);
  }
  static tc::SmemOptIn opt_in;
  const cudaError_t e = opt_in.ensure((const void*)gemm_w4a4_kernel, kSmemBytes);
  if (e != cudaSuccess) return e;
  void* args[] = {&tw, &tx, (void*)&s_mma, (void*)&sx, (void*)&g, (void*)&x_amax, &Y, &ldy, &m, &n, &k, &sw};
  const int64_t tiles = (N + kBM - 1) / kBM * ((M + kBN - 1) / kBN);
  const unsigned grid = (unsigned)(tiles < sms ? tiles : sms);  // one persistent CTA per SM at most
  return tc::launch_pdl((const void*)gemm_w4a4_kernel, dim3(grid), dim3(kThreads), kSmemBytes, stream, args);
}

cudaError_t read_and_clear_w4a4_timeouts(unsigned int* count) {
  cudaError_t e = cudaMemcpyFromSymbol(count, g_w4a4_wait_timeouts, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  const unsigned int zero = 0;
  return cudaMemcpyToSymbol(g_w4a4_wait_timeouts, &zero, sizeof(unsigned int));
}

}  // namespace nvfp4

// gemm_tc.cu -- W4A16 NVFP4 GEMM on the sm_100a tensor cores (tcgen05).
//
// Y[m, n] = bf16(g * sum_k W_deq[n, k] * X[m, k]) for the 32-user batched
// decode and the 512-token prefill of a 27B-class layer (model card
// "Qwen3.8-27B-NVFP4", "Measurements"; imp docs/quantization.md, "Dense layers"
// pipeline: the prefill GEMM reads the packed NVFP4 weights).  The pages'
// prefill runs a CUTLASS block-scaled FP4 x FP4 GEMM on sm_120; here the
// activations stay BF16 (weight-only quantization, "What is quantized"), so
// the weights are dequantized on chip and the contraction runs as a BF16
// tcgen05 MMA with fp32 accumulation in tensor memory.
//
// Tile: 128 weight rows (MMA M, "swap AB": weights are operand A) x BN
// activation rows (MMA N), 64 k per pipeline stage.  Per stage:
//   - warp 0 (one thread) issues two TMA tile loads into shared memory: the
//     BF16 X tile [BN, 64] with the 128-byte swizzle (the UMMA K-major layout)
//     and the packed W tile [128 rows, 32 bytes];
//   - warps 4..7 (one thread per weight row) turn the 32 packed bytes and 4
//     E4M3 scales of their row into 64 BF16 values e2m1 * e4m3 (exact in BF16)
//     and store them into the swizzled A tile;
//   - warp 1 (one thread) issues four 128 x BN x 16 MMAs into the TMEM
//     accumulator and commits them to the stage's "empty" barrier.
// After the last stage warps 4..7 read the accumulator from TMEM, apply the
// FP32 tensor scale g and store BF16 Y.  Every mbarrier wait is bounded.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdio>

#include "nvfp4_device.cuh"
#include "nvfp4_kernels.h"
#include "sm100_ptx.cuh"

namespace nvfp4 {

// Number of CTAs whose pipeline wait ran past its time limit (diagnostic).
__device__ unsigned int g_gemm_wait_timeouts = 0;

namespace {

constexpr int kBM = 128;            // weight rows per tile (MMA M)
constexpr int kBK = 64;             // k per stage: one 128-byte swizzle row of BF16
constexpr int kThreads = 256;
constexpr int kDeqWarp0 = 4;        // warps 4..7: dequantize, then epilogue
constexpr uint64_t kWaitLimitNs = 2000000000ull;

struct Bars {
  uint64_t full[8];   // TMA bytes of stage landed
  uint64_t deq[8];    // BF16 A tile of stage written (128 arrivals)
  uint64_t empty[8];  // MMAs reading the stage finished
  uint64_t tmem_full; // last MMA finished
  uint32_t tmem_addr;
  volatile int err;
};

template <int BN>
struct Cfg {
  static constexpr int kXBytes = BN * 128;
  static constexpr int kWdBytes = kBM * 128;
  static constexpr int kWrBytes = kBM * 32;
  static constexpr int kStageBytes = kXBytes + kWdBytes + kWrBytes;
  static constexpr int kStagesFit = (200 * 1024) / kStageBytes;
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  static constexpr int kSmemBytes = kStages * kStageBytes + (int)sizeof(Bars) + 1024;
  static constexpr uint32_t kTmemCols = BN < 32 ? 32 : BN;
  static constexpr uint32_t kIdesc = ptx::idesc_bf16_f32(kBM, BN);
  static_assert(kStages >= 2, "pipeline needs two stages");
  static_assert(BN % 16 == 0 && BN <= 256, "MMA N");
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

// Eight E2M1 codes (one 32-bit word, low nibble first) times an fp32 scale ->
// eight BF16 (exact: the products have at most 6 significant bits).
__device__ __forceinline__ uint4 dequant8_bf16(uint32_t word, float sc) {
  uint32_t o[4];
  const float2 p0 = f16x2_to_float2(e2m1x2_byte_to_f16x2<0>(word));
  const float2 p1 = f16x2_to_float2(e2m1x2_byte_to_f16x2<1>(word));
  const float2 p2 = f16x2_to_float2(e2m1x2_byte_to_f16x2<2>(word));
  const float2 p3 = f16x2_to_float2(e2m1x2_byte_to_f16x2<3>(word));
  const float2 s2 = make_float2(sc, sc);
  const float2 q0 = __fmul2_rn(p0, s2), q1 = __fmul2_rn(p1, s2), q2 = __fmul2_rn(p2, s2),
               q3 = __fmul2_rn(p3, s2);
  __nv_bfloat162 b0 = __floats2bfloat162_rn(q0.x, q0.y), b1 = __floats2bfloat162_rn(q1.x, q1.y),
                 b2 = __floats2bfloat162_rn(q2.x, q2.y), b3 = __floats2bfloat162_rn(q3.x, q3.y);
  o[0] = *reinterpret_cast<uint32_t*>(&b0);
  o[1] = *reinterpret_cast<uint32_t*>(&b1);
  o[2] = *reinterpret_cast<uint32_t*>(&b2);
  o[3] = *reinterpret_cast<uint32_t*>(&b3);
  return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
               : "memory");
  return v;
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                   const uint8_t* __restrict__ s, const float* __restrict__ g, uint16_t* __restrict__ Y,
                   int64_t ldy, int M, int N, int K) {
  using C = Cfg<BN>;
  constexpr int NS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  Bars* bars = reinterpret_cast<Bars*>(smem + NS * C::kStageBytes);
  auto x_tile = [&](int st) { return smem + st * C::kStageBytes; };
  auto wd_tile = [&](int st) { return smem + st * C::kStageBytes + C::kXBytes; };
  auto wr_tile = [&](int st) { return smem + st * C::kStageBytes + C::kXBytes + C::kWdBytes; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kBM, m0 = blockIdx.y * BN;
  const int num_kb = K / kBK;

  if (threadIdx.x == 0) {
    for (int st = 0; st < NS; ++st) {
      ptx::mbar_init(&bars->full[st], 1);
      ptx::mbar_init(&bars->deq[st], 128);
      ptx::mbar_init(&bars->empty[st], 1);
    }
    ptx::mbar_init(&bars->tmem_full, 1);
    bars->err = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tmap_x);
    ptx::prefetch_tmap(&tmap_w);
  }
  if (warp == 1) {
    ptx::tmem_alloc(&bars->tmem_addr, C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_addr;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      for (int kb = 0; kb < num_kb; ++kb) {
        const int st = kb % NS, round = kb / NS;
        if (round > 0 && !wait_or_fail(&bars->empty[st], (round - 1) & 1, bars)) break;
        ptx::mbar_arrive_expect_tx(&bars->full[st], C::kXBytes + C::kWrBytes);
        ptx::tma_load_2d(x_tile(st), &tmap_x, &bars->full[st], kb * kBK, m0);
        ptx::tma_load_2d(wr_tile(st), &tmap_w, &bars->full[st], kb * (kBK / 2), n0);
        ++issued;
      }
      if (bars->err) {
        // let the copies already issued land before the CTA exits
        for (int kb = issued > NS ? issued - NS : 0; kb < issued; ++kb)
          ptx::mbar_wait(&bars->full[kb % NS], (kb / NS) & 1, kWaitLimitNs);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int issued = 0;
      for (int kb = 0; kb < num_kb; ++kb) {
        const int st = kb % NS, round = kb / NS;
        if (!wait_or_fail(&bars->deq[st], round & 1, bars)) break;
        if (!wait_or_fail(&bars->full[st], round & 1, bars)) break;
        ptx::tc_fence_after();
        const uint32_t a0 = ptx::smem_u32(wd_tile(st)), b0 = ptx::smem_u32(x_tile(st));
#pragma unroll
        for (int j = 0; j < kBK / 16; ++j) {
          ptx::mma_bf16(tmem, ptx::sw128_kmajor_desc(a0 + 32 * j), ptx::sw128_kmajor_desc(b0 + 32 * j),
                        C::kIdesc, (kb | j) != 0);
        }
        ptx::mma_commit(&bars->empty[st]);
        ++issued;
      }
      // arrives when every MMA above is done (also on the error path, so that
      // TMEM is never freed under a running MMA)
      ptx::mma_commit(&bars->tmem_full);
      if (bars->err) ptx::mbar_wait(&bars->tmem_full, 0, kWaitLimitNs);
    }
  } else if (warp >= kDeqWarp0) {
    // ------------------------------------------------ dequantize, then epilogue
    const int t = threadIdx.x - kDeqWarp0 * 32;  // weight row within the tile
    const int row = n0 + t;
    const bool row_ok = row < N;
    const uint8_t* srow = s + (int64_t)(row_ok ? row : 0) * (K / 16);
    const uint32_t swz = (uint32_t)(t & 7);
    for (int kb = 0; kb < num_kb; ++kb) {
      const int st = kb % NS, round = kb / NS;
      const uint32_t sc4 = row_ok ? *reinterpret_cast<const uint32_t*>(srow + kb * 4) : 0u;
      if (!wait_or_fail(&bars->full[st], round & 1, bars)) break;
      const uint32_t src = ptx::smem_u32(wr_tile(st)) + t * 32;
      const uint4 c0 = ld_shared_v4(src), c1 = ld_shared_v4(src + 16);
      const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      const float2 sa = f16x2_to_float2(e4m3x2_to_f16x2(sc4 & 0xFFFFu));
      const float2 sb = f16x2_to_float2(e4m3x2_to_f16x2(sc4 >> 16));
      const float scl[4] = {sa.x, sa.y, sb.x, sb.y};
      const uint32_t dst = ptx::smem_u32(wd_tile(st)) + t * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) st_shared_v4(dst + ((c ^ swz) << 4), dequant8_bf16(words[c], scl[c >> 1]));
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(&bars->deq[st]);
    }
    // epilogue: TMEM lane (32 * (warp % 4) + lane) holds weight row n, columns = m
    const bool acc_ready = __all_sync(0xFFFFFFFFu, wait_or_fail(&bars->tmem_full, 0, bars));
    if (acc_ready) {
      ptx::tc_fence_after();
      const int q = warp & 3;
      const int n = n0 + 32 * q + lane;
      const float gv = *g;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t r[32];
        ptx::tmem_ld_32cols(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, r);
        ptx::tmem_ld_wait();
        if (n < N) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int m = m0 + c0 + j;
            if (c0 + j < BN && m < M) {
              const __nv_bfloat16 o = __float2bfloat16_rn(__uint_as_float(r[j]) * gv);
              Y[(int64_t)m * ldy + n] = *reinterpret_cast<const uint16_t*>(&o);
            }
          }
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

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

template <int BN>
cudaError_t launch_bn(const uint16_t* X, int64_t ldx, const uint8_t* q, const uint8_t* s, const float* g,
                      uint16_t* Y, int64_t ldy, int M, int N, int K, cudaStream_t stream) {
  using C = Cfg<BN>;
  auto enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap tx, tw;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)ldx * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)BN};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(X), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)N};
    const cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    const cuuint32_t box[2] = {(cuuint32_t)(kBK / 2), (cuuint32_t)kBM};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(q), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  static bool attr_set[64] = {};  // per device ordinal
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(gemm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  dim3 grid((N + kBM - 1) / kBM, (M + BN - 1) / BN);
  gemm_tc_kernel<BN><<<grid, kThreads, C::kSmemBytes, stream>>>(tx, tw, s, g, Y, ldy, M, N, K);
  return cudaGetLastError();
}

}  // namespace

bool gemm_tc_supported(int64_t M, int64_t N, int64_t K) {
  return M >= 2 && N >= 1 && K % 256 == 0 && K <= (int64_t)1 << 30 && N <= ((int64_t)1 << 31) - 128 &&
         M <= ((int64_t)1 << 31) - 256;
}

cudaError_t launch_gemm_tc(const uint16_t* X, int64_t ldx, const uint8_t* q, const uint8_t* s, const float* g,
                           uint16_t* Y, int64_t ldy, int64_t M, int64_t N, int64_t K, cudaStream_t stream) {
  const int m = (int)M, n = (int)N, k = (int)K;
  if (M <= 16) return launch_bn<16>(X, ldx, q, s, g, Y, ldy, m, n, k, stream);
  if (M <= 32) return launch_bn<32>(X, ldx, q, s, g, Y, ldy, m, n, k, stream);
  if (M <= 64) return launch_bn<64>(X, ldx, q, s, g, Y, ldy, m, n, k, stream);
  if (M <= 128) return launch_bn<128>(X, ldx, q, s, g, Y, ldy, m, n, k, stream);
  return launch_bn<256>(X, ldx, q, s, g, Y, ldy, m, n, k, stream);
}

cudaError_t read_and_clear_gemm_timeouts(unsigned int* count) {
  cudaError_t e = cudaMemcpyFromSymbol(count, g_gemm_wait_timeouts, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  const unsigned int zero = 0;
  return cudaMemcpyToSymbol(g_gemm_wait_timeouts, &zero, sizeof(unsigned int));
}

}  // namespace nvfp4

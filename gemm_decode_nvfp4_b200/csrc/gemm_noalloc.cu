// gemm_noalloc.cu -- nvfp4_gemm_noalloc: the GEMM of nvfp4_gemm with its
// scratch taken from a fixed array compiled into this library instead of a
// caller-supplied workspace.
//
// Who needs it: a caller that has no device allocator of its own to hand (a
// plain C host program driving the library through the C ABI, with no memory
// pool), or one that must not allocate while it runs a step (a serving engine
// that reserved HBM up front and whose allocator is closed for the step; an
// allocation there can also synchronize the device).  Such a caller still gets
// the tensor-core path, which needs a per-call f16 copy of X and the row
// exponents, up to the size limit below.
//
// The array is one per device (a __device__ variable has an instance in every
// device context the library is loaded into) and every call on that device
// shares it, so it keeps whatever the last call left there.  Nothing in it
// needs to start at zero: the GEMM's pre-pass writes every byte the GEMM then
// reads (the exponent of each row of X and its f16 copy) before that read.
// Two calls whose work overlaps on the GPU (different streams with no ordering
// between them, or host threads racing on one device) use the same bytes and
// race; calls must be ordered, e.g. issued on one stream.
//
// Set-up: the first call in each CUDA context (normally a device's primary
// context), with that context current, looks up the array's device address
// with cudaGetSymbolAddress (the host-side name of a __device__ array is not a
// device address) and caches it under the context's unique id.  A later call
// in another context (after cudaDeviceReset, or when the caller made a
// different context current) looks it up again instead of reusing an address
// of a context that may be gone.  Make the first call in a context before any
// stream capture in it begins.  Nothing here calls cudaMalloc, cudaFree or any
// other allocating routine.
#include <mutex>

#include "nvfp4.h"
#include "nvfp4_kernels.h"
#include "tc_host.h"

namespace {

constexpr size_t kScratchBytes = NVFP4_GEMM_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxContexts = 64;

}  // namespace

// Scratch of the tensor-core GEMM: the row exponents, then the f16 copy of X.
static __device__ __align__(256) unsigned char g_gemm_scratch[kScratchBytes];

namespace {

// Address of g_gemm_scratch per context id; a context's entry is replaced when
// its slot is reused after kMaxContexts others.
struct ScratchSlot {
  unsigned long long ctx;
  void* ptr;
};
std::mutex g_setup_mutex;
ScratchSlot g_slots[kMaxContexts];
int g_used = 0, g_next = 0;

// Device address of g_gemm_scratch in the context current on this thread.
nvfp4_status scratch_for_current_context(void** out) {
  unsigned long long ctx = 0;
  cudaError_t e = nvfp4::tc::current_context_id(&ctx);
  if (e != cudaSuccess) return nvfp4::report_cuda_error(e, "reading the current CUDA context");
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  for (int i = 0; i < g_used; ++i)
    if (ctx != 0 && g_slots[i].ctx == ctx) {
      *out = g_slots[i].ptr;
      return NVFP4_OK;
    }
  // (with no context current yet, this creates the device's primary context)
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_gemm_scratch);
  if (e != cudaSuccess || !p)
    return nvfp4::report_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidSymbol,
                                    "cudaGetSymbolAddress of the built-in GEMM scratch");
  if (ctx == 0 && (e = nvfp4::tc::current_context_id(&ctx)) != cudaSuccess)
    return nvfp4::report_cuda_error(e, "reading the current CUDA context");
  g_slots[g_used < kMaxContexts ? g_used++ : (g_next++ % kMaxContexts)] = {ctx, p};
  *out = p;
  return NVFP4_OK;
}

}  // namespace

NVFP4_API nvfp4_status nvfp4_gemm_noalloc(const uint16_t* X, int64_t ldx, const uint8_t* q, const uint8_t* s,
                                           const float* g, uint16_t* Y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                                           uint32_t flags, nvfp4_stream_t stream) {
  // the shape checks of nvfp4_gemm_ex, first, so that a bad shape gets the same status here
  if (K <= 0 || K % 16 != 0)
    return nvfp4::report_error(NVFP4_ERR_SHAPE, "K=%lld must be a positive multiple of 16", (long long)K);
  if (M < 0 || N < 0)
    return nvfp4::report_error(NVFP4_ERR_SHAPE, "negative size M=%lld N=%lld", (long long)M, (long long)N);
  const size_t need = nvfp4_gemm_workspace_size(M, N, K);
  if (need > kScratchBytes) {
    return nvfp4::report_error(NVFP4_ERR_WORKSPACE,
                               "M=%lld K=%lld needs %zu bytes of scratch; the built-in scratch of "
                               "nvfp4_gemm_noalloc holds %zu (enough for M <= 1024 with M*K <= 2^22); use nvfp4_gemm "
                               "with a workspace",
                               (long long)M, (long long)K, need, kScratchBytes);
  }
  void* scratch = nullptr;
  const nvfp4_status st = scratch_for_current_context(&scratch);
  if (st != NVFP4_OK) return st;
  return nvfp4_gemm_ex(X, ldx, q, s, g, Y, ldy, M, N, K, scratch, kScratchBytes, flags, stream);
}

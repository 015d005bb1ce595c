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
// Set-up: the first call on each device, with that device current, looks up
// the array's device address with cudaGetSymbolAddress (the host-side name of
// a __device__ array is not a device address) and caches it.  Make that first
// call before any stream capture on the device begins.  Nothing here calls
// cudaMalloc, cudaFree or any other allocating routine.
#include <atomic>
#include <mutex>

#include "nvfp4.h"
#include "nvfp4_kernels.h"

namespace {

constexpr size_t kScratchBytes = NVFP4_GEMM_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

}  // namespace

// Scratch of the tensor-core GEMM: the row exponents, then the f16 copy of X.
static __device__ __align__(256) unsigned char g_gemm_scratch[kScratchBytes];

namespace {

std::mutex g_setup_mutex;
std::atomic<void*> g_scratch_ptr[kMaxDevices];

// Device address of g_gemm_scratch on the current device (set up once).
nvfp4_status scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return nvfp4::report_cuda_error(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return nvfp4::report_error(NVFP4_ERR_UNSUPPORTED, "device ordinal %d", dev);
  void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (!p) {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
    if (!p) {
      e = cudaGetSymbolAddress(&p, g_gemm_scratch);
      if (e != cudaSuccess || !p) {
        return nvfp4::report_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidSymbol,
                                        "cudaGetSymbolAddress of the built-in GEMM scratch");
      }
      g_scratch_ptr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return NVFP4_OK;
}

}  // namespace

NVFP4_API nvfp4_status nvfp4_gemm_noalloc(const uint16_t* X, int64_t ldx, const uint8_t* q, const uint8_t* s,
                                           const float* g, uint16_t* Y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                                           uint32_t flags, nvfp4_stream_t stream) {
  const size_t need = nvfp4_gemm_workspace_size(M, N, K);
  if (need > kScratchBytes) {
    return nvfp4::report_error(NVFP4_ERR_WORKSPACE,
                               "M=%lld K=%lld needs %zu bytes of scratch; the built-in scratch of "
                               "nvfp4_gemm_noalloc holds %zu (enough for M <= 1024 with M*K <= 2^22); use nvfp4_gemm "
                               "with a workspace",
                               (long long)M, (long long)K, need, kScratchBytes);
  }
  void* scratch = nullptr;
  const nvfp4_status st = scratch_for_current_device(&scratch);
  if (st != NVFP4_OK) return st;
  return nvfp4_gemm_ex(X, ldx, q, s, g, Y, ldy, M, N, K, scratch, kScratchBytes, flags, stream);
}

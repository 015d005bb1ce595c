// tc_host.h -- host-side helpers shared by the kernel launchers: TMA
// tensor-map encoding (through the driver entry point, no libcuda link),
// kernel launch with programmatic dependent launch enabled, and per-context
// state that several host threads may set up at once.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

namespace nvfp4 {
namespace tc {

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  // (a function-local static is initialised once, also under concurrent first calls)
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
  }();
  return fn;
}

// 2-D row-major tensor [outer, inner] with `row_bytes` between rows, copied in
// boxes of [box_outer, box_inner]; out-of-range elements read as zero.
inline bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType type, const void* base, uint64_t inner,
                         uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                         CUtensorMapSwizzle swizzle) {
  auto enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, type, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D row-major tensor [depth, outer, inner] (`row_bytes` between rows,
// `plane_bytes` between planes), copied in boxes of [1, box_outer, box_inner].
inline bool make_tmap_3d(CUtensorMap* map, CUtensorMapDataType type, const void* base, uint64_t inner,
                         uint64_t outer, uint64_t depth, uint64_t row_bytes, uint64_t plane_bytes,
                         uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  auto enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)outer, (cuuint64_t)depth};
  const cuuint64_t strides[2] = {(cuuint64_t)row_bytes, (cuuint64_t)plane_bytes};
  const cuuint32_t box[3] = {box_inner, box_outer, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, type, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel on the stream is finishing (it orders itself with
// griddepcontrol.wait).
inline cudaError_t launch_pdl(const void* func, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              void** args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, func, args);
}

// Unique id of the CUDA context current on this host thread, 0 when none is
// current yet (cuCtxGetCurrent / cuCtxGetId through the driver entry points).
// Ids are never reused, so state keyed by them cannot outlive its context
// (cudaDeviceReset, or a caller that makes another context current).
inline cudaError_t current_context_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (!get_current || !get_id) return cudaErrorNotSupported;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  *id = 0;
  if (ctx && get_id(ctx, id) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  return cudaSuccess;
}

// The largest dynamic shared memory a kernel has been allowed
// (cudaFuncAttributeMaxDynamicSharedMemorySize) in each context it ran in.
// The attribute belongs to the kernel's module in one context, so it is
// recorded per context id; the limit only ever grows, under a lock, so a
// launch that needs less never lowers the limit another thread set for a
// larger one.
class SmemOptIn {
 public:
  cudaError_t ensure(const void* func, int bytes) {
    unsigned long long ctx = 0;
    cudaError_t e = current_context_id(&ctx);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu_);
    for (int i = 0; i < used_; ++i)
      if (ctx != 0 && slot_[i].ctx == ctx && slot_[i].bytes >= bytes) return cudaSuccess;
    // (this also creates the device's primary context when none was current)
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    if (ctx == 0 && (e = current_context_id(&ctx)) != cudaSuccess) return e;
    for (int i = 0; i < used_; ++i)
      if (slot_[i].ctx == ctx) {
        slot_[i].bytes = bytes > slot_[i].bytes ? bytes : slot_[i].bytes;
        return cudaSuccess;
      }
    slot_[used_ < kSlots ? used_++ : (next_++ % kSlots)] = {ctx, bytes};
    return cudaSuccess;
  }

 private:
  static constexpr int kSlots = 64;
  struct Slot {
    unsigned long long ctx;
    int bytes;
  };
  std::mutex mu_;
  Slot slot_[kSlots] = {};
  int used_ = 0, next_ = 0;
};

}  // namespace tc
}  // namespace nvfp4

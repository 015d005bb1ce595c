// abi.cu -- the extern "C" entry points of include/nvfp4.h: host-side argument
// validation, device capability check and dispatch to the kernels.  Nothing
// here allocates device memory or synchronizes.
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "mxfp4.h"
#include "nvfp4.h"
#include "nvfp4_kernels.h"
#include "nvfp4_w4a4.h"

namespace {

thread_local char t_last_error[512] = "";

nvfp4_status fail(nvfp4_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
  va_end(ap);
  return st;
}

nvfp4_status cuda_fail(cudaError_t e, const char* what) {
  return fail(NVFP4_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool aligned2(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 1u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
  return na && nb && pa < pb + nb && pb < pa + na;
}

constexpr uint32_t kKnownFlags = NVFP4_FLAG_STATIC_WEIGHTS;
constexpr uint32_t kGemvFlags = NVFP4_FLAG_STATIC_WEIGHTS | NVFP4_FLAG_KSPLIT_MASK;
constexpr uint32_t kW4a4Flags = NVFP4_FLAG_STATIC_WEIGHTS | NVFP4_FLAG_W4A4_PAIR;

// The K split a decode GEMV call asks for (0 = the library's choice), or -1
// for a value other than 1, 2, 4, 8.
int ksplit_of(uint32_t flags) {
  const int c = (int)((flags & NVFP4_FLAG_KSPLIT_MASK) >> 8);
  return (c == 0 || c == 1 || c == 2 || c == 4 || c == 8) ? c : -1;
}

constexpr int kMaxDevices = 64;
int g_dev_state[kMaxDevices];  // 0 unknown, 1 ok, 2 unsupported
int g_dev_sms[kMaxDevices];

// The current device must be a B200-class part (compute capability 10.0).
nvfp4_status check_device(int* sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(NVFP4_ERR_UNSUPPORTED, "device ordinal %d", dev);
  if (g_dev_state[dev] == 0) {
    int major = 0, minor = 0, n = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    g_dev_sms[dev] = n;
    g_dev_state[dev] = (major == 10 && minor == 0) ? 1 : 2;
    if (g_dev_state[dev] == 2)
      return fail(NVFP4_ERR_UNSUPPORTED, "device %d has compute capability %d.%d; this library is built for sm_100a",
                  dev, major, minor);
  }
  if (g_dev_state[dev] == 2) return fail(NVFP4_ERR_UNSUPPORTED, "device %d is not sm_100", dev);
  *sms = g_dev_sms[dev];
  return NVFP4_OK;
}

nvfp4_status check_k(int64_t K) {
  if (K <= 0 || K % 16 != 0) return fail(NVFP4_ERR_SHAPE, "K=%lld must be a positive multiple of 16", (long long)K);
  return NVFP4_OK;
}

}  // namespace

nvfp4_status nvfp4::report_error(nvfp4_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
  va_end(ap);
  return st;
}

nvfp4_status nvfp4::report_cuda_error(cudaError_t e, const char* what) { return cuda_fail(e, what); }

extern "C" {

int nvfp4_version(void) { return 100; }

const char* nvfp4_last_error(void) { return t_last_error; }

const char* nvfp4_status_string(nvfp4_status st) {
  switch (st) {
    case NVFP4_OK: return "NVFP4_OK";
    case NVFP4_ERR_INVALID_ARG: return "NVFP4_ERR_INVALID_ARG";
    case NVFP4_ERR_SHAPE: return "NVFP4_ERR_SHAPE";
    case NVFP4_ERR_ALIGNMENT: return "NVFP4_ERR_ALIGNMENT";
    case NVFP4_ERR_UNSUPPORTED: return "NVFP4_ERR_UNSUPPORTED";
    case NVFP4_ERR_CUDA: return "NVFP4_ERR_CUDA";
    case NVFP4_ERR_WORKSPACE: return "NVFP4_ERR_WORKSPACE";
    case NVFP4_ERR_TIMEOUT: return "NVFP4_ERR_TIMEOUT";
  }
  return "NVFP4_ERR_UNKNOWN";
}

nvfp4_status nvfp4_amax(const uint16_t* w, int64_t rows, int64_t cols, int64_t ldw,
                        float* amax_inout, nvfp4_stream_t stream) {
  if (rows < 0 || cols < 0) return fail(NVFP4_ERR_SHAPE, "negative size rows=%lld cols=%lld", (long long)rows, (long long)cols);
  if (cols % 8 != 0) return fail(NVFP4_ERR_SHAPE, "cols=%lld must be a multiple of 8", (long long)cols);
  if (rows == 0 || cols == 0) return NVFP4_OK;
  if (!w || !amax_inout) return fail(NVFP4_ERR_INVALID_ARG, "null pointer (w=%p amax=%p)", (const void*)w, (void*)amax_inout);
  if (ldw < cols) return fail(NVFP4_ERR_INVALID_ARG, "ldw=%lld < cols=%lld", (long long)ldw, (long long)cols);
  if (!aligned16(w) || ldw % 8 != 0) return fail(NVFP4_ERR_ALIGNMENT, "w must be 16-byte aligned and ldw a multiple of 8");
  if (!aligned4(amax_inout)) return fail(NVFP4_ERR_ALIGNMENT, "amax must be 4-byte aligned");
  int sms = 0;
  nvfp4_status st = check_device(&sms);
  if (st != NVFP4_OK) return st;
  cudaError_t e = nvfp4::launch_amax(w, rows, cols, ldw, amax_inout, (cudaStream_t)stream, sms);
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "amax launch");
}

}  // extern "C"

namespace {

// nvfp4_quantize (window < 0) and nvfp4_quantize_mse (window >= 0): same
// arguments, same checks, the same amax handling.
nvfp4_status quantize_any(const uint16_t* w, int64_t N, int64_t K, int64_t ldw, const float* amax, uint8_t* q,
                          uint8_t* s, float* g_out, nvfp4_stream_t stream, int window) {
  nvfp4_status st = check_k(K);
  if (st != NVFP4_OK) return st;
  if (N < 0) return fail(NVFP4_ERR_SHAPE, "N=%lld < 0", (long long)N);
  if (!amax && !g_out) return fail(NVFP4_ERR_INVALID_ARG, "amax and g_out are both NULL");
  if (amax && g_out && (const void*)amax == (const void*)g_out)
    return fail(NVFP4_ERR_INVALID_ARG, "amax must not alias g_out");
  if (N > 0 && (!w || !q || !s)) return fail(NVFP4_ERR_INVALID_ARG, "null tensor pointer");
  if (N > 0 && ldw < K) return fail(NVFP4_ERR_INVALID_ARG, "ldw=%lld < K=%lld", (long long)ldw, (long long)K);
  if (N > 0 && (!aligned16(w) || !aligned16(q) || !aligned16(s) || ldw % 8 != 0))
    return fail(NVFP4_ERR_ALIGNMENT, "w, q, s must be 16-byte aligned and ldw a multiple of 8");
  if ((amax && !aligned4(amax)) || (g_out && !aligned4(g_out)))
    return fail(NVFP4_ERR_ALIGNMENT, "amax and g_out must be 4-byte aligned");
  if (N > 0) {
    const size_t wb = (size_t)((N - 1) * ldw + K) * 2, qb = (size_t)(N * K / 2), sb = (size_t)(N * K / 16);
    if (overlaps(w, wb, q, qb) || overlaps(w, wb, s, sb) || overlaps(q, qb, s, sb) ||
        (g_out && (overlaps(g_out, 4, q, qb) || overlaps(g_out, 4, s, sb) || overlaps(g_out, 4, w, wb))))
      return fail(NVFP4_ERR_INVALID_ARG, "w, q, s and g_out must not overlap");
  }
  int sms = 0;
  st = check_device(&sms);
  if (st != NVFP4_OK) return st;
  cudaStream_t cs = (cudaStream_t)stream;
  cudaError_t e;
  auto quant = [&](const float* a, float* gout) {
    return window < 0 ? nvfp4::launch_quantize(w, N, K, ldw, a, q, s, gout, cs, sms)
                      : nvfp4::launch_quantize_mse(w, N, K, ldw, a, window, q, s, gout, cs, sms);
  };
  if (amax) {
    e = quant(amax, g_out);
    return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "quantize launch");
  }
  // g_out first accumulates this tensor's amax, then is overwritten with g.
  if ((e = cudaMemsetAsync(g_out, 0, sizeof(float), cs)) != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  if (N > 0 && (e = nvfp4::launch_amax(w, N, K, ldw, g_out, cs, sms)) != cudaSuccess) return cuda_fail(e, "amax launch");
  if ((e = quant(g_out, nullptr)) != cudaSuccess) return cuda_fail(e, "quantize launch");
  if ((e = nvfp4::launch_finalize_scale(g_out, cs)) != cudaSuccess) return cuda_fail(e, "finalize launch");
  return NVFP4_OK;
}

}  // namespace

extern "C" {

nvfp4_status nvfp4_quantize(const uint16_t* w, int64_t N, int64_t K, int64_t ldw,
                            const float* amax, uint8_t* q, uint8_t* s, float* g_out,
                            nvfp4_stream_t stream) {
  return quantize_any(w, N, K, ldw, amax, q, s, g_out, stream, -1);
}

nvfp4_status nvfp4_quantize_mse(const uint16_t* w, int64_t N, int64_t K, int64_t ldw, const float* amax,
                                int32_t window, uint8_t* q, uint8_t* s, float* g_out, nvfp4_stream_t stream) {
  if (window < 0 || window > 125)
    return fail(NVFP4_ERR_INVALID_ARG, "window=%d must be in 0..125 (E4M3 codes either side)", (int)window);
  return quantize_any(w, N, K, ldw, amax, q, s, g_out, stream, window);
}

nvfp4_status nvfp4_gemv(const uint16_t* x, const uint8_t* q, const uint8_t* s, const float* g,
                        uint16_t* y, int64_t N, int64_t K, nvfp4_stream_t stream) {
  return nvfp4_gemv_ex(x, q, s, g, y, N, K, 0u, stream);
}

nvfp4_status nvfp4_gemv_ex(const uint16_t* x, const uint8_t* q, const uint8_t* s, const float* g,
                           uint16_t* y, int64_t N, int64_t K, uint32_t flags, nvfp4_stream_t stream) {
  if (flags & ~kGemvFlags) return fail(NVFP4_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  const int splits = ksplit_of(flags);
  if (splits < 0) return fail(NVFP4_ERR_INVALID_ARG, "NVFP4_FLAG_KSPLIT(c) needs c in {1, 2, 4, 8}");
  nvfp4_status st = check_k(K);
  if (st != NVFP4_OK) return st;
  if (N < 0) return fail(NVFP4_ERR_SHAPE, "N=%lld < 0", (long long)N);
  if (K > nvfp4::kGemvMaxK) return fail(NVFP4_ERR_SHAPE, "K=%lld exceeds the GEMV limit %lld", (long long)K, (long long)nvfp4::kGemvMaxK);
  if (N > (int64_t)0x3FFFFFFF) return fail(NVFP4_ERR_SHAPE, "N=%lld too large", (long long)N);
  if (N == 0) return NVFP4_OK;
  if (!x || !q || !s || !g || !y) return fail(NVFP4_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(q) || !aligned16(s))
    return fail(NVFP4_ERR_ALIGNMENT, "x, q, s must be 16-byte aligned");
  if (!aligned2(y)) return fail(NVFP4_ERR_ALIGNMENT, "y must be 2-byte aligned");
  if (!aligned4(g)) return fail(NVFP4_ERR_ALIGNMENT, "g must be 4-byte aligned");
  const size_t yb = (size_t)N * 2;
  if (overlaps(y, yb, x, (size_t)K * 2) || overlaps(y, yb, q, (size_t)(N * K / 2)) ||
      overlaps(y, yb, s, (size_t)(N * K / 16)) || overlaps(y, yb, g, 4))
    return fail(NVFP4_ERR_INVALID_ARG, "y must not overlap x, q, s or g");
  int sms = 0;
  st = check_device(&sms);
  if (st != NVFP4_OK) return st;
  const bool static_w = (flags & NVFP4_FLAG_STATIC_WEIGHTS) != 0;
  if (splits > 1 && !nvfp4::gemv_split_fits(N, K, sms, false, splits))
    return fail(NVFP4_ERR_SHAPE, "a K split of %d does not fit N=%lld K=%lld (it needs K %% 256 == 0, at least %d "
                "512-element columns, and at most 11520 elements of x per CTA)", splits, (long long)N, (long long)K,
                splits);
  cudaError_t e;
  e = nvfp4::launch_gemv(x, q, s, g, y, N, K, sms, static_w, (cudaStream_t)stream, splits);
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "gemv launch");
}

nvfp4_status nvfp4_gemv_grouped(const uint16_t* X, int64_t ldx, const uint8_t* q, const uint8_t* s,
                                const float* g, const int32_t* expert_ids, const int32_t* token_ids, uint16_t* Y,
                                int64_t ldy, int64_t P, int64_t E, int64_t T, int64_t N, int64_t K, uint32_t flags,
                                nvfp4_stream_t stream) {
  if (flags & ~kKnownFlags) return fail(NVFP4_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  nvfp4_status st = check_k(K);
  if (st != NVFP4_OK) return st;
  if (P < 0 || E < 1 || T < 1 || N < 0)
    return fail(NVFP4_ERR_SHAPE, "P=%lld E=%lld T=%lld N=%lld: need P >= 0, E >= 1, T >= 1, N >= 0", (long long)P,
                (long long)E, (long long)T, (long long)N);
  if (P > 65535) return fail(NVFP4_ERR_SHAPE, "P=%lld exceeds 65535 problems per call", (long long)P);
  if (K > nvfp4::kGemvMaxK) return fail(NVFP4_ERR_SHAPE, "K=%lld exceeds the GEMV limit %lld", (long long)K, (long long)nvfp4::kGemvMaxK);
  if (N > (int64_t)0x3FFFFFFF || E > (int64_t)0x7FFFFFFF || T > (int64_t)0x7FFFFFFF)
    return fail(NVFP4_ERR_SHAPE, "N, E or T too large");
  if (P == 0 || N == 0) return NVFP4_OK;
  if (!X || !q || !s || !g || !expert_ids || !token_ids || !Y) return fail(NVFP4_ERR_INVALID_ARG, "null pointer");
  if (ldx < K || ldy < N) return fail(NVFP4_ERR_INVALID_ARG, "ldx=%lld < K or ldy=%lld < N", (long long)ldx, (long long)ldy);
  if (!aligned16(X) || ldx % 8 != 0 || !aligned16(q) || !aligned16(s))
    return fail(NVFP4_ERR_ALIGNMENT, "X, q, s must be 16-byte aligned and ldx a multiple of 8");
  if (!aligned2(Y) || !aligned4(g) || !aligned4(expert_ids) || !aligned4(token_ids))
    return fail(NVFP4_ERR_ALIGNMENT, "Y needs 2-byte, g and the id arrays 4-byte alignment");
  const size_t yb = (size_t)((P - 1) * ldy + N) * 2;
  if (overlaps(Y, yb, X, (size_t)((T - 1) * ldx + K) * 2) || overlaps(Y, yb, q, (size_t)(E * N * K / 2)) ||
      overlaps(Y, yb, s, (size_t)(E * N * K / 16)) || overlaps(Y, yb, g, (size_t)E * 4) ||
      overlaps(Y, yb, expert_ids, (size_t)P * 4) || overlaps(Y, yb, token_ids, (size_t)P * 4))
    return fail(NVFP4_ERR_INVALID_ARG, "Y must not overlap the inputs");
  int sms = 0;
  st = check_device(&sms);
  if (st != NVFP4_OK) return st;
  cudaError_t e = nvfp4::launch_gemv_grouped(X, ldx, q, s, g, expert_ids, token_ids, Y, ldy, P, E, T, N, K, sms,
                                             (cudaStream_t)stream);
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "grouped gemv launch");
}

nvfp4_status mxfp4_quantize(const uint16_t* w, int64_t N, int64_t K, int64_t ldw, uint8_t* q, uint8_t* s,
                            nvfp4_stream_t stream) {
  if (K <= 0 || K % 32 != 0) return fail(NVFP4_ERR_SHAPE, "K=%lld must be a positive multiple of 32", (long long)K);
  if (N < 0) return fail(NVFP4_ERR_SHAPE, "N=%lld < 0", (long long)N);
  if (N == 0) return NVFP4_OK;
  if (!w || !q || !s) return fail(NVFP4_ERR_INVALID_ARG, "null tensor pointer");
  if (ldw < K) return fail(NVFP4_ERR_INVALID_ARG, "ldw=%lld < K=%lld", (long long)ldw, (long long)K);
  if (!aligned16(w) || !aligned16(q) || !aligned16(s) || ldw % 8 != 0)
    return fail(NVFP4_ERR_ALIGNMENT, "w, q, s must be 16-byte aligned and ldw a multiple of 8");
  const size_t wb = (size_t)((N - 1) * ldw + K) * 2, qb = (size_t)(N * K / 2), sb = (size_t)(N * K / 32);
  if (overlaps(w, wb, q, qb) || overlaps(w, wb, s, sb) || overlaps(q, qb, s, sb))
    return fail(NVFP4_ERR_INVALID_ARG, "w, q and s must not overlap");
  int sms = 0;
  nvfp4_status st = check_device(&sms);
  if (st != NVFP4_OK) return st;
  cudaError_t e = nvfp4::launch_mx_quantize(w, N, K, ldw, q, s, (cudaStream_t)stream, sms);
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "mxfp4 quantize launch");
}

nvfp4_status mxfp4_to_nvfp4_scales(const uint8_t* q, const uint8_t* s_mx, int64_t N, int64_t K, uint8_t* s_nv,
                                   float* g_out, nvfp4_stream_t stream) {
  if (K <= 0 || K % 32 != 0) return fail(NVFP4_ERR_SHAPE, "K=%lld must be a positive multiple of 32", (long long)K);
  if (N < 0) return fail(NVFP4_ERR_SHAPE, "N=%lld < 0", (long long)N);
  if (N == 0) return NVFP4_OK;
  if (!q || !s_mx || !s_nv || !g_out) return fail(NVFP4_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(s_mx) || !aligned16(s_nv) || !aligned4(g_out))
    return fail(NVFP4_ERR_ALIGNMENT, "q, s_mx, s_nv must be 16-byte and g_out 4-byte aligned");
  const size_t qb = (size_t)(N * K / 2), mb = (size_t)(N * K / 32), nb = (size_t)(N * K / 16);
  if (overlaps(s_nv, nb, q, qb) || overlaps(s_nv, nb, s_mx, mb) || overlaps(g_out, 4, q, qb) ||
      overlaps(g_out, 4, s_mx, mb) || overlaps(g_out, 4, s_nv, nb))
    return fail(NVFP4_ERR_INVALID_ARG, "s_nv and g_out must not overlap the inputs or each other");
  int sms = 0;
  nvfp4_status st = check_device(&sms);
  if (st != NVFP4_OK) return st;
  cudaError_t e = nvfp4::launch_mx_to_nvfp4(q, s_mx, N, K, s_nv, g_out, (cudaStream_t)stream, sms);
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "mxfp4 scale conversion launch");
}

nvfp4_status mxfp4_gemv(const uint16_t* x, const uint8_t* q, const uint8_t* s, uint16_t* y, int64_t N,
                        int64_t K, nvfp4_stream_t stream) {
  return mxfp4_gemv_ex(x, q, s, y, N, K, 0u, stream);
}

nvfp4_status mxfp4_gemv_ex(const uint16_t* x, const uint8_t* q, const uint8_t* s, uint16_t* y, int64_t N,
                           int64_t K, uint32_t flags, nvfp4_stream_t stream) {
  if (flags & ~kGemvFlags) return fail(NVFP4_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  const int splits = ksplit_of(flags);
  if (splits < 0) return fail(NVFP4_ERR_INVALID_ARG, "NVFP4_FLAG_KSPLIT(c) needs c in {1, 2, 4, 8}");
  if (K <= 0 || K % 32 != 0) return fail(NVFP4_ERR_SHAPE, "K=%lld must be a positive multiple of 32", (long long)K);
  if (N < 0) return fail(NVFP4_ERR_SHAPE, "N=%lld < 0", (long long)N);
  if (K > nvfp4::kGemvMaxK) return fail(NVFP4_ERR_SHAPE, "K=%lld exceeds the GEMV limit %lld", (long long)K, (long long)nvfp4::kGemvMaxK);
  if (N > (int64_t)0x3FFFFFFF) return fail(NVFP4_ERR_SHAPE, "N=%lld too large", (long long)N);
  if (N == 0) return NVFP4_OK;
  if (!x || !q || !s || !y) return fail(NVFP4_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(q) || !aligned16(s))
    return fail(NVFP4_ERR_ALIGNMENT, "x, q, s must be 16-byte aligned");
  if (!aligned2(y)) return fail(NVFP4_ERR_ALIGNMENT, "y must be 2-byte aligned");
  const size_t yb = (size_t)N * 2;
  if (overlaps(y, yb, x, (size_t)K * 2) || overlaps(y, yb, q, (size_t)(N * K / 2)) ||
      overlaps(y, yb, s, (size_t)(N * K / 32)))
    return fail(NVFP4_ERR_INVALID_ARG, "y must not overlap x, q or s");
  int sms = 0;
  nvfp4_status st = check_device(&sms);
  if (st != NVFP4_OK) return st;
  const bool static_w = (flags & NVFP4_FLAG_STATIC_WEIGHTS) != 0;
  if (splits > 1 && !nvfp4::gemv_split_fits(N, K, sms, true, splits))
    return fail(NVFP4_ERR_SHAPE, "a K split of %d does not fit N=%lld K=%lld (it needs K %% 512 == 0, at least %d "
                "512-element columns, and at most 11520 elements of x per CTA)", splits, (long long)N, (long long)K,
                splits);
  cudaError_t e = nvfp4::launch_gemv_mx(x, q, s, y, N, K, sms, static_w, (cudaStream_t)stream, splits);
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "mxfp4 gemv launch");
}

size_t nvfp4_gemm_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M < 2 || N < 1) return 0;
  if (M <= 64 && nvfp4::gemm_small_supported(M, N, K)) return nvfp4::gemm_small_workspace_bytes(M, K);
  if (!nvfp4::gemm_tc_supported(M, N, K)) return 0;
  return nvfp4::gemm_tc_workspace_bytes(M, K);
}

nvfp4_status nvfp4_gemm(const uint16_t* X, int64_t ldx, const uint8_t* q, const uint8_t* s,
                        const float* g, uint16_t* Y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                        void* workspace, size_t workspace_bytes, nvfp4_stream_t stream) {
  return nvfp4_gemm_ex(X, ldx, q, s, g, Y, ldy, M, N, K, workspace, workspace_bytes, 0u, stream);
}

nvfp4_status nvfp4_gemm_ex(const uint16_t* X, int64_t ldx, const uint8_t* q, const uint8_t* s,
                           const float* g, uint16_t* Y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                           void* workspace, size_t workspace_bytes, uint32_t flags, nvfp4_stream_t stream) {
  if (flags & ~kKnownFlags) return fail(NVFP4_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  nvfp4_status st = check_k(K);
  if (st != NVFP4_OK) return st;
  if (M < 0 || N < 0) return fail(NVFP4_ERR_SHAPE, "negative size M=%lld N=%lld", (long long)M, (long long)N);
  if (M == 0 || N == 0) return NVFP4_OK;
  if (!X || !q || !s || !g || !Y) return fail(NVFP4_ERR_INVALID_ARG, "null pointer");
  if (ldx < K || ldy < N) return fail(NVFP4_ERR_INVALID_ARG, "ldx=%lld < K or ldy=%lld < N", (long long)ldx, (long long)ldy);
  if (!aligned16(X) || !aligned16(q) || !aligned16(s) || ldx % 8)
    return fail(NVFP4_ERR_ALIGNMENT, "X, q, s must be 16-byte aligned and ldx a multiple of 8");
  if (!aligned2(Y)) return fail(NVFP4_ERR_ALIGNMENT, "Y must be 2-byte aligned");
  if (!aligned4(g)) return fail(NVFP4_ERR_ALIGNMENT, "g must be 4-byte aligned");
  {
    const size_t xb = (size_t)((M - 1) * ldx + K) * 2, yb = (size_t)((M - 1) * ldy + N) * 2;
    if (overlaps(Y, yb, X, xb) || overlaps(Y, yb, q, (size_t)(N * K / 2)) || overlaps(Y, yb, s, (size_t)(N * K / 16)) ||
        overlaps(Y, yb, g, 4))
      return fail(NVFP4_ERR_INVALID_ARG, "Y must not overlap X, q, s or g");
  }
  if (M == 1) return nvfp4_gemv_ex(X, q, s, g, Y, N, K, flags, stream);
  int sms = 0;
  st = check_device(&sms);
  if (st != NVFP4_OK) return st;
  cudaError_t e;
  const bool static_w = (flags & NVFP4_FLAG_STATIC_WEIGHTS) != 0;
  auto check_workspace = [&](size_t need) -> nvfp4_status {
    if (need == 0) return NVFP4_OK;
    if (!workspace || workspace_bytes < need)
      return fail(NVFP4_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace_bytes);
    if (!aligned16(workspace)) return fail(NVFP4_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
    const size_t xb = (size_t)((M - 1) * ldx + K) * 2, yb = (size_t)((M - 1) * ldy + N) * 2;
    if (overlaps(workspace, need, X, xb) || overlaps(workspace, need, Y, yb) ||
        overlaps(workspace, need, q, (size_t)(N * K / 2)) || overlaps(workspace, need, s, (size_t)(N * K / 16)) ||
        overlaps(workspace, need, g, 4))
      return fail(NVFP4_ERR_INVALID_ARG, "workspace must not overlap X, Y, q, s or g");
    return NVFP4_OK;
  };
  if (M <= 64 && nvfp4::gemm_small_supported(M, N, K)) {
    const size_t need = nvfp4::gemm_small_workspace_bytes(M, K);
    st = check_workspace(need);
    if (st != NVFP4_OK) return st;
    e = nvfp4::launch_gemm_small(X, ldx, q, s, g, Y, ldy, M, N, K, need ? workspace : nullptr, static_w,
                                 (cudaStream_t)stream);
    return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "tensor-core gemm launch");
  }
  if (nvfp4::gemm_tc_supported(M, N, K)) {
    st = check_workspace(nvfp4::gemm_tc_workspace_bytes(M, K));
    if (st != NVFP4_OK) return st;
    e = nvfp4::launch_gemm_tc(X, ldx, q, s, g, Y, ldy, M, N, K, workspace, static_w, (cudaStream_t)stream);
    return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "tensor-core gemm launch");
  }
  // K not a multiple of 256: one decode GEMV per row of X (same arithmetic).
  if (K > nvfp4::kGemvMaxK) return fail(NVFP4_ERR_SHAPE, "K=%lld: the GEMM needs K %% 256 == 0 or K <= %lld",
                                        (long long)K, (long long)nvfp4::kGemvMaxK);
  for (int64_t m = 0; m < M; ++m) {
    e = nvfp4::launch_gemv(X + m * ldx, q, s, g, Y + m * ldy, N, K, sms, false, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "gemv launch");
  }
  return NVFP4_OK;
}

// ------------------------------------------------------------------- W4A4

namespace {

size_t round_up(size_t v, size_t m) { return (v + m - 1) / m * m; }

nvfp4_status check_w4a4_shape(int64_t M, int64_t N, int64_t K) {
  if (K <= 0 || K % 256 != 0 || K > ((int64_t)1 << 24))
    return fail(NVFP4_ERR_SHAPE, "K=%lld must be a positive multiple of 256, at most 2^24", (long long)K);
  if (M < 0 || N < 0) return fail(NVFP4_ERR_SHAPE, "negative size M=%lld N=%lld", (long long)M, (long long)N);
  if (M > ((int64_t)1 << 24) || N > ((int64_t)1 << 31) - 128)
    return fail(NVFP4_ERR_SHAPE, "M=%lld or N=%lld too large", (long long)M, (long long)N);
  // the GEMM numbers its 128 x 256 output tiles with 32-bit integers
  if ((N + 127) / 128 * ((M + 255) / 256) > (int64_t)INT32_MAX)
    return fail(NVFP4_ERR_SHAPE, "M=%lld x N=%lld has too many 128 x 256 tiles", (long long)M, (long long)N);
  return NVFP4_OK;
}

}  // namespace

size_t nvfp4_w4a4_weight_scales_bytes(int64_t N, int64_t K) {
  if (N <= 0 || K <= 0 || K % 256) return 0;
  return round_up((size_t)N, 128) * (size_t)(K / 16);
}

size_t nvfp4_w4a4_x_scales_bytes(int64_t M, int64_t K) {
  if (M <= 0 || K <= 0 || K % 256) return 0;
  return round_up((size_t)M, 256) * (size_t)(K / 16);
}

size_t nvfp4_w4a4_workspace_size(int64_t M, int64_t K) {
  if (M <= 0 || K <= 0 || K % 256) return 0;
  return round_up((size_t)(M * K / 2), 16) + nvfp4_w4a4_x_scales_bytes(M, K) + NVFP4_W4A4_AMAX_FLOATS * 4;
}

nvfp4_status nvfp4_w4a4_prepare_weights(const uint8_t* s, int64_t N, int64_t K, uint8_t* s_mma,
                                        nvfp4_stream_t stream) {
  nvfp4_status st = check_w4a4_shape(1, N, K);
  if (st != NVFP4_OK) return st;
  if (N == 0) return NVFP4_OK;
  if (!s || !s_mma) return fail(NVFP4_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(s) || !aligned16(s_mma)) return fail(NVFP4_ERR_ALIGNMENT, "s and s_mma must be 16-byte aligned");
  if (overlaps(s, (size_t)(N * K / 16), s_mma, nvfp4_w4a4_weight_scales_bytes(N, K)))
    return fail(NVFP4_ERR_INVALID_ARG, "s_mma must not overlap s");
  int sms = 0;
  st = check_device(&sms);
  if (st != NVFP4_OK) return st;
  cudaError_t e = nvfp4::launch_scales_to_mma(s, N, K, s_mma, (cudaStream_t)stream, sms);
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "scale rearrangement launch");
}

nvfp4_status nvfp4_w4a4_quantize_x(const uint16_t* X, int64_t ldx, int64_t M, int64_t K, uint8_t* qx, uint8_t* sx,
                                   float* x_amax, uint32_t flags, nvfp4_stream_t stream) {
  if (flags & ~NVFP4_W4A4_GIVEN_AMAX) return fail(NVFP4_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  nvfp4_status st = check_w4a4_shape(M, 1, K);
  if (st != NVFP4_OK) return st;
  if (M == 0) return NVFP4_OK;
  if (!X || !qx || !sx || !x_amax) return fail(NVFP4_ERR_INVALID_ARG, "null pointer");
  if (ldx < K) return fail(NVFP4_ERR_INVALID_ARG, "ldx=%lld < K=%lld", (long long)ldx, (long long)K);
  if (!aligned16(X) || !aligned16(qx) || !aligned16(sx) || ldx % 8 || !aligned4(x_amax))
    return fail(NVFP4_ERR_ALIGNMENT, "X, qx, sx must be 16-byte aligned, ldx a multiple of 8, x_amax 4-byte aligned");
  const bool given = (flags & NVFP4_W4A4_GIVEN_AMAX) != 0;
  const size_t xb = (size_t)((M - 1) * ldx + K) * 2, qb = (size_t)(M * K / 2), sb = nvfp4_w4a4_x_scales_bytes(M, K);
  const size_t ab = given ? 4 : NVFP4_W4A4_AMAX_FLOATS * 4;
  if (overlaps(X, xb, qx, qb) || overlaps(X, xb, sx, sb) || overlaps(qx, qb, sx, sb) || overlaps(x_amax, ab, X, xb) ||
      overlaps(x_amax, ab, qx, qb) || overlaps(x_amax, ab, sx, sb))
    return fail(NVFP4_ERR_INVALID_ARG, "X, qx, sx and x_amax must not overlap");
  int sms = 0;
  st = check_device(&sms);
  if (st != NVFP4_OK) return st;
  cudaError_t e = nvfp4::launch_quantize_x_mma(X, ldx, M, K, x_amax, given, qx, sx, (cudaStream_t)stream, sms);
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "activation quantize launch");
}

nvfp4_status nvfp4_w4a4_gemm(const uint8_t* qx, const uint8_t* sx, const float* x_amax, const uint8_t* q,
                             const uint8_t* s_mma, const float* g, uint16_t* Y, int64_t ldy, int64_t M, int64_t N,
                             int64_t K, uint32_t flags, nvfp4_stream_t stream) {
  if (flags & ~kW4a4Flags) return fail(NVFP4_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  nvfp4_status st = check_w4a4_shape(M, N, K);
  if (st != NVFP4_OK) return st;
  if (M == 0 || N == 0) return NVFP4_OK;
  if (!qx || !sx || !x_amax || !q || !s_mma || !g || !Y) return fail(NVFP4_ERR_INVALID_ARG, "null pointer");
  if (ldy < N) return fail(NVFP4_ERR_INVALID_ARG, "ldy=%lld < N=%lld", (long long)ldy, (long long)N);
  if (!aligned16(qx) || !aligned16(sx) || !aligned16(q) || !aligned16(s_mma))
    return fail(NVFP4_ERR_ALIGNMENT, "qx, sx, q and s_mma must be 16-byte aligned");
  if (!aligned4(x_amax) || !aligned4(g) || !aligned2(Y))
    return fail(NVFP4_ERR_ALIGNMENT, "x_amax and g must be 4-byte aligned, Y 2-byte aligned");
  const size_t yb = (size_t)((M - 1) * ldy + N) * 2;
  if (overlaps(Y, yb, qx, (size_t)(M * K / 2)) || overlaps(Y, yb, sx, nvfp4_w4a4_x_scales_bytes(M, K)) ||
      overlaps(Y, yb, q, (size_t)(N * K / 2)) || overlaps(Y, yb, s_mma, nvfp4_w4a4_weight_scales_bytes(N, K)) ||
      overlaps(Y, yb, g, 4) || overlaps(Y, yb, x_amax, 4))
    return fail(NVFP4_ERR_INVALID_ARG, "Y must not overlap an input");
  int sms = 0;
  st = check_device(&sms);
  if (st != NVFP4_OK) return st;
  cudaError_t e = nvfp4::launch_gemm_w4a4(qx, sx, x_amax, q, s_mma, g, Y, ldy, M, N, K,
                                          (flags & NVFP4_FLAG_STATIC_WEIGHTS) != 0, (flags & NVFP4_FLAG_W4A4_PAIR) != 0,
                                          (cudaStream_t)stream, sms);
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "W4A4 GEMM launch");
}

nvfp4_status nvfp4_w4a4_linear(const uint16_t* X, int64_t ldx, const float* x_amax, const uint8_t* q,
                               const uint8_t* s_mma, const float* g, uint16_t* Y, int64_t ldy, int64_t M, int64_t N,
                               int64_t K, void* workspace, size_t workspace_bytes, uint32_t flags,
                               nvfp4_stream_t stream) {
  if (flags & ~kW4a4Flags) return fail(NVFP4_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  nvfp4_status st = check_w4a4_shape(M, N, K);
  if (st != NVFP4_OK) return st;
  if (M == 0 || N == 0) return NVFP4_OK;
  const size_t need = nvfp4_w4a4_workspace_size(M, K);
  if (!workspace || workspace_bytes < need)
    return fail(NVFP4_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace_bytes);
  if (!aligned16(workspace)) return fail(NVFP4_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
  if (X && ldx >= K) {
    const size_t xb = (size_t)((M - 1) * ldx + K) * 2, yb = ldy >= N ? (size_t)((M - 1) * ldy + N) * 2 : 0;
    if (overlaps(workspace, need, X, xb) || overlaps(workspace, need, Y, yb) ||
        overlaps(workspace, need, q, (size_t)(N * K / 2)) ||
        overlaps(workspace, need, s_mma, nvfp4_w4a4_weight_scales_bytes(N, K)) || overlaps(workspace, need, g, 4) ||
        (x_amax && overlaps(workspace, need, x_amax, 4)))
      return fail(NVFP4_ERR_INVALID_ARG, "workspace must not overlap the other buffers");
  }
  uint8_t* qx = static_cast<uint8_t*>(workspace);
  uint8_t* sx = qx + round_up((size_t)(M * K / 2), 16);
  // the dynamic amax (and its per-CTA maxima) goes to the workspace's end; a given one is only read
  float* amax = x_amax ? const_cast<float*>(x_amax) : reinterpret_cast<float*>(sx + nvfp4_w4a4_x_scales_bytes(M, K));
  st = nvfp4_w4a4_quantize_x(X, ldx, M, K, qx, sx, amax, x_amax ? NVFP4_W4A4_GIVEN_AMAX : 0u, stream);
  if (st != NVFP4_OK) return st;
  return nvfp4_w4a4_gemm(qx, sx, amax, q, s_mma, g, Y, ldy, M, N, K, flags, stream);
}

nvfp4_status nvfp4_check_device_errors(void) {
  unsigned int n = 0, k = 0, v = 0, w = 0;
  cudaError_t e = nvfp4::read_and_clear_gemm_timeouts(&n);
  if (e == cudaSuccess) e = nvfp4::read_and_clear_w4a4_timeouts(&w);
  n += w;
  if (e == cudaSuccess) e = nvfp4::read_and_clear_small_timeouts(&k);
  if (e == cudaSuccess) e = nvfp4::read_and_clear_gemv_timeouts(&v);
  unsigned int bad = 0, window = 0;
  if (e == cudaSuccess) e = nvfp4::read_and_clear_gemv_bad_ids(&bad);
  if (e == cudaSuccess) e = nvfp4::read_and_clear_mx_out_of_window(&window);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error counter");
  if (n || k || v)
    return fail(NVFP4_ERR_TIMEOUT, "%u GEMM, %u small-M GEMM and %u GEMV CTA(s) gave up on a pipeline wait", n, k, v);
  if (bad) return fail(NVFP4_ERR_INVALID_ARG, "%u grouped GEMV problem(s) had an out-of-range expert or token id", bad);
  if (window)
    return fail(NVFP4_ERR_INVALID_ARG, "%u MXFP4 block(s) could not be restated as NVFP4 scales (more than 17 binades "
                "below the largest, or NaN)", window);
  return NVFP4_OK;
}

}  // extern "C"

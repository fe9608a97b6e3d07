// gptq2d_quantize_noalloc: the rounding entry point for callers that cannot
// allocate device memory.
//
// Some callers of this library may not call cudaMalloc at all: code that runs
// inside a host framework whose memory pool owns every device byte (a raw
// allocation would bypass its accounting and budget), services that plan all
// device memory up front and forbid allocation once they are serving, and
// latency-sensitive callers for whom cudaMalloc's implicit device-wide
// synchronization is unacceptable.  gptq2d_quantize asks such a caller for a
// workspace it cannot obtain; this variant needs none.
//
// Its scratch is one file-scope device array of GPTQ2D_NOALLOC_SCRATCH_BYTES.
// Every GPU that loads the library holds that array until the process exits.
// All calls share it: two calls whose kernels overlap on the GPU (for example
// on two streams, or from two threads) race on it and give wrong results, so
// callers must order them.  The array keeps whatever the previous call left;
// the rounding clears the parts that must start at zero (the two feedback
// buffers) at the start of every call and fully writes everything else before
// reading it.
//
// In host code the array's name is only a host-side stand-in, not a device
// address, so the first call on each device resolves the real address with
// cudaGetSymbolAddress while that device is current, and caches it.  That
// first call may load the library's device code and should therefore come
// before any stream capture.  A cudaDeviceReset makes the cached address stale
// (as it does the library's internal streams): the library must not be called
// on a device after it was reset.  No call allocates: no cudaMalloc, cudaFree or
// allocating library routine is used on this path.
#include <mutex>

#include "common.cuh"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[GPTQ2D_NOALLOC_SCRATCH_BYTES];

using gptq2d::kMaxDevices;
constexpr int64_t kMaxDim = (int64_t)1 << 20;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (resolved once per device).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GPTQ2D_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GPTQ2D_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return GPTQ2D_OK;
}

}  // namespace

extern "C" int gptq2d_quantize_noalloc(const void* W, int w_dtype, int64_t m, int64_t n,
                                       int64_t ldw, const double* M_L, int64_t ldl,
                                       const double* M_R, int64_t ldr, const float* scales,
                                       int bits, int clamp, int8_t* Q, int64_t ldq,
                                       gptq2d_stats* stats, void* stream) {
  if (m < 0 || n < 0 || m > kMaxDim || n > kMaxDim) return GPTQ2D_ERR_INVALID_ARG;
  if (w_dtype != GPTQ2D_F32 && w_dtype != GPTQ2D_BF16 && w_dtype != GPTQ2D_F64)
    return GPTQ2D_ERR_INVALID_ARG;
  if (bits < 2 || bits > 8 || (clamp != 0 && clamp != 1)) return GPTQ2D_ERR_INVALID_ARG;
  if (!stats) return GPTQ2D_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (m == 0 || n == 0)
    return gptq2d::quantize_launch(W, w_dtype, (int)m, (int)n, ldw, M_L, ldl, M_R, ldr, scales,
                                   bits, clamp, Q, ldq, stats, nullptr, s);
  if (!W || !M_L || !M_R || !scales || !Q) return GPTQ2D_ERR_INVALID_ARG;
  if (ldw < n || ldl < m || ldr < n || ldq < n) return GPTQ2D_ERR_INVALID_ARG;
  // the problem's scratch need must fit the static array
  if (gptq2d::quantize_ws_bytes(m, n) > (size_t)GPTQ2D_NOALLOC_SCRATCH_BYTES)
    return GPTQ2D_ERR_WORKSPACE;
  if (gptq2d::check_device_pointers({W, M_L, M_R, scales, Q, stats}) != GPTQ2D_OK)
    return GPTQ2D_ERR_INVALID_ARG;
  void* ws = nullptr;
  const int rc = scratch_address(&ws);
  if (rc != GPTQ2D_OK) return rc;
  return gptq2d::quantize_launch(W, w_dtype, (int)m, (int)n, ldw, M_L, ldl, M_R, ldr, scales,
                                 bits, clamp, Q, ldq, stats, ws, s);
}

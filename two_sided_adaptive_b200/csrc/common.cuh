// Internal helpers shared by the GPTQ-2D kernels (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <atomic>
#include <initializer_list>
#include <mutex>

#include "gptq2d.h"

namespace gptq2d {

// Edge of the square tiles the rounding sweep and the factor preparation work on.
constexpr int TB = 64;

// Counts every kernel launch the library issues (gptq2d_launch_count).
extern std::atomic<int64_t> g_launches;
inline void count_launch(int n = 1) { g_launches.fetch_add(n, std::memory_order_relaxed); }

// Kernel classes of the optional per-launch event profiler (gptq2d_profile_*).
enum KernelClass {
  KC_PREP_PANEL = 0,     // factor preparation: diagonal block + block-row solve
  KC_PREP_TRAILING = 1,  // factor preparation: rank-64 trailing update
  KC_SWEEP = 2,          // anti-diagonal tile sweep
  KC_PROPAGATE = 3,      // band products to tiles two or more tiles away
  KC_OTHER = 4,          // conversions, diagonals, statistics
  KC_COUNT = 5
};
// When profiling is on, records a CUDA event pair around the launch on `s`.
struct ProfScope {
  int cls;
  cudaStream_t s;
  cudaEvent_t e0 = nullptr;
  ProfScope(int c, cudaStream_t st);
  ~ProfScope();
};
#define GPTQ2D_LAUNCH(cls, stream, ...)             \
  do {                                              \
    ::gptq2d::ProfScope _ps((cls), (stream));       \
    __VA_ARGS__;                                    \
    ::gptq2d::count_launch();                       \
  } while (0)

// Most devices the library keeps per-device state for (internal streams, the
// no-allocation scratch address).
constexpr int kMaxDevices = 64;

// GPTQ2D_OK when every non-null pointer is memory the current device may
// dereference: device memory of the current device, managed memory, or
// page-locked host memory; GPTQ2D_ERR_INVALID_ARG for another device's memory or
// pageable host memory (a kernel given either would fault or read the wrong GPU).
int check_device_pointers(std::initializer_list<const void*> ps);

inline int64_t round_up(int64_t x, int64_t r) { return (x + r - 1) / r * r; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Sets the dynamic shared-memory limit of `fn` once per device.
template <typename F>
inline cudaError_t ensure_smem(F* fn, int bytes, std::atomic<uint64_t>& done_mask) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = (dev < 64) ? (uint64_t(1) << dev) : 0;
  if (bit && (done_mask.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(reinterpret_cast<const void*>(fn),
                           cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done_mask.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// ---------------------------------------------------------------------------
// Element loads with conversion to fp64
// ---------------------------------------------------------------------------
__device__ __forceinline__ double to_f64(float v) { return static_cast<double>(v); }
__device__ __forceinline__ double to_f64(double v) { return v; }
__device__ __forceinline__ double to_f64(__nv_bfloat16 v) {
  return static_cast<double>(__bfloat162float(v));
}

// ---------------------------------------------------------------------------
// FP64 tensor-core MMA (DMMA), m8n8k4, row.col.
// Fragments (lane = 4*g + t, g = lane>>2, t = lane&3):
//   A 8x4 : a = A[g][t]        B 4x8 : b = B[t][g]
//   C 8x8 : c0 = C[g][2t], c1 = C[g][2t+1]
// ---------------------------------------------------------------------------
__device__ __forceinline__ void dmma_m8n8k4(double& c0, double& c1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};\n"
               : "+d"(c0), "+d"(c1)
               : "d"(a), "d"(b));
}

// 64x64x64 product of two shared-memory tiles on 4 warps (128 threads).  Warp w
// owns the 32x32 quadrant (w>>1, w&1) as 4x4 fragments of 8x8.  `fa(row, k)`
// and `fb(k, col)` return the operand elements from shared memory.
template <typename FA, typename FB>
__device__ __forceinline__ void mma_64x64x64_w(double (&acc)[4][4][2], int warp, FA fa, FB fb,
                                               int kmax = TB) {
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int wr = (warp >> 1) * 32, wc = (warp & 1) * 32;
#pragma unroll 4
  for (int kk = 0; kk < kmax; kk += 4) {
    double a[4], b[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = fa(wr + i * 8 + g, kk + t);
#pragma unroll
    for (int j = 0; j < 4; ++j) b[j] = fb(kk + t, wc + j * 8 + g);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) dmma_m8n8k4(acc[i][j][0], acc[i][j][1], a[i], b[j]);
  }
}

template <typename FA, typename FB>
__device__ __forceinline__ void mma_64x64x64(double (&acc)[4][4][2], FA fa, FB fb, int kmax = TB) {
  mma_64x64x64_w(acc, (int)(threadIdx.x >> 5), fa, fb, kmax);
}

// ---------------------------------------------------------------------------
// cp.async helpers (Ampere-style asynchronous copies, available on sm_100a)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cp_async16_zfill(void* smem, const void* gmem, bool valid) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  const int n = valid ? 16 : 0;  // src-size 0: nothing is read, 16 zero bytes are written
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(n));
}
__device__ __forceinline__ void cp_async8_zfill(void* smem, const void* gmem, bool valid) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  const int n = valid ? 8 : 0;
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;\n" ::"r"(s), "l"(gmem), "r"(n));
}
__device__ __forceinline__ void cp_async_commit_group() {
  asm volatile("cp.async.commit_group;\n" ::);
}
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

// Per-tile partial statistics of one rounding sweep.
struct TileStat {
  double loss;
  long long clamped, near_tie, nonfinite, out_of_range;
};

// ---------------------------------------------------------------------------
// Per-device internal streams (streams.cu): two highest-priority and two
// lowest-priority non-blocking streams plus events to fork from / join to the
// caller's stream.  `mu` serialises the enqueue sequences that use them.
// ---------------------------------------------------------------------------
constexpr int RING = 4;
struct DevStreams {
  std::recursive_mutex mu;  // held across nested enqueues (round_host -> prepare, quantize)
  bool ready = false;
  int sms = 148;
  cudaStream_t hi = nullptr, lo = nullptr, hi2 = nullptr, lo2 = nullptr;
  cudaStream_t hi3 = nullptr, lo3 = nullptr;  // a second factor pair, beside a rounding
  cudaStream_t cp = nullptr;  // host<->device copies of round_host
  cudaStream_t blk_p = nullptr, blk_q = nullptr;  // block scheduler: factor and rounding lanes
  cudaEvent_t fork = nullptr, setup = nullptr, join_hi = nullptr, join_lo = nullptr;
  cudaEvent_t join_hi2 = nullptr, join_lo2 = nullptr, join_hi3 = nullptr, join_lo3 = nullptr;
  cudaEvent_t blk_start = nullptr, blk_prep[2] = {}, blk_quant[2] = {}, blk_end[2] = {};
  cudaEvent_t cp_ev[3] = {};  // H_L, H_R, W + scales copied
  cudaEvent_t q_ev[4] = {};   // rows of Q final (round_host copies them out early)
  cudaEvent_t sw[RING] = {}, far[RING] = {}, farb[RING] = {};
  cudaEvent_t panel_done[2][RING] = {}, rest_done[2][RING] = {};  // factor preparation
};
int dev_streams(DevStreams** out);

// ---------------------------------------------------------------------------
// Host-side launchers (defined in prepare.cu / quantize.cu / kron.cu)
// ---------------------------------------------------------------------------
size_t prepare_ws_bytes(int64_t k);
int prepare_launch(const void* H, int h_dtype, int k, int64_t ldh, double* M, int64_t ldm,
                   void* ws, cudaStream_t s);

// Both factors at once, interleaved step by step on the internal streams
// (panels on the high-priority ones, trailing updates on the low-priority
// ones), forked from and joined back to `s`.
// ready_l / ready_r (may be null): events that H_L / H_R wait for beyond `s`.
// alt: run on the second factor pairs (hi2/lo2 and hi3/lo3), leaving hi/lo to a
// rounding that runs beside it.
int prepare_pair_launch(const void* H_L, int64_t m, int64_t ldhl, const void* H_R, int64_t n,
                        int64_t ldhr, int h_dtype, double* M_L, int64_t ldml, double* M_R,
                        int64_t ldmr, void* ws_l, void* ws_r, cudaStream_t s,
                        cudaEvent_t ready_l = nullptr, cudaEvent_t ready_r = nullptr,
                        bool alt = false);

// Gram of activations on the tcgen05 tensor cores (defined in gram.cu): H's lower
// 128-block triangle (+)= X^T X (X bf16, N x k, k and ldx multiples of 8); then
// H <- H / total_rows with diagonal damping.
int gram_accumulate_launch(const void* X, int64_t N, int k, int64_t ldx, float* H, int64_t ldh,
                           int beta, int* err, cudaStream_t s);
int gram_finalize_launch(float* H, int k, int64_t ldh, int64_t total_rows, double damp,
                         double* diag_sum, cudaStream_t s);

// Kronecker product of nf lower factors into out (defined in kron.cu).
int kron_factor_launch(int nf, const double* const* M, const int64_t* dims, const int64_t* ldm,
                       double* out, int64_t ldo, cudaStream_t s);

size_t quantize_ws_bytes(int64_t m, int64_t n);
int check_wait_timeout(long long limit_ns, cudaStream_t s);  // synchronizes s

// Grid of a rounding call beyond bits/clamp (default: one scale per row, symmetric,
// one byte per entry).
struct GridSpec {
  int64_t group = 0;              // columns per scale group (multiple of 8, or >= n); 0: per row
  int64_t lds = 1;                // row stride of scales and zeros, in groups
  const uint8_t* zero = nullptr;  // integer zero points (asymmetric grid), or null
  int packed = 0;                 // two 4-bit codes per byte
};

// The right factor of a k-way rounding given per mode (gptq2d_quantize_kron):
// M_R = M[0] (x) ... (x) M[nf-1], never formed.  The last factors whose sizes
// multiply to m_in (8, 16, 32 or 64, a divisor of the 64-column tile) form the
// inner group; kron_inner finds it.
struct KronSpec {
  int nf = 0;
  const double* const* M = nullptr;  // HOST array of DEVICE pointers
  const int64_t* dims = nullptr;
  const int64_t* ldm = nullptr;
};
// m_in of these modes (the product of the longest suffix of dims dividing 64, when
// it is at least 8), or 0 when the per-mode path does not apply; *nin = its factors.
int kron_inner(int nf, const int64_t* dims, int* nin);
size_t quantize_kron_ws_bytes(int64_t m, int nf, const int64_t* dims);

// Optional row events: row_ev[k] is recorded once the tile rows 0..row_tile[k] of
// Q are final (row_tile ascending), so a caller can copy them out early.  With
// `kron`, MR and ldr are unused and the workspace is quantize_kron_ws_bytes.
int quantize_launch(const void* W, int w_dtype, int m, int n, int64_t ldw, const double* ML,
                    int64_t ldl, const double* MR, int64_t ldr, const float* scales, int bits,
                    int clamp, int8_t* Q, int64_t ldq, gptq2d_stats* stats, void* ws,
                    cudaStream_t s, int n_row_ev = 0, const int* row_tile = nullptr,
                    cudaEvent_t* row_ev = nullptr, const GridSpec* grid = nullptr,
                    const KronSpec* kron = nullptr);

}  // namespace gptq2d

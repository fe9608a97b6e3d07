// extern "C" entry points of libgptq2d (declared and documented in include/gptq2d.h).
// Argument checks run on the host before anything is enqueued.
#include <algorithm>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "common.cuh"

namespace gptq2d {
std::atomic<int64_t> g_launches{0};

namespace {
std::atomic<bool> g_prof_on{false};
std::mutex g_prof_mu;
std::vector<std::pair<cudaEvent_t, cudaEvent_t>> g_prof_ev[KC_COUNT];
struct ProfRec { int cls; cudaEvent_t e0, e1; };
std::vector<ProfRec> g_prof_order;  // every recorded launch, in enqueue order
std::vector<cudaEvent_t> g_prof_pool;

cudaEvent_t prof_event() {
  if (!g_prof_pool.empty()) {
    cudaEvent_t e = g_prof_pool.back();
    g_prof_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}
}  // namespace

ProfScope::ProfScope(int c, cudaStream_t st) : cls(c), s(st) {
  if (!g_prof_on.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  e0 = prof_event();
  if (e0) cudaEventRecord(e0, s);
}

ProfScope::~ProfScope() {
  if (!e0) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  cudaEvent_t e1 = prof_event();
  if (e1 && cudaEventRecord(e1, s) == cudaSuccess)
  {
    g_prof_ev[cls].emplace_back(e0, e1);
    g_prof_order.push_back(ProfRec{cls, e0, e1});
  }
  else
    g_prof_pool.push_back(e0);
}
int check_device_pointers(std::initializer_list<const void*> ps) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GPTQ2D_ERR_CUDA;
  for (const void* p : ps) {
    if (!p) continue;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
      cudaGetLastError();  // not sticky: clear it
      return GPTQ2D_ERR_INVALID_ARG;
    }
    if (at.type == cudaMemoryTypeUnregistered) return GPTQ2D_ERR_INVALID_ARG;
    if (at.type == cudaMemoryTypeDevice && at.device != dev) return GPTQ2D_ERR_INVALID_ARG;
  }
  return GPTQ2D_OK;
}
}  // namespace gptq2d

using namespace gptq2d;

namespace {

// Largest edge handled: keeps every 64-tile count and padded product within int32.
constexpr int64_t kMaxDim = (int64_t)1 << 20;

bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

size_t elem_size(int dt) {
  switch (dt) {
    case GPTQ2D_F32: return 4;
    case GPTQ2D_BF16: return 2;
    case GPTQ2D_F64: return 8;
    default: return 0;
  }
}

struct HostWs {
  size_t off_W, off_HL, off_HR, off_s, off_ML, off_MR, off_Q, off_stats, off_pl, off_pr, off_q,
      total;
};

HostWs host_layout(int64_t m, int64_t n, int w_dtype, int h_dtype) {
  HostWs L;
  size_t o = 0;
  L.off_W = o; o += align256((size_t)m * n * elem_size(w_dtype));
  L.off_HL = o; o += align256((size_t)m * m * elem_size(h_dtype));
  L.off_HR = o; o += align256((size_t)n * n * elem_size(h_dtype));
  L.off_s = o; o += align256((size_t)m * sizeof(float));
  L.off_ML = o; o += align256((size_t)m * m * sizeof(double));
  L.off_MR = o; o += align256((size_t)n * n * sizeof(double));
  L.off_Q = o; o += align256((size_t)m * n);
  L.off_stats = o; o += align256(sizeof(gptq2d_stats));
  L.off_pl = o; o += align256(prepare_ws_bytes(m));
  L.off_pr = o; o += align256(prepare_ws_bytes(n));
  L.off_q = o; o += align256(quantize_ws_bytes(m, n));
  L.total = o;
  return L;
}

// The pivot word of a factorization: -1 fine, >= 0 the first bad pivot.
int pivot_status(long long info) { return info >= 0 ? GPTQ2D_ERR_NOT_SPD : GPTQ2D_OK; }

int read_pivot(const void* ws, cudaStream_t s, int64_t* bad_pivot) {
  long long info = -1;
  if (cudaMemcpyAsync(&info, ws, sizeof(info), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return GPTQ2D_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return GPTQ2D_ERR_CUDA;
  if (bad_pivot) *bad_pivot = info >= 0 ? info : -1;
  return pivot_status(info);
}

}  // namespace

extern "C" {

const char* gptq2d_status_string(int status) {
  switch (status) {
    case GPTQ2D_OK: return "GPTQ2D_OK";
    case GPTQ2D_ERR_INVALID_ARG: return "GPTQ2D_ERR_INVALID_ARG: invalid argument";
    case GPTQ2D_ERR_NOT_SPD: return "GPTQ2D_ERR_NOT_SPD: factor is not positive definite";
    case GPTQ2D_ERR_NONFINITE: return "GPTQ2D_ERR_NONFINITE: non-finite input or invalid scale";
    case GPTQ2D_ERR_WORKSPACE: return "GPTQ2D_ERR_WORKSPACE: workspace too small or misaligned";
    case GPTQ2D_ERR_TIMEOUT: return "GPTQ2D_ERR_TIMEOUT: bounded device wait gave up";
    case GPTQ2D_ERR_CUDA: return "GPTQ2D_ERR_CUDA: CUDA runtime error";
    case GPTQ2D_ERR_RANGE: return "GPTQ2D_ERR_RANGE: an unclamped integer does not fit its byte";
    default: return "GPTQ2D: unknown status";
  }
}

int gptq2d_version(void) { return (1 << 16) | 0; }

int64_t gptq2d_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int gptq2d_check_wait_timeout(int64_t limit_ns, void* stream) {
  if (limit_ns < 1000 || limit_ns > 10000000000ll) return GPTQ2D_ERR_INVALID_ARG;
  return check_wait_timeout(limit_ns, static_cast<cudaStream_t>(stream));
}

void gptq2d_profile_enable(int on) { g_prof_on.store(on != 0); }

int gptq2d_profile_read(int kernel_class, int64_t* launches, double* total_ms) {
  if (kernel_class < 0 || kernel_class >= KC_COUNT || !launches || !total_ms)
    return GPTQ2D_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  double ms = 0.0;
  for (auto& pr : g_prof_ev[kernel_class]) {
    if (cudaEventSynchronize(pr.second) != cudaSuccess) return GPTQ2D_ERR_CUDA;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, pr.first, pr.second) != cudaSuccess) return GPTQ2D_ERR_CUDA;
    ms += t;
  }
  *launches = (int64_t)g_prof_ev[kernel_class].size();
  *total_ms = ms;
  return GPTQ2D_OK;
}

int gptq2d_profile_timeline(int64_t max_entries, int32_t* cls, double* start_ms, double* end_ms,
                            int64_t* n_out) {
  if (!n_out || (max_entries > 0 && (!cls || !start_ms || !end_ms))) return GPTQ2D_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  *n_out = (int64_t)g_prof_order.size();
  if (g_prof_order.empty()) return GPTQ2D_OK;
  const cudaEvent_t base = g_prof_order.front().e0;
  for (auto& r : g_prof_order)
    if (cudaEventSynchronize(r.e1) != cudaSuccess) return GPTQ2D_ERR_CUDA;
  const int64_t n = std::min<int64_t>(max_entries, (int64_t)g_prof_order.size());
  for (int64_t i = 0; i < n; ++i) {
    float a = 0.f, b = 0.f;
    if (cudaEventElapsedTime(&a, base, g_prof_order[i].e0) != cudaSuccess ||
        cudaEventElapsedTime(&b, base, g_prof_order[i].e1) != cudaSuccess)
      return GPTQ2D_ERR_CUDA;
    cls[i] = g_prof_order[i].cls;
    start_ms[i] = a;
    end_ms[i] = b;
  }
  return GPTQ2D_OK;
}

void gptq2d_profile_reset(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_order.clear();
  for (auto& v : g_prof_ev) {
    for (auto& pr : v) {
      g_prof_pool.push_back(pr.first);
      g_prof_pool.push_back(pr.second);
    }
    v.clear();
  }
}

size_t gptq2d_prepare_workspace_size(int64_t k) {
  if (k < 0 || k > kMaxDim) return 0;
  return prepare_ws_bytes(k);
}

int gptq2d_prepare(const void* H, int h_dtype, int64_t k, int64_t ldh, double* M, int64_t ldm,
                   void* ws, size_t ws_bytes, void* stream, int64_t* bad_pivot) {
  if (k < 0 || k > kMaxDim) return GPTQ2D_ERR_INVALID_ARG;
  if (h_dtype != GPTQ2D_F32 && h_dtype != GPTQ2D_F64) return GPTQ2D_ERR_INVALID_ARG;
  if (k == 0) {
    if (bad_pivot) *bad_pivot = -1;
    return GPTQ2D_OK;
  }
  if (!H || !M || ldh < k || ldm < k) return GPTQ2D_ERR_INVALID_ARG;
  if (static_cast<const void*>(M) == H) return GPTQ2D_ERR_INVALID_ARG;
  if (!ws || !aligned256(ws) || ws_bytes < prepare_ws_bytes(k)) return GPTQ2D_ERR_WORKSPACE;
  int rc = check_device_pointers({H, M, ws});
  if (rc != GPTQ2D_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  rc = prepare_launch(H, h_dtype, (int)k, ldh, M, ldm, ws, s);
  if (rc != GPTQ2D_OK) return rc;
  if (bad_pivot) return read_pivot(ws, s, bad_pivot);
  return GPTQ2D_OK;
}

size_t gptq2d_gram_workspace_size(void) { return 256; }

int gptq2d_gram_accumulate(const void* X, int x_dtype, int64_t rows, int64_t k, int64_t ldx,
                           float* H, int64_t ldh, int accumulate, void* ws, size_t ws_bytes,
                           void* stream) {
  // rows: the TMA row coordinate is a 32-bit integer
  if (x_dtype != GPTQ2D_BF16 || rows < 0 || rows > INT32_MAX || k < 0 || k > kMaxDim)
    return GPTQ2D_ERR_INVALID_ARG;
  if (accumulate != 0 && accumulate != 1) return GPTQ2D_ERR_INVALID_ARG;
  if (k == 0) return GPTQ2D_OK;
  if (!H || ldh < k || k % 8 != 0) return GPTQ2D_ERR_INVALID_ARG;
  if (rows > 0 && (!X || ldx < k || ldx % 8 != 0 ||
                   (reinterpret_cast<uintptr_t>(X) & 15u) != 0))
    return GPTQ2D_ERR_INVALID_ARG;
  if (!ws || !aligned256(ws) || ws_bytes < 256) return GPTQ2D_ERR_WORKSPACE;
  const int rc = check_device_pointers({rows > 0 ? X : nullptr, H, ws});
  if (rc != GPTQ2D_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* err = reinterpret_cast<int*>(static_cast<char*>(ws) + 8);
  if (!accumulate && cudaMemsetAsync(err, 0, sizeof(int), s) != cudaSuccess) return GPTQ2D_ERR_CUDA;
  return gram_accumulate_launch(X, rows, (int)k, ldx, H, ldh, accumulate, err, s);
}

int gptq2d_gram_finalize(float* H, int64_t k, int64_t ldh, int64_t total_rows, double damp,
                         void* ws, size_t ws_bytes, void* stream, int* status) {
  if (k < 0 || k > kMaxDim || total_rows < 1 || !(damp >= 0.0)) return GPTQ2D_ERR_INVALID_ARG;
  if (!ws || !aligned256(ws) || ws_bytes < 256) return GPTQ2D_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (k > 0) {
    if (!H || ldh < k) return GPTQ2D_ERR_INVALID_ARG;
    if (check_device_pointers({H, ws}) != GPTQ2D_OK) return GPTQ2D_ERR_INVALID_ARG;
    const int rc = gram_finalize_launch(H, (int)k, ldh, total_rows, damp,
                                        reinterpret_cast<double*>(ws), s);
    if (rc != GPTQ2D_OK) return rc;
  }
  if (!status) return GPTQ2D_OK;
  int err = 0;
  if (cudaMemcpyAsync(&err, static_cast<char*>(ws) + 8, sizeof(int), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return GPTQ2D_ERR_CUDA;
  *status = err ? GPTQ2D_ERR_TIMEOUT : GPTQ2D_OK;
  return *status;
}

int gptq2d_kron_factor(int nf, const double* const* M, const int64_t* dims, const int64_t* ldm,
                       double* out, int64_t ldo, void* stream) {
  if (nf < 1 || nf > GPTQ2D_MAX_KRON_FACTORS || !M || !dims || !ldm) return GPTQ2D_ERR_INVALID_ARG;
  int64_t n = 1;
  for (int f = 0; f < nf; ++f) {
    if (dims[f] < 0 || dims[f] > kMaxDim) return GPTQ2D_ERR_INVALID_ARG;
    n *= dims[f];
    if (n > kMaxDim) return GPTQ2D_ERR_INVALID_ARG;
  }
  if (n == 0) return GPTQ2D_OK;
  if (!out || ldo < n) return GPTQ2D_ERR_INVALID_ARG;
  const char* o0 = reinterpret_cast<const char*>(out);
  const char* o1 = o0 + (size_t)((n - 1) * ldo + n) * sizeof(double);
  for (int f = 0; f < nf; ++f) {
    if (!M[f] || ldm[f] < dims[f]) return GPTQ2D_ERR_INVALID_ARG;
    const char* m0 = reinterpret_cast<const char*>(M[f]);
    const char* m1 = m0 + (size_t)((dims[f] - 1) * ldm[f] + dims[f]) * sizeof(double);
    if (m0 < o1 && o0 < m1) return GPTQ2D_ERR_INVALID_ARG;  // overlaps the output
    if (check_device_pointers({M[f]}) != GPTQ2D_OK) return GPTQ2D_ERR_INVALID_ARG;
  }
  if (check_device_pointers({out}) != GPTQ2D_OK) return GPTQ2D_ERR_INVALID_ARG;
  return kron_factor_launch(nf, M, dims, ldm, out, ldo, static_cast<cudaStream_t>(stream));
}

int gptq2d_prepare_pair(const void* H_L, int64_t m, int64_t ldhl, const void* H_R, int64_t n,
                        int64_t ldhr, int h_dtype, double* M_L, int64_t ldml, double* M_R,
                        int64_t ldmr, void* ws, size_t ws_bytes, void* stream,
                        int64_t* bad_pivot, int* which_factor) {
  if (m < 0 || n < 0 || m > kMaxDim || n > kMaxDim) return GPTQ2D_ERR_INVALID_ARG;
  if (h_dtype != GPTQ2D_F32 && h_dtype != GPTQ2D_F64) return GPTQ2D_ERR_INVALID_ARG;
  if (m > 0 && (!H_L || !M_L || ldhl < m || ldml < m || static_cast<const void*>(M_L) == H_L))
    return GPTQ2D_ERR_INVALID_ARG;
  if (n > 0 && (!H_R || !M_R || ldhr < n || ldmr < n || static_cast<const void*>(M_R) == H_R))
    return GPTQ2D_ERR_INVALID_ARG;
  if (!ws || !aligned256(ws) || ws_bytes < 512) return GPTQ2D_ERR_WORKSPACE;
  if (check_device_pointers({m > 0 ? H_L : nullptr, m > 0 ? M_L : nullptr,
                             n > 0 ? H_R : nullptr, n > 0 ? M_R : nullptr, ws}) != GPTQ2D_OK)
    return GPTQ2D_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* b = static_cast<char*>(ws);
  const int rc = prepare_pair_launch(H_L, m, ldhl, H_R, n, ldhr, h_dtype, M_L, ldml, M_R, ldmr,
                                     b, b + 256, s);
  if (rc != GPTQ2D_OK) return rc;
  if (!bad_pivot && !which_factor) return GPTQ2D_OK;
  long long piv[2] = {-1, -1};
  if (m > 0 && cudaMemcpyAsync(&piv[0], b, 8, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return GPTQ2D_ERR_CUDA;
  if (n > 0 && cudaMemcpyAsync(&piv[1], b + 256, 8, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return GPTQ2D_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return GPTQ2D_ERR_CUDA;
  for (int f = 0; f < 2; ++f)
    if (pivot_status(piv[f]) != GPTQ2D_OK) {
      if (bad_pivot) *bad_pivot = piv[f] >= 0 ? piv[f] : -1;
      if (which_factor) *which_factor = f;
      return pivot_status(piv[f]);
    }
  if (bad_pivot) *bad_pivot = -1;
  if (which_factor) *which_factor = -1;
  return GPTQ2D_OK;
}

int gptq2d_prepare_info(const void* ws, void* stream, int64_t* bad_pivot) {
  if (!ws || !bad_pivot) return GPTQ2D_ERR_INVALID_ARG;
  return read_pivot(ws, static_cast<cudaStream_t>(stream), bad_pivot);
}

size_t gptq2d_quantize_workspace_size(int64_t m, int64_t n) {
  if (m < 0 || n < 0 || m > kMaxDim || n > kMaxDim) return 0;
  if (m == 0 || n == 0) return 256;
  return quantize_ws_bytes(m, n);
}

int gptq2d_quantize(const void* W, int w_dtype, int64_t m, int64_t n, int64_t ldw,
                    const double* M_L, int64_t ldl, const double* M_R, int64_t ldr,
                    const float* scales, int bits, int clamp, int8_t* Q, int64_t ldq,
                    gptq2d_stats* stats, void* ws, size_t ws_bytes, void* stream) {
  if (m < 0 || n < 0 || m > kMaxDim || n > kMaxDim) return GPTQ2D_ERR_INVALID_ARG;
  if (elem_size(w_dtype) == 0) return GPTQ2D_ERR_INVALID_ARG;
  if (bits < 2 || bits > 8 || (clamp != 0 && clamp != 1)) return GPTQ2D_ERR_INVALID_ARG;
  if (!stats) return GPTQ2D_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (m == 0 || n == 0)
    return quantize_launch(W, w_dtype, (int)m, (int)n, ldw, M_L, ldl, M_R, ldr, scales, bits,
                           clamp, Q, ldq, stats, ws, s);
  if (!W || !M_L || !M_R || !scales || !Q) return GPTQ2D_ERR_INVALID_ARG;
  if (ldw < n || ldl < m || ldr < n || ldq < n) return GPTQ2D_ERR_INVALID_ARG;
  if (!ws || !aligned256(ws) || ws_bytes < quantize_ws_bytes(m, n)) return GPTQ2D_ERR_WORKSPACE;
  if (check_device_pointers({W, M_L, M_R, scales, Q, stats, ws}) != GPTQ2D_OK)
    return GPTQ2D_ERR_INVALID_ARG;
  return quantize_launch(W, w_dtype, (int)m, (int)n, ldw, M_L, ldl, M_R, ldr, scales, bits, clamp,
                         Q, ldq, stats, ws, s);
}

namespace {
// Host checks of a rounding call on a grid (everything but the factors and the
// workspace); fills `gs`.  m == 0 or n == 0 passes (nothing to round).
int check_grid_call(const void* W, int w_dtype, int64_t m, int64_t n, int64_t ldw,
                    const gptq2d_grid* grid, const void* Q, int64_t ldq, const gptq2d_stats* stats,
                    GridSpec* gs) {
  if (m < 0 || n < 0 || m > kMaxDim || n > kMaxDim) return GPTQ2D_ERR_INVALID_ARG;
  if (elem_size(w_dtype) == 0 || !grid || !stats) return GPTQ2D_ERR_INVALID_ARG;
  const int bits = grid->bits, clamp = grid->clamp;
  if (bits < 2 || bits > 8 || (clamp != 0 && clamp != 1)) return GPTQ2D_ERR_INVALID_ARG;
  if (grid->packed != 0 && grid->packed != 1) return GPTQ2D_ERR_INVALID_ARG;
  if (grid->packed && (bits > 4 || !clamp)) return GPTQ2D_ERR_INVALID_ARG;
  if (grid->zeros && !clamp) return GPTQ2D_ERR_INVALID_ARG;  // codes must fit their byte
  const int64_t G = grid->group_size;
  if (G < 0 || (G > 0 && G % 8 != 0 && G < n)) return GPTQ2D_ERR_INVALID_ARG;
  gs->group = G;
  gs->lds = grid->ld_scales;
  gs->zero = grid->zeros;
  gs->packed = grid->packed;
  if (m == 0 || n == 0) return GPTQ2D_OK;
  const int64_t groups = (G == 0 || G >= n) ? 1 : (n + G - 1) / G;
  if (!W || !grid->scales || !Q) return GPTQ2D_ERR_INVALID_ARG;
  if (grid->ld_scales < groups) return GPTQ2D_ERR_INVALID_ARG;
  if (ldw < n || ldq < (grid->packed ? (n + 1) / 2 : n)) return GPTQ2D_ERR_INVALID_ARG;
  return GPTQ2D_OK;
}
}  // namespace

int gptq2d_quantize_grid(const void* W, int w_dtype, int64_t m, int64_t n, int64_t ldw,
                         const double* M_L, int64_t ldl, const double* M_R, int64_t ldr,
                         const gptq2d_grid* grid, void* Q, int64_t ldq, gptq2d_stats* stats,
                         void* ws, size_t ws_bytes, void* stream) {
  GridSpec gs;
  const int rc = check_grid_call(W, w_dtype, m, n, ldw, grid, Q, ldq, stats, &gs);
  if (rc != GPTQ2D_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (m == 0 || n == 0)
    return quantize_launch(W, w_dtype, (int)m, (int)n, ldw, M_L, ldl, M_R, ldr, grid->scales,
                           grid->bits, grid->clamp, static_cast<int8_t*>(Q), ldq, stats, ws, s, 0,
                           nullptr, nullptr, &gs);
  if (!M_L || !M_R || ldl < m || ldr < n) return GPTQ2D_ERR_INVALID_ARG;
  if (!ws || !aligned256(ws) || ws_bytes < quantize_ws_bytes(m, n)) return GPTQ2D_ERR_WORKSPACE;
  if (check_device_pointers({W, M_L, M_R, grid->scales, grid->zeros, Q, stats, ws}) != GPTQ2D_OK)
    return GPTQ2D_ERR_INVALID_ARG;
  return quantize_launch(W, w_dtype, (int)m, (int)n, ldw, M_L, ldl, M_R, ldr, grid->scales,
                         grid->bits, grid->clamp, static_cast<int8_t*>(Q), ldq, stats, ws, s, 0,
                         nullptr, nullptr, &gs);
}

int gptq2d_per_mode_order(int nf, const int64_t* dims, int* order) {
  if (nf < 1 || nf > GPTQ2D_MAX_KRON_FACTORS || !dims || !order) return -1;
  for (int f = 0; f < nf; ++f)
    if (dims[f] < 1) return -1;
  for (int f = 0; f < nf; ++f) order[f] = f;
  int best_mask = 0;
  int64_t best_p = 0;
  for (int mask = 1; mask < (1 << nf); ++mask) {
    int64_t p = 1;
    for (int f = 0; f < nf && p <= 64; ++f)
      if ((mask >> f) & 1) p *= dims[f];
    if ((p == 8 || p == 16 || p == 32 || p == 64) && p > best_p) {
      best_p = p;
      best_mask = mask;
    }
  }
  if (best_p == 0) return 0;
  int nin = 0;
  if (kron_inner(nf, dims, &nin) == best_p) return (int)best_p;  // the given order reaches it
  int k = 0;
  for (int f = 0; f < nf; ++f)
    if (!((best_mask >> f) & 1)) order[k++] = f;
  for (int f = 0; f < nf; ++f)
    if ((best_mask >> f) & 1) order[k++] = f;
  return (int)best_p;
}

size_t gptq2d_quantize_kron_workspace_size(int64_t m, int nf, const int64_t* dims) {
  if (m < 0 || m > kMaxDim || nf < 1 || nf > GPTQ2D_MAX_KRON_FACTORS || !dims) return 0;
  int64_t n = 1;
  for (int f = 0; f < nf; ++f) {
    if (dims[f] < 1 || dims[f] > kMaxDim) return 0;
    n *= dims[f];
    if (n > kMaxDim) return 0;
  }
  return quantize_kron_ws_bytes(m, nf, dims);
}

int gptq2d_quantize_kron_grid(const void* W, int w_dtype, int64_t m, int64_t ldw,
                              const double* M_L, int64_t ldl, int nf, const double* const* M,
                              const int64_t* dims, const int64_t* ldm, const gptq2d_grid* grid,
                              void* Q, int64_t ldq, gptq2d_stats* stats, void* ws, size_t ws_bytes,
                              void* stream) {
  if (m < 0 || m > kMaxDim || nf < 1 || nf > GPTQ2D_MAX_KRON_FACTORS || !M || !dims || !ldm)
    return GPTQ2D_ERR_INVALID_ARG;
  int64_t n = 1;
  for (int f = 0; f < nf; ++f) {
    if (dims[f] < 0 || dims[f] > kMaxDim) return GPTQ2D_ERR_INVALID_ARG;
    n *= dims[f];
    if (n > kMaxDim) return GPTQ2D_ERR_INVALID_ARG;
  }
  GridSpec gs;
  const int rc = check_grid_call(W, w_dtype, m, n, ldw, grid, Q, ldq, stats, &gs);
  if (rc != GPTQ2D_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (m == 0 || n == 0)
    return quantize_launch(W, w_dtype, (int)m, (int)n, ldw, M_L, ldl, nullptr, 0, grid->scales,
                           grid->bits, grid->clamp, static_cast<int8_t*>(Q), ldq, stats, ws, s, 0,
                           nullptr, nullptr, &gs);
  int nin = 0;
  if (kron_inner(nf, dims, &nin) == 0) return GPTQ2D_ERR_INVALID_ARG;
  if (!M_L || ldl < m) return GPTQ2D_ERR_INVALID_ARG;
  for (int f = 0; f < nf; ++f)
    if (!M[f] || ldm[f] < dims[f]) return GPTQ2D_ERR_INVALID_ARG;
  if (!ws || !aligned256(ws) || ws_bytes < quantize_kron_ws_bytes(m, nf, dims))
    return GPTQ2D_ERR_WORKSPACE;
  if (check_device_pointers({W, M_L, grid->scales, grid->zeros, Q, stats, ws}) != GPTQ2D_OK)
    return GPTQ2D_ERR_INVALID_ARG;
  for (int f = 0; f < nf; ++f)
    if (check_device_pointers({M[f]}) != GPTQ2D_OK) return GPTQ2D_ERR_INVALID_ARG;
  KronSpec ks;
  ks.nf = nf;
  ks.M = M;
  ks.dims = dims;
  ks.ldm = ldm;
  return quantize_launch(W, w_dtype, (int)m, (int)n, ldw, M_L, ldl, nullptr, 0, grid->scales,
                         grid->bits, grid->clamp, static_cast<int8_t*>(Q), ldq, stats, ws, s, 0,
                         nullptr, nullptr, &gs, &ks);
}

int gptq2d_quantize_kron(const void* W, int w_dtype, int64_t m, int64_t ldw, const double* M_L,
                         int64_t ldl, int nf, const double* const* M, const int64_t* dims,
                         const int64_t* ldm, const float* scales, int bits, int clamp, int8_t* Q,
                         int64_t ldq, gptq2d_stats* stats, void* ws, size_t ws_bytes,
                         void* stream) {
  // the symmetric grid with one scale per row
  gptq2d_grid g{};
  g.bits = bits;
  g.clamp = clamp;
  g.group_size = 0;
  g.scales = scales;
  g.ld_scales = 1;
  g.zeros = nullptr;
  g.packed = 0;
  return gptq2d_quantize_kron_grid(W, w_dtype, m, ldw, M_L, ldl, nf, M, dims, ldm, &g, Q, ldq,
                                   stats, ws, ws_bytes, stream);
}

// ---------------------------------------------------------------------------
// A block of layers (gptq2d_quantize_block)
// ---------------------------------------------------------------------------
namespace {
struct BlockLayout {
  size_t slot, off_piv, off_q, total;
};
// Two factor slots (each holds one layer's M_L then M_R, both dense with ld = m, n),
// 512 bytes of pivot words per layer, one rounding workspace for the largest layer.
BlockLayout block_layout(const gptq2d_layer* L, int nl) {
  BlockLayout B{0, 0, 0, 0};
  size_t q = 256;
  for (int i = 0; i < nl; ++i) {
    const size_t fl = align256((size_t)L[i].m * L[i].m * sizeof(double)) +
                      align256((size_t)L[i].n * L[i].n * sizeof(double));
    B.slot = std::max(B.slot, fl);
    if (L[i].m > 0 && L[i].n > 0) q = std::max(q, quantize_ws_bytes(L[i].m, L[i].n));
  }
  B.off_piv = 2 * B.slot;
  B.off_q = B.off_piv + align256((size_t)nl * 512);
  B.total = B.off_q + align256(q);
  return B;
}
}  // namespace

size_t gptq2d_block_workspace_size(const gptq2d_layer* layers, int nl) {
  if (nl < 0 || (nl > 0 && !layers)) return 0;
  for (int i = 0; i < nl; ++i)
    if (layers[i].m < 0 || layers[i].n < 0 || layers[i].m > kMaxDim || layers[i].n > kMaxDim)
      return 0;
  return block_layout(layers, nl).total;
}

int gptq2d_quantize_block(const gptq2d_layer* L, int nl, void* ws, size_t ws_bytes, void* stream,
                          int64_t* bad_layer, int64_t* bad_pivot, int* which_factor) {
  if (bad_layer) *bad_layer = -1;
  if (bad_pivot) *bad_pivot = -1;
  if (which_factor) *which_factor = -1;
  if (nl < 0 || (nl > 0 && !L)) return GPTQ2D_ERR_INVALID_ARG;
  if (nl == 0) return GPTQ2D_OK;
  std::vector<GridSpec> gs(nl);
  for (int i = 0; i < nl; ++i) {
    const gptq2d_layer& l = L[i];
    const int rc = check_grid_call(l.W, l.w_dtype, l.m, l.n, l.ldw, &l.grid, l.Q, l.ldq, l.stats,
                                   &gs[i]);
    if (rc != GPTQ2D_OK) return rc;
    if (l.h_dtype != GPTQ2D_F32 && l.h_dtype != GPTQ2D_F64) return GPTQ2D_ERR_INVALID_ARG;
    if (l.m > 0 && (!l.H_L || l.ldhl < l.m)) return GPTQ2D_ERR_INVALID_ARG;
    if (l.n > 0 && (!l.H_R || l.ldhr < l.n)) return GPTQ2D_ERR_INVALID_ARG;
  }
  const BlockLayout B = block_layout(L, nl);
  if (!ws || !aligned256(ws) || ws_bytes < B.total) return GPTQ2D_ERR_WORKSPACE;
  for (int i = 0; i < nl; ++i) {
    const gptq2d_layer& l = L[i];
    if (l.m == 0 || l.n == 0) continue;
    if (check_device_pointers({l.W, l.H_L, l.H_R, l.grid.scales, l.grid.zeros, l.Q, l.stats}) !=
        GPTQ2D_OK)
      return GPTQ2D_ERR_INVALID_ARG;
  }
  if (check_device_pointers({ws}) != GPTQ2D_OK) return GPTQ2D_ERR_INVALID_ARG;
  DevStreams* ds = nullptr;
  int rc = dev_streams(&ds);
  if (rc != GPTQ2D_OK) return rc;
  std::lock_guard<std::recursive_mutex> lk(ds->mu);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(ws);
  bool ok = cudaEventRecord(ds->blk_start, s) == cudaSuccess &&
            cudaStreamWaitEvent(ds->blk_p, ds->blk_start, 0) == cudaSuccess &&
            cudaStreamWaitEvent(ds->blk_q, ds->blk_start, 0) == cudaSuccess;
  if (!ok) return GPTQ2D_ERR_CUDA;
  auto ML = [&](int i) { return reinterpret_cast<double*>(base + (i & 1) * B.slot); };
  auto MR = [&](int i) {
    return reinterpret_cast<double*>(base + (i & 1) * B.slot +
                                     align256((size_t)L[i].m * L[i].m * sizeof(double)));
  };
  // The factors of layer i on the second factor pairs, beside the rounding of layer
  // i - 1; slot i & 1 is free once layer i - 2 is rounded.
  auto prep = [&](int i) -> int {
    const gptq2d_layer& l = L[i];
    if (i >= 2 && cudaStreamWaitEvent(ds->blk_p, ds->blk_quant[i & 1], 0) != cudaSuccess)
      return GPTQ2D_ERR_CUDA;
    char* pv = base + B.off_piv + (size_t)i * 512;
    if (cudaMemsetAsync(pv, 0xFF, 512, ds->blk_p) != cudaSuccess) return GPTQ2D_ERR_CUDA;
    const int r = prepare_pair_launch(l.H_L, l.m, l.ldhl, l.H_R, l.n, l.ldhr, l.h_dtype, ML(i), l.m,
                                      MR(i), l.n, pv, pv + 256, ds->blk_p, nullptr, nullptr, true);
    if (r != GPTQ2D_OK) return r;
    return cudaEventRecord(ds->blk_prep[i & 1], ds->blk_p) == cudaSuccess ? GPTQ2D_OK
                                                                           : GPTQ2D_ERR_CUDA;
  };
  auto quant = [&](int i) -> int {
    const gptq2d_layer& l = L[i];
    if (cudaStreamWaitEvent(ds->blk_q, ds->blk_prep[i & 1], 0) != cudaSuccess) return GPTQ2D_ERR_CUDA;
    const int r = quantize_launch(l.W, l.w_dtype, (int)l.m, (int)l.n, l.ldw, ML(i), l.m, MR(i), l.n,
                                  l.grid.scales, l.grid.bits, l.grid.clamp,
                                  static_cast<int8_t*>(l.Q), l.ldq, l.stats, base + B.off_q,
                                  ds->blk_q, 0, nullptr, nullptr, &gs[i]);
    if (r != GPTQ2D_OK) return r;
    return cudaEventRecord(ds->blk_quant[i & 1], ds->blk_q) == cudaSuccess ? GPTQ2D_OK
                                                                            : GPTQ2D_ERR_CUDA;
  };
  rc = prep(0);
  if (rc == GPTQ2D_OK && nl > 1) rc = prep(1);
  for (int i = 0; i < nl && rc == GPTQ2D_OK; ++i) {
    rc = quant(i);
    if (rc == GPTQ2D_OK && i + 2 < nl) rc = prep(i + 2);
  }
  ok = cudaEventRecord(ds->blk_end[0], ds->blk_p) == cudaSuccess &&
       cudaEventRecord(ds->blk_end[1], ds->blk_q) == cudaSuccess &&
       cudaStreamWaitEvent(s, ds->blk_end[0], 0) == cudaSuccess &&
       cudaStreamWaitEvent(s, ds->blk_end[1], 0) == cudaSuccess;
  if (rc != GPTQ2D_OK) return rc;
  if (!ok) return GPTQ2D_ERR_CUDA;
  // pivot words of every layer (two per layer: left, right)
  std::vector<long long> piv((size_t)nl * 64);
  if (cudaMemcpyAsync(piv.data(), base + B.off_piv, (size_t)nl * 512, cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return GPTQ2D_ERR_CUDA;
  for (int i = 0; i < nl; ++i)
    for (int side = 0; side < 2; ++side) {
      const long long p = piv[(size_t)i * 64 + side * 32];
      if (p >= 0 && ((side == 0 && L[i].m > 0) || (side == 1 && L[i].n > 0))) {
        if (bad_layer) *bad_layer = i;
        if (bad_pivot) *bad_pivot = p;
        if (which_factor) *which_factor = side;
        return GPTQ2D_ERR_NOT_SPD;
      }
    }
  return GPTQ2D_OK;
}

size_t gptq2d_round_host_workspace_size(int64_t m, int64_t n, int w_dtype, int h_dtype) {
  if (m <= 0 || n <= 0 || m > kMaxDim || n > kMaxDim) return 0;
  if (elem_size(w_dtype) == 0 || (h_dtype != GPTQ2D_F32 && h_dtype != GPTQ2D_F64)) return 0;
  return host_layout(m, n, w_dtype, h_dtype).total;
}

int gptq2d_round_host(const void* W, int w_dtype, int64_t m, int64_t n, const void* H_L,
                      const void* H_R, int h_dtype, const float* scales, int bits, int clamp,
                      int8_t* Q, gptq2d_stats* stats, void* ws, size_t ws_bytes, void* stream,
                      int64_t* bad_pivot, int* which_factor) {
  if (m <= 0 || n <= 0 || m > kMaxDim || n > kMaxDim) return GPTQ2D_ERR_INVALID_ARG;
  if (elem_size(w_dtype) == 0 || (h_dtype != GPTQ2D_F32 && h_dtype != GPTQ2D_F64))
    return GPTQ2D_ERR_INVALID_ARG;
  if (bits < 2 || bits > 8 || (clamp != 0 && clamp != 1)) return GPTQ2D_ERR_INVALID_ARG;
  if (!W || !H_L || !H_R || !scales || !Q || !stats) return GPTQ2D_ERR_INVALID_ARG;
  const HostWs L = host_layout(m, n, w_dtype, h_dtype);
  if (!ws || !aligned256(ws) || ws_bytes < L.total) return GPTQ2D_ERR_WORKSPACE;
  if (check_device_pointers({ws}) != GPTQ2D_OK) return GPTQ2D_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* b = static_cast<char*>(ws);
  const size_t hs = elem_size(h_dtype);
  DevStreams* ds = nullptr;
  int rc = dev_streams(&ds);
  if (rc != GPTQ2D_OK) return rc;
  // Inputs go over one copy stream in the order they are needed: the Grams, then W
  // and the scales.  Each factor starts once its Gram is in, and the rounding once
  // both factors and W are done, so the later copies run under the factorizations.
  // Only the lower triangle of a Gram is read, so each 64-row block is copied up to
  // the end of its diagonal block (about half of the matrix).
  auto copy_lower = [&](char* dst, const void* src, int64_t k) -> bool {
    for (int64_t r0 = 0; r0 < k; r0 += 64) {
      const int64_t rows = std::min<int64_t>(64, k - r0), cols = std::min<int64_t>(k, r0 + 64);
      if (cudaMemcpy2DAsync(dst + (size_t)r0 * k * hs, (size_t)k * hs,
                            static_cast<const char*>(src) + (size_t)r0 * k * hs, (size_t)k * hs,
                            (size_t)cols * hs, (size_t)rows, cudaMemcpyHostToDevice,
                            ds->cp) != cudaSuccess)
        return false;
    }
    return true;
  };
  std::lock_guard<std::recursive_mutex> lk(ds->mu);
  // the larger Gram first: its factorization takes longer
  const bool r_first = n > m;
  if (cudaEventRecord(ds->fork, s) != cudaSuccess ||
      cudaStreamWaitEvent(ds->cp, ds->fork, 0) != cudaSuccess ||
      !(r_first ? copy_lower(b + L.off_HR, H_R, n) : copy_lower(b + L.off_HL, H_L, m)) ||
      cudaEventRecord(ds->cp_ev[r_first ? 1 : 0], ds->cp) != cudaSuccess ||
      !(r_first ? copy_lower(b + L.off_HL, H_L, m) : copy_lower(b + L.off_HR, H_R, n)) ||
      cudaEventRecord(ds->cp_ev[r_first ? 0 : 1], ds->cp) != cudaSuccess ||
      cudaMemcpyAsync(b + L.off_W, W, (size_t)m * n * elem_size(w_dtype), cudaMemcpyHostToDevice,
                      ds->cp) ||
      cudaMemcpyAsync(b + L.off_s, scales, (size_t)m * sizeof(float), cudaMemcpyHostToDevice,
                      ds->cp) ||
      cudaEventRecord(ds->cp_ev[2], ds->cp) != cudaSuccess)
    return GPTQ2D_ERR_CUDA;
  double* ML = reinterpret_cast<double*>(b + L.off_ML);
  double* MR = reinterpret_cast<double*>(b + L.off_MR);
  rc = prepare_pair_launch(b + L.off_HL, m, m, b + L.off_HR, n, n, h_dtype, ML, m, MR, n,
                           b + L.off_pl, b + L.off_pr, s, ds->cp_ev[0], ds->cp_ev[1]);
  if (rc == GPTQ2D_OK && cudaStreamWaitEvent(s, ds->cp_ev[2], 0) != cudaSuccess)
    rc = GPTQ2D_ERR_CUDA;
  // Q goes back in up to four bands of tile rows, each as soon as its rows are final
  const int Tm = (int)((m + 63) / 64);
  int row_tile[4], nband = 0;
  for (int k = 0; k < 4; ++k) {
    const int last = (int)(((int64_t)(k + 1) * Tm + 3) / 4) - 1;
    if (last >= 0 && (nband == 0 || last > row_tile[nband - 1])) row_tile[nband++] = last;
  }
  if (rc == GPTQ2D_OK)
    rc = quantize_launch(b + L.off_W, w_dtype, (int)m, (int)n, n, ML, m, MR, n,
                         reinterpret_cast<const float*>(b + L.off_s), bits, clamp,
                         reinterpret_cast<int8_t*>(b + L.off_Q), n,
                         reinterpret_cast<gptq2d_stats*>(b + L.off_stats), b + L.off_q, s, nband,
                         row_tile, ds->q_ev);
  if (rc != GPTQ2D_OK) return rc;
  for (int k = 0, r0 = 0; k < nband; ++k) {
    const int r1 = (int)std::min<int64_t>(m, (int64_t)(row_tile[k] + 1) * 64);
    if (cudaStreamWaitEvent(ds->cp, ds->q_ev[k], 0) != cudaSuccess ||
        cudaMemcpyAsync(Q + (size_t)r0 * n, b + L.off_Q + (size_t)r0 * n, (size_t)(r1 - r0) * n,
                        cudaMemcpyDeviceToHost, ds->cp) != cudaSuccess)
      return GPTQ2D_ERR_CUDA;
    r0 = r1;
  }
  long long piv[2] = {-1, -1};
  if (cudaEventRecord(ds->cp_ev[2], ds->cp) != cudaSuccess ||
      cudaStreamWaitEvent(s, ds->cp_ev[2], 0) != cudaSuccess ||
      cudaMemcpyAsync(stats, b + L.off_stats, sizeof(gptq2d_stats), cudaMemcpyDeviceToHost, s) ||
      cudaMemcpyAsync(&piv[0], b + L.off_pl, sizeof(long long), cudaMemcpyDeviceToHost, s) ||
      cudaMemcpyAsync(&piv[1], b + L.off_pr, sizeof(long long), cudaMemcpyDeviceToHost, s))
    return GPTQ2D_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return GPTQ2D_ERR_CUDA;
  for (int f = 0; f < 2; ++f)
    if (pivot_status(piv[f]) != GPTQ2D_OK) {
      if (bad_pivot) *bad_pivot = piv[f] >= 0 ? piv[f] : -1;
      if (which_factor) *which_factor = f;
      return pivot_status(piv[f]);
    }
  if (bad_pivot) *bad_pivot = -1;
  if (which_factor) *which_factor = -1;
  return (int)stats->status;
}

}  // extern "C"

// The proxy loss of a given rounding, and of round-to-nearest.
//
// The two-sided quadratic metric (mind-verse.de "Neue Ansätze ... durch GPTQ-2D",
// "GPTQ-2D: Eine Weiterentwicklung der adaptiven Rundung"; arxivlens "GPTQ-2D:
// Cubic-Time Two-Sided Adaptive Rounding", Abstract) with dW = W - diag(s) Q and
// lower factors M^T M = H is
//     L(Q) = tr(dW^T H_L dW H_R) = || M_L dW M_R^T ||_F^2 .
// Round-to-nearest, q = clamp(rint(W / s)), is the baseline the pages measure GPTQ-2D
// against.  Unlike the rounding's own loss (accumulated entry by entry from the
// nearest-plane residual identity), this is a full quadratic form: two triangular
// matrix products of about mn(m + n) flops, as much work as the rounding.
//
//   dw_kernel      D = W - s q on the tile-padded m x n grid (zeros outside);
//   tri_kernel(R)  T = D M_R^T, T[i,j] = sum_{j' <= j} D[i,j'] M_R[j,j'];
//   tri_kernel(L)  U = M_L T,   U[i,j] = sum_{i' <= i} M_L[i,i'] T[i',j], and per tile
//                  the sum of U^2 (U itself is not stored);
//   sum_kernel     the tiles' sums in a fixed order (deterministic) into *loss.
// One CTA per 64 x 64 output tile, four warps on FP64 tensor-core products (a 32 x 32
// quadrant each), operand chunks double-buffered with cp.async.  Only the lower
// triangles of M_L and M_R are read (their upper triangles are ignored, as in the
// rounding).
#include <algorithm>

#include "common.cuh"

namespace gptq2d {
namespace {

constexpr int LLD = TB + 4;  // 68: row stride of the shared operand chunks
constexpr int LOSS_THREADS = 128;
constexpr int LOSS_SMEM = 4 * TB * LLD * (int)sizeof(double);  // A and B, double-buffered

struct LossArgs {
  const void* W;
  int64_t ldw;
  int m, n;
  const int8_t* Q;  // null: round to nearest
  int64_t ldq;
  const float* scales;
  double lo, hi;    // admissible integers (infinite without clamp)
  const double* ML;
  int64_t ldl;
  const double* MR;
  int64_t ldr;
  double* D;        // mp x np
  double* T;        // mp x np
  double* part;     // Tm x Tn tile sums
  int64_t mp, np;
  int Tm, Tn;
};

template <typename TW>
__global__ void __launch_bounds__(256) dw_kernel(LossArgs a) {
  const int64_t total = a.mp * a.np;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int i = (int)(e / a.np), j = (int)(e % a.np);
    double d = 0.0;
    if (i < a.m && j < a.n) {
      const double w = to_f64(static_cast<const TW*>(a.W)[(int64_t)i * a.ldw + j]);
      const double s = (double)a.scales[i];
      double q;
      if (a.Q) {
        q = (double)a.Q[(int64_t)i * a.ldq + j];
      } else {
        q = rint(w / s);
        q = q < a.lo ? a.lo : (q > a.hi ? a.hi : q);
      }
      d = w - s * q;
    }
    a.D[e] = d;
  }
}

// Copies the 64 x 64 block of M at (r0, c0) into shared memory [r][c] (stride LLD),
// keeping only the lower triangle of M (c <= r) and zero outside the k x k matrix.
// 8-byte copies: the caller's leading dimension may be odd.
__device__ __forceinline__ void load_lower(double* dst, const double* M, int64_t ld, int k, int r0,
                                           int c0) {
  for (int x = threadIdx.x; x < TB * TB; x += LOSS_THREADS) {
    const int r = x >> 6, c = x & 63;
    const bool ok = r0 + r < k && c0 + c < k && c0 + c <= r0 + r;
    cp_async8_zfill(dst + r * LLD + c, ok ? M + (int64_t)(r0 + r) * ld + c0 + c : M, ok);
  }
}
// Copies the 64 x 64 tile (R, C) of a tile-padded mp x np buffer (16-byte rows).
__device__ __forceinline__ void load_tile(double* dst, const double* X, int64_t ld, int R, int C) {
  for (int x = threadIdx.x; x < TB * TB / 2; x += LOSS_THREADS) {
    const int r = x >> 5, c2 = (x & 31) * 2;
    cp_async16_zfill(dst + r * LLD + c2, X + (int64_t)(R * TB + r) * ld + C * TB + c2, true);
  }
}

// right = true:  tile (I, J) of T = D M_R^T, chunks K = 0 .. J:  A = D[I,K] as [i][k],
//                B(k, j) = M_R[J-block row j][K-block col k] (stored [j][k]);
// right = false: tile (I, J) of U = M_L T, chunks K = 0 .. I:  A = M_L[I,K] as [i][k],
//                B(k, j) = T[K,J] (stored [k][j]); the tile's sum of squares to part.
template <bool RIGHT>
__global__ void __launch_bounds__(LOSS_THREADS, 1) tri_kernel(LossArgs a) {
  extern __shared__ __align__(128) double sm[];
  const int I = blockIdx.x / a.Tn, J = blockIdx.x % a.Tn;
  const int nk = (RIGHT ? J : I) + 1;
  auto stage_a = [&](int s) { return sm + (2 * s) * TB * LLD; };
  auto stage_b = [&](int s) { return sm + (2 * s + 1) * TB * LLD; };
  auto load = [&](int K, int s) {
    if (RIGHT) {
      load_tile(stage_a(s), a.D, a.np, I, K);
      load_lower(stage_b(s), a.MR, a.ldr, a.n, J * TB, K * TB);
    } else {
      load_lower(stage_a(s), a.ML, a.ldl, a.m, I * TB, K * TB);
      load_tile(stage_b(s), a.T, a.np, K, J);
    }
    cp_async_commit_group();
  };
  double acc[4][4][2] = {};
  load(0, 0);
  for (int K = 0; K < nk; ++K) {
    const int s = K & 1;
    if (K + 1 < nk) {
      load(K + 1, s ^ 1);
      cp_async_wait_group<1>();
    } else {
      cp_async_wait_group<0>();
    }
    __syncthreads();
    const double* As = stage_a(s);
    const double* Bs = stage_b(s);
    if (RIGHT)
      mma_64x64x64(acc, [&](int r, int k) { return As[r * LLD + k]; },
                   [&](int k, int c) { return Bs[c * LLD + k]; });
    else
      mma_64x64x64(acc, [&](int r, int k) { return As[r * LLD + k]; },
                   [&](int k, int c) { return Bs[k * LLD + c]; });
    __syncthreads();  // the stage is refilled by the next iteration's load
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int wr = (warp >> 1) * 32, wc = (warp & 1) * 32;
  if (RIGHT) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        double* o = a.T + (int64_t)(I * TB + wr + 8 * i + g) * a.np + J * TB + wc + 8 * j + 2 * t;
        *reinterpret_cast<double2*>(o) = make_double2(acc[i][j][0], acc[i][j][1]);
      }
  } else {
    double ss = 0.0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) ss += acc[i][j][0] * acc[i][j][0] + acc[i][j][1] * acc[i][j][1];
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_down_sync(0xffffffffu, ss, o);
    __shared__ double red[LOSS_THREADS / 32];
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    if (threadIdx.x == 0) {
      double tot = 0.0;
      for (int w = 0; w < LOSS_THREADS / 32; ++w) tot += red[w];
      a.part[blockIdx.x] = tot;
    }
  }
}

__global__ void __launch_bounds__(256) sum_kernel(const double* part, int n, double* out) {
  __shared__ double s[256];
  double v = 0.0;
  for (int i = threadIdx.x; i < n; i += 256) v += part[i];
  s[threadIdx.x] = v;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) s[threadIdx.x] += s[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) *out = s[0];
}

struct LossLayout {
  int64_t mp, np;
  int Tm, Tn;
  size_t off_D, off_T, off_part, total;
};
LossLayout loss_layout(int64_t m, int64_t n) {
  LossLayout L;
  L.mp = round_up(m, TB);
  L.np = round_up(n, TB);
  L.Tm = (int)(L.mp / TB);
  L.Tn = (int)(L.np / TB);
  size_t o = 0;
  L.off_D = o; o += align256((size_t)L.mp * L.np * sizeof(double));
  L.off_T = o; o += align256((size_t)L.mp * L.np * sizeof(double));
  L.off_part = o; o += align256((size_t)L.Tm * L.Tn * sizeof(double));
  L.total = o;
  return L;
}

constexpr int64_t kLossMaxDim = (int64_t)1 << 20;
std::atomic<uint64_t> g_loss_smem_set[2];

}  // namespace
}  // namespace gptq2d

using namespace gptq2d;

extern "C" size_t gptq2d_proxy_loss_workspace_size(int64_t m, int64_t n) {
  if (m < 0 || n < 0 || m > kLossMaxDim || n > kLossMaxDim) return 0;
  if (m == 0 || n == 0) return 256;
  return loss_layout(m, n).total;
}

extern "C" int gptq2d_proxy_loss(const void* W, int w_dtype, int64_t m, int64_t n, int64_t ldw,
                                 const int8_t* Q, int64_t ldq, const float* scales, int bits,
                                 int clamp, const double* M_L, int64_t ldl, const double* M_R,
                                 int64_t ldr, double* loss, void* ws, size_t ws_bytes,
                                 void* stream) {
  if (m < 0 || n < 0 || m > kLossMaxDim || n > kLossMaxDim) return GPTQ2D_ERR_INVALID_ARG;
  if (w_dtype != GPTQ2D_F32 && w_dtype != GPTQ2D_BF16 && w_dtype != GPTQ2D_F64)
    return GPTQ2D_ERR_INVALID_ARG;
  if (bits < 2 || bits > 8 || (clamp != 0 && clamp != 1) || !loss) return GPTQ2D_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (m == 0 || n == 0) {
    if (check_device_pointers({loss}) != GPTQ2D_OK) return GPTQ2D_ERR_INVALID_ARG;
    return cudaMemsetAsync(loss, 0, sizeof(double), s) == cudaSuccess ? GPTQ2D_OK
                                                                      : GPTQ2D_ERR_CUDA;
  }
  if (!W || !scales || !M_L || !M_R) return GPTQ2D_ERR_INVALID_ARG;
  if (ldw < n || ldl < m || ldr < n || (Q && ldq < n)) return GPTQ2D_ERR_INVALID_ARG;
  const LossLayout L = loss_layout(m, n);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || ws_bytes < L.total)
    return GPTQ2D_ERR_WORKSPACE;
  if (check_device_pointers({W, Q, scales, M_L, M_R, loss, ws}) != GPTQ2D_OK)
    return GPTQ2D_ERR_INVALID_ARG;
  if (ensure_smem(tri_kernel<true>, LOSS_SMEM, g_loss_smem_set[0]) != cudaSuccess ||
      ensure_smem(tri_kernel<false>, LOSS_SMEM, g_loss_smem_set[1]) != cudaSuccess)
    return GPTQ2D_ERR_CUDA;
  char* b = static_cast<char*>(ws);
  LossArgs a;
  a.W = W;
  a.ldw = ldw;
  a.m = (int)m;
  a.n = (int)n;
  a.Q = Q;
  a.ldq = ldq;
  a.scales = scales;
  a.lo = clamp ? -(double)(1 << (bits - 1)) : -HUGE_VAL;
  a.hi = clamp ? (double)((1 << (bits - 1)) - 1) : HUGE_VAL;
  a.ML = M_L;
  a.ldl = ldl;
  a.MR = M_R;
  a.ldr = ldr;
  a.D = reinterpret_cast<double*>(b + L.off_D);
  a.T = reinterpret_cast<double*>(b + L.off_T);
  a.part = reinterpret_cast<double*>(b + L.off_part);
  a.mp = L.mp;
  a.np = L.np;
  a.Tm = L.Tm;
  a.Tn = L.Tn;
  const int tiles = L.Tm * L.Tn;
  const int eb = (int)std::min<int64_t>((L.mp * L.np + 255) / 256, 148 * 16);
  switch (w_dtype) {
    case GPTQ2D_F32: GPTQ2D_LAUNCH(KC_OTHER, s, dw_kernel<float><<<eb, 256, 0, s>>>(a)); break;
    case GPTQ2D_BF16:
      GPTQ2D_LAUNCH(KC_OTHER, s, dw_kernel<__nv_bfloat16><<<eb, 256, 0, s>>>(a));
      break;
    default: GPTQ2D_LAUNCH(KC_OTHER, s, dw_kernel<double><<<eb, 256, 0, s>>>(a)); break;
  }
  GPTQ2D_LAUNCH(KC_OTHER, s, tri_kernel<true><<<tiles, LOSS_THREADS, LOSS_SMEM, s>>>(a));
  GPTQ2D_LAUNCH(KC_OTHER, s, tri_kernel<false><<<tiles, LOSS_THREADS, LOSS_SMEM, s>>>(a));
  GPTQ2D_LAUNCH(KC_OTHER, s, sum_kernel<<<1, 256, 0, s>>>(a.part, tiles, loss));
  return cudaGetLastError() == cudaSuccess ? GPTQ2D_OK : GPTQ2D_ERR_CUDA;
}

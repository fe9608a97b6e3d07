// Factor preparation: H = M^T M with M lower triangular ("reverse" Cholesky).
//
// The bases of the two-sided problem are fixed, so each Kronecker factor is
// factored once before rounding (arxivlens "GPTQ-2D: Cubic-Time Two-Sided
// Adaptive Rounding", Analysis > Limitations and Future work, on the fixed
// bases and their Gram factorizations).  With M_L, M_R lower and M^T M = H,
// M_R (x) M_L is the lower-triangular factor of the Kronecker Gram in the
// column-major order of vec(W), which is what the index-0-first nearest-plane
// sweep needs.
//
// Blocked, right-looking, eliminating from the LAST block row upwards.  For
// block row K (rows [64K, 64K + nb)) of the still-unfactored leading part A:
//   1. M_KK^T M_KK = A_KK            (in-SM factorization of one 64x64 block)
//   2. M_Kb = M_KK^{-T} A_Kb, b < K  (triangular solve of the block row)
//   3. A_IJ -= M_KI^T M_KJ, J<=I<K   (rank-64 trailing update on FP64 tensor cores)
// Everything is fp64.  A pivot that is not positive and finite stops the
// factorization and is reported through a pivot word in the workspace.
#include <algorithm>

#include "common.cuh"

namespace gptq2d {

namespace {

constexpr int PLD = TB + 1;  // leading dimension of the in-SM factor / panel tiles
constexpr int KLD = TB + 8;  // leading dimension of [k][*] operand tiles (72: conflict-free fragments)
constexpr int TR_THREADS = 128;
constexpr int MAX_TR_GROUPS = 512;

template <typename TH>
__global__ void __launch_bounds__(256) convert_lower_kernel(const TH* __restrict__ H, int64_t ldh,
                                                            int k, double* __restrict__ M,
                                                            int64_t ldm, long long* info) {
  if (blockIdx.x == 0 && threadIdx.x == 0) *info = -1;
  const int64_t total = (int64_t)k * k;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int i = (int)(e / k), j = (int)(e % k);
    M[(int64_t)i * ldm + j] = (j <= i) ? to_f64(H[(int64_t)i * ldh + j]) : 0.0;
  }
}

// One launch per block row K.  CTA K factors the diagonal block and writes it;
// CTAs b < K factor the same block redundantly (cheaper than a separate launch)
// and solve their block M_Kb = M_KK^{-T} A_Kb.
//
// Both phases keep their 64 x 64 block in registers: thread (i = tid/4, q =
// tid%4) holds row i, columns q + 4u (u < 16).  The pivot and solve loops are
// unrolled so that every register index is a compile-time constant.  Per pivot
// p (last row first): the four threads of row p scale it by 1/sqrt(A[p][p]) and
// publish it to a double-buffered shared row; after one barrier every row i < p
// applies A[i][j] -= M[p][i] M[p][j] from broadcast reads.  The strict upper
// part of the register block is never read (published rows are zero beyond p).
__global__ void __launch_bounds__(256) panel_kernel(double* __restrict__ M, int64_t ldm, int k,
                                                    int K, long long* info) {
  if (*(volatile long long*)info >= 0) return;
  __shared__ double S[TB * PLD];      // the factored diagonal block M_KK
  __shared__ double rowb[2][TB];      // published pivot row / solved row
  __shared__ double invd[TB];         // 1 / M_KK[p][p]
  __shared__ int bad;
  const int tid = threadIdx.x, lane = tid & 31;
  const int i = tid >> 2, q = tid & 3;
  const int rb = K * TB, nb = min(TB, k - rb);
  const int b = blockIdx.x;
  if (tid == 0) bad = -1;

  double v[TB / 4];
#pragma unroll
  for (int u = 0; u < TB / 4; ++u) {
    const int j = q + 4 * u;
    v[u] = (i < nb && j <= i) ? M[(int64_t)(rb + i) * ldm + rb + j] : 0.0;
  }
  __syncthreads();

#pragma unroll
  for (int p = TB - 1; p >= 0; --p) {
    if (p < nb) {
      // every lane takes part in the shuffle; row p's four threads use the value
      const double piv = __shfl_sync(0xffffffffu, v[p >> 2], (lane & ~3) | (p & 3));
      if (i == p) {
        const bool ok = piv > 0.0 && isfinite(piv);
        const double r = ok ? rsqrt(piv) : 0.0;
#pragma unroll
        for (int u = 0; u < TB / 4; ++u) {
          const int j = q + 4 * u;
          v[u] = (j <= p) ? v[u] * r : 0.0;
          rowb[p & 1][j] = v[u];
        }
        if (q == 0) {
          invd[p] = r;
          if (!ok) bad = rb + p;
        }
      }
      __syncthreads();
      if (bad >= 0) {  // uniform: every thread reads the flag after the barrier
        if (tid == 0) *info = bad;
        return;
      }
      if (i < p) {
        const double mi = rowb[p & 1][i];
#pragma unroll
        for (int u = 0; u < TB / 4; ++u) v[u] = fma(-mi, rowb[p & 1][q + 4 * u], v[u]);
      }
    }
  }
  // registers now hold M_KK (lower part); the diagonal is A[p][p] * (1/sqrt(A[p][p]))
#pragma unroll
  for (int u = 0; u < TB / 4; ++u) {
    const int j = q + 4 * u;
    S[i * PLD + j] = (i < nb && j <= i) ? v[u] : 0.0;
  }
  __syncthreads();
  if (b == K) {
    for (int e = tid; e < nb * TB; e += blockDim.x) {
      const int r = e >> 6, c = e & 63;
      if (c < nb) M[(int64_t)(rb + r) * ldm + rb + c] = S[r * PLD + c];
    }
    return;
  }

  // X <- M_KK^{-T} X by back substitution (M_KK^T is upper triangular)
#pragma unroll
  for (int u = 0; u < TB / 4; ++u)
    v[u] = (i < nb) ? M[(int64_t)(rb + i) * ldm + (int64_t)b * TB + q + 4 * u] : 0.0;
#pragma unroll
  for (int r = TB - 1; r >= 0; --r) {
    if (r < nb) {
      if (i == r) {
        const double iv = invd[r];
#pragma unroll
        for (int u = 0; u < TB / 4; ++u) {
          v[u] *= iv;
          rowb[r & 1][q + 4 * u] = v[u];
        }
      }
      __syncthreads();
      if (i < r) {
        const double mr = S[r * PLD + i];
#pragma unroll
        for (int u = 0; u < TB / 4; ++u) v[u] = fma(-mr, rowb[r & 1][q + 4 * u], v[u]);
      }
    }
  }
  if (i < nb) {
#pragma unroll
    for (int u = 0; u < TB / 4; ++u)
      M[(int64_t)(rb + i) * ldm + (int64_t)b * TB + q + 4 * u] = v[u];
  }
}

// Copies the nb x 64 block of M at (row0, col0) into shared memory [r][c] with
// row stride KLD, zero rows beyond nb.  16-byte copies when every row start is
// 16-byte aligned, else 8-byte copies.
template <bool V16>
__device__ __forceinline__ void load_rows(double* dst, const double* M, int64_t ldm, int row0,
                                          int col0, int nb) {
  if (V16) {
    for (int x = threadIdx.x; x < TB * TB / 2; x += TR_THREADS) {
      const int r = x >> 5, c2 = (x & 31) * 2;
      const bool ok = r < nb;
      const double* src = ok ? M + (int64_t)(row0 + r) * ldm + col0 + c2 : M;
      cp_async16_zfill(dst + r * KLD + c2, src, ok);
    }
  } else {
    for (int x = threadIdx.x; x < TB * TB; x += TR_THREADS) {
      const int r = x >> 6, c = x & 63;
      const bool ok = r < nb;
      const double* src = ok ? M + (int64_t)(row0 + r) * ldm + col0 + c : M;
      cp_async8_zfill(dst + r * KLD + c, src, ok);
    }
  }
}

struct TrailPlan {
  int K, I0, ng;                 // block row, first group, number of groups
  int per_cta;                   // blocks J per CTA
  int start[MAX_TR_GROUPS + 1];  // first CTA of each group; group g updates A[I0+g][0..I0+g]
};

constexpr int TR_SMEM = 3 * TB * KLD * (int)sizeof(double);

// A_IJ -= M_KI^T M_KJ.  Each CTA keeps M_KI in shared memory and streams the
// M_KJ blocks of its range of J through a double buffer.
template <bool V16>
__global__ void __launch_bounds__(TR_THREADS, 2) trailing_kernel(double* __restrict__ M,
                                                                 int64_t ldm, int k,
                                                                 const long long* info,
                                                                 TrailPlan pl) {
  if (*(volatile const long long*)info >= 0) return;
  extern __shared__ __align__(16) double sm[];
  double* Xs = sm;  // Xs[r][i] = M[rb + r][64 I + i]
  double* const Y0 = sm + TB * KLD;
  auto ybuf = [&](int bsel) { return Y0 + bsel * (TB * KLD); };
  const int cta = blockIdx.x;
  int g;
  {
    int lo = 0, hi = pl.ng;  // largest g with start[g] <= cta
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pl.start[mid] <= cta) lo = mid; else hi = mid;
    }
    g = lo;
  }
  const int I = pl.I0 + g;
  const int first = (cta - pl.start[g]) * pl.per_cta;
  const int last = min(first + pl.per_cta, I + 1);
  if (first >= last) return;
  const int rb = pl.K * TB, nb = min(TB, k - rb);

  load_rows<V16>(Xs, M, ldm, rb, I * TB, nb);
  load_rows<V16>(ybuf(0), M, ldm, rb, first * TB, nb);
  cp_async_commit_group();

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5, g8 = lane >> 2, t4 = lane & 3;
  const int wr = (warp >> 1) * 32, wc = (warp & 1) * 32;
  for (int J = first; J < last; ++J) {
    const int bsel = (J - first) & 1;
    if (J + 1 < last) {
      load_rows<V16>(ybuf(bsel ^ 1), M, ldm, rb, (J + 1) * TB, nb);
      cp_async_commit_group();
      cp_async_wait_group<1>();
    } else {
      cp_async_wait_group<0>();
    }
    __syncthreads();
    const double* Ys = ybuf(bsel);
    double acc[4][4][2] = {};
    mma_64x64x64(
        acc, [&](int row, int kk) { return Xs[kk * KLD + row]; },
        [&](int kk, int col) { return Ys[kk * KLD + col]; }, (nb + 3) & ~3);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = wr + i * 8 + g8, c = wc + j * 8 + 2 * t4;
        double* dst = M + (int64_t)(I * TB + r) * ldm + (int64_t)J * TB + c;
        if (I != J || c <= r) dst[0] -= acc[i][j][0];
        if (I != J || c + 1 <= r) dst[1] -= acc[i][j][1];
      }
    __syncthreads();
  }
}

std::atomic<uint64_t> g_trailing_smem_set[2];
std::atomic<uint64_t> g_panel_smem_set{0};

int sm_count() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms > 0 ? sms : 148;
}

int prepare_enqueue(const void* H, int h_dtype, int k, int64_t ldh, double* M, int64_t ldm,
                    void* ws, cudaStream_t s, int sms) {
  long long* info = static_cast<long long*>(ws);
  const int T = (k + TB - 1) / TB;
  const int cblocks = (int)std::min<int64_t>(((int64_t)k * k + 255) / 256, (int64_t)sms * 16);
  if (h_dtype == GPTQ2D_F32)
    GPTQ2D_LAUNCH(KC_OTHER, s,
                  convert_lower_kernel<float><<<cblocks, 256, 0, s>>>(
                      static_cast<const float*>(H), ldh, k, M, ldm, info));
  else
    GPTQ2D_LAUNCH(KC_OTHER, s,
                  convert_lower_kernel<double><<<cblocks, 256, 0, s>>>(
                      static_cast<const double*>(H), ldh, k, M, ldm, info));
  const int psmem = 0;
  const bool v16 = (ldm % 2 == 0) && ((reinterpret_cast<uintptr_t>(M) & 15u) == 0);
  if (ensure_smem(trailing_kernel<true>, TR_SMEM, g_trailing_smem_set[0]) != cudaSuccess ||
      ensure_smem(trailing_kernel<false>, TR_SMEM, g_trailing_smem_set[1]) != cudaSuccess ||
      ensure_smem(panel_kernel, psmem, g_panel_smem_set) != cudaSuccess)
    return GPTQ2D_ERR_CUDA;
  const int target = 2 * sms;
  for (int K = T - 1; K >= 0; --K) {
    GPTQ2D_LAUNCH(KC_PREP_PANEL, s, panel_kernel<<<K + 1, 256, psmem, s>>>(M, ldm, k, K, info));
    if (K == 0) continue;
    const long long total = (long long)K * (K + 1) / 2;
    const int per_cta = (int)std::max<long long>(1, (total + target - 1) / target);
    for (int g0 = 0; g0 < K; g0 += MAX_TR_GROUPS) {
      TrailPlan pl;
      pl.K = K;
      pl.I0 = g0;
      pl.ng = std::min(K - g0, MAX_TR_GROUPS);
      pl.per_cta = per_cta;
      int ctas = 0;
      for (int gi = 0; gi < pl.ng; ++gi) {
        pl.start[gi] = ctas;
        ctas += (g0 + gi + 1 + per_cta - 1) / per_cta;
      }
      pl.start[pl.ng] = ctas;
      if (v16)
        GPTQ2D_LAUNCH(KC_PREP_TRAILING, s,
                      trailing_kernel<true><<<ctas, TR_THREADS, TR_SMEM, s>>>(M, ldm, k, info, pl));
      else
        GPTQ2D_LAUNCH(KC_PREP_TRAILING, s,
                      trailing_kernel<false><<<ctas, TR_THREADS, TR_SMEM, s>>>(M, ldm, k, info, pl));
    }
  }
  return cudaGetLastError() == cudaSuccess ? GPTQ2D_OK : GPTQ2D_ERR_CUDA;
}

}  // namespace

size_t prepare_ws_bytes(int64_t) { return 256; }

int prepare_launch(const void* H, int h_dtype, int k, int64_t ldh, double* M, int64_t ldm,
                   void* ws, cudaStream_t s) {
  return prepare_enqueue(H, h_dtype, k, ldh, M, ldm, ws, s, sm_count());
}

int prepare_pair_launch(const void* H_L, int64_t m, int64_t ldhl, const void* H_R, int64_t n,
                        int64_t ldhr, int h_dtype, double* M_L, int64_t ldml, double* M_R,
                        int64_t ldmr, void* ws_l, void* ws_r, cudaStream_t s) {
  DevStreams* ds = nullptr;
  int rc = dev_streams(&ds);
  if (rc != GPTQ2D_OK) return rc;
  std::lock_guard<std::mutex> lk(ds->mu);
  if (cudaEventRecord(ds->fork, s) != cudaSuccess ||
      cudaStreamWaitEvent(ds->hi, ds->fork, 0) != cudaSuccess ||
      cudaStreamWaitEvent(ds->lo, ds->fork, 0) != cudaSuccess)
    return GPTQ2D_ERR_CUDA;
  if (m > 0) rc = prepare_enqueue(H_L, h_dtype, (int)m, ldhl, M_L, ldml, ws_l, ds->hi, ds->sms);
  if (rc == GPTQ2D_OK && n > 0)
    rc = prepare_enqueue(H_R, h_dtype, (int)n, ldhr, M_R, ldmr, ws_r, ds->lo, ds->sms);
  const bool ok = cudaEventRecord(ds->join_hi, ds->hi) == cudaSuccess &&
                  cudaEventRecord(ds->join_lo, ds->lo) == cudaSuccess &&
                  cudaStreamWaitEvent(s, ds->join_hi, 0) == cudaSuccess &&
                  cudaStreamWaitEvent(s, ds->join_lo, 0) == cudaSuccess;
  if (rc != GPTQ2D_OK) return rc;
  return ok ? GPTQ2D_OK : GPTQ2D_ERR_CUDA;
}

}  // namespace gptq2d

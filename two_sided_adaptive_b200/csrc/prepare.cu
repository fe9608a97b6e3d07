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
#include "common.cuh"

namespace gptq2d {

namespace {

constexpr int PLD = TB + 1;   // leading dimension of the in-SM factor / panel tiles
constexpr int SLD = TB + 8;   // leading dimension of [k][*] operand tiles (72: conflict-free fragments)

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
// CTAs b < K factor the same block redundantly in shared memory (cheaper than a
// separate launch) and solve their block M_Kb.
__global__ void __launch_bounds__(256) panel_kernel(double* __restrict__ M, int64_t ldm, int k,
                                                    int K, long long* info) {
  if (*(volatile long long*)info >= 0) return;
  extern __shared__ double psm[];
  double* S = psm;            // diagonal block, factored in place
  double* X = psm + TB * PLD; // block M_Kb being solved
  const int tid = threadIdx.x;
  const int rb = K * TB, nb = min(TB, k - rb);
  const int b = blockIdx.x;

  for (int e = tid; e < TB * TB; e += blockDim.x) {
    const int r = e >> 6, c = e & 63;
    S[r * PLD + c] = (r < nb && c <= r) ? M[(int64_t)(rb + r) * ldm + rb + c] : 0.0;
    if (b < K) X[r * PLD + c] = (r < nb) ? M[(int64_t)(rb + r) * ldm + (int64_t)b * TB + c] : 0.0;
  }
  __syncthreads();

  // Reverse factorization of the diagonal block: the last row first.
  for (int p = nb - 1; p >= 0; --p) {
    const double piv = S[p * PLD + p];
    if (!(piv > 0.0) || !isfinite(piv)) {  // uniform: every thread read the same value
      if (tid == 0) *info = rb + p;  // every CTA of this launch finds the same pivot
      return;
    }
    const double dp = sqrt(piv);
    __syncthreads();
    for (int j = tid; j < p; j += blockDim.x) S[p * PLD + j] /= dp;
    if (tid == 0) S[p * PLD + p] = dp;
    __syncthreads();
    for (int e = tid; e < p * TB; e += blockDim.x) {
      const int i = e >> 6, j = e & 63;
      if (j <= i) S[i * PLD + j] -= S[p * PLD + i] * S[p * PLD + j];
    }
    __syncthreads();
  }

  if (b == K) {
    for (int e = tid; e < nb * TB; e += blockDim.x) {
      const int r = e >> 6, c = e & 63;
      if (c < nb) M[(int64_t)(rb + r) * ldm + rb + c] = (c <= r) ? S[r * PLD + c] : 0.0;
    }
    return;
  }

  // X <- M_KK^{-T} X by back substitution (M_KK^T is upper triangular).
  for (int r = nb - 1; r >= 0; --r) {
    if (tid < TB) X[r * PLD + tid] /= S[r * PLD + r];
    __syncthreads();
    for (int e = tid; e < r * TB; e += blockDim.x) {
      const int r2 = e >> 6, c = e & 63;
      X[r2 * PLD + c] -= S[r * PLD + r2] * X[r * PLD + c];
    }
    __syncthreads();
  }
  for (int e = tid; e < nb * TB; e += blockDim.x) {
    const int r = e >> 6, c = e & 63;
    M[(int64_t)(rb + r) * ldm + (int64_t)b * TB + c] = X[r * PLD + c];
  }
}

// A_IJ -= M_KI^T M_KJ for the lower block pairs J <= I < K (blockIdx.x enumerates them).
__global__ void __launch_bounds__(128) trailing_kernel(double* __restrict__ M, int64_t ldm, int k,
                                                       int K, const long long* info) {
  if (*(volatile const long long*)info >= 0) return;
  extern __shared__ double sm[];
  double* Xs = sm;             // Xs[r][i] = M[rb + r][64 I + i]
  double* Ys = sm + TB * SLD;  // Ys[r][j] = M[rb + r][64 J + j]
  const int e = blockIdx.x;
  int I = (int)((sqrt(8.0 * e + 1.0) - 1.0) * 0.5);
  while ((I + 1) * (I + 2) / 2 <= e) ++I;
  while (I * (I + 1) / 2 > e) --I;
  const int J = e - I * (I + 1) / 2;
  const int rb = K * TB, nb = min(TB, k - rb);
  const int tid = threadIdx.x;

  for (int x = tid; x < TB * TB / 2; x += blockDim.x) {
    const int r = x >> 5, c2 = (x & 31) * 2;
    double2 vx = make_double2(0.0, 0.0), vy = make_double2(0.0, 0.0);
    if (r < nb) {
      const double* row = M + (int64_t)(rb + r) * ldm;
      vx = make_double2(row[(int64_t)I * TB + c2], row[(int64_t)I * TB + c2 + 1]);
      vy = make_double2(row[(int64_t)J * TB + c2], row[(int64_t)J * TB + c2 + 1]);
    }
    Xs[r * SLD + c2] = vx.x;
    Xs[r * SLD + c2 + 1] = vx.y;
    Ys[r * SLD + c2] = vy.x;
    Ys[r * SLD + c2 + 1] = vy.y;
  }
  __syncthreads();

  double acc[4][4][2] = {};
  mma_64x64x64(
      acc, [&](int row, int kk) { return Xs[kk * SLD + row]; },
      [&](int kk, int col) { return Ys[kk * SLD + col]; }, (nb + 3) & ~3);

  const int lane = tid & 31, warp = tid >> 5, g = lane >> 2, t = lane & 3;
  const int wr = (warp >> 1) * 32, wc = (warp & 1) * 32;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = wr + i * 8 + g, c = wc + j * 8 + 2 * t;
      double* dst = M + (int64_t)(I * TB + r) * ldm + (int64_t)J * TB + c;
      if (I != J || c <= r) dst[0] -= acc[i][j][0];
      if (I != J || c + 1 <= r) dst[1] -= acc[i][j][1];
    }
}

std::atomic<uint64_t> g_trailing_smem_set{0};
std::atomic<uint64_t> g_panel_smem_set{0};

}  // namespace

size_t prepare_ws_bytes(int64_t) { return 256; }

int prepare_launch(const void* H, int h_dtype, int k, int64_t ldh, double* M, int64_t ldm,
                   void* ws, cudaStream_t s) {
  long long* info = static_cast<long long*>(ws);
  const int T = (k + TB - 1) / TB;
  const int cblocks = (int)std::min<int64_t>(((int64_t)k * k + 255) / 256, 148 * 16);
  if (h_dtype == GPTQ2D_F32)
    GPTQ2D_LAUNCH(KC_OTHER, s,
                  convert_lower_kernel<float><<<cblocks, 256, 0, s>>>(
                      static_cast<const float*>(H), ldh, k, M, ldm, info));
  else
    GPTQ2D_LAUNCH(KC_OTHER, s,
                  convert_lower_kernel<double><<<cblocks, 256, 0, s>>>(
                      static_cast<const double*>(H), ldh, k, M, ldm, info));
  const int tsmem = 2 * TB * SLD * (int)sizeof(double);
  const int psmem = 2 * TB * PLD * (int)sizeof(double);
  if (ensure_smem(trailing_kernel, tsmem, g_trailing_smem_set) != cudaSuccess ||
      ensure_smem(panel_kernel, psmem, g_panel_smem_set) != cudaSuccess)
    return GPTQ2D_ERR_CUDA;
  for (int K = T - 1; K >= 0; --K) {
    GPTQ2D_LAUNCH(KC_PREP_PANEL, s, panel_kernel<<<K + 1, 256, psmem, s>>>(M, ldm, k, K, info));
    if (K > 0)
      GPTQ2D_LAUNCH(KC_PREP_TRAILING, s,
                    trailing_kernel<<<K * (K + 1) / 2, 128, tsmem, s>>>(M, ldm, k, K, info));
  }
  return cudaGetLastError() == cudaSuccess ? GPTQ2D_OK : GPTQ2D_ERR_CUDA;
}

}  // namespace gptq2d

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
// Step 3 is organised in strips of r block rows (r = 1 for up to 128 block rows,
// 4 beyond): each panel applies the factored rows of its own strip
// and of the strip below it left-looking, and one rank-64r trailing update per
// strip applies the strip to the rows below the next strip, on a second stream
// beside the next strip's panels.  With r = 1 this is the lookahead of one block
// row (panel(K-1) applies row K; rows I <= K-2 get row K from the trailing
// update).  Everything is fp64.  A pivot that is not
// positive and finite stops the factorization and is reported through a pivot
// word in the workspace.
#include <algorithm>

#include "common.cuh"
#include "pipeline.cuh"

namespace gptq2d {

namespace {

constexpr int OLD = TB + 4;  // 68: row stride of shared 64x64 tiles (conflict-free DMMA fragments)
constexpr int PANEL_THREADS = 384;   // 8 factor warps + 4 warps for the block-row lookahead
constexpr int FACTOR_THREADS = 256;

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

// Copies the rows x cols block of M at (row0, col0) into shared memory [r][c]
// with row stride OLD, zero outside.  V16: 16-byte copies, which needs 16-byte
// aligned row starts and an even `cols`; else 8-byte copies.
template <bool V16, int NT>
__device__ __forceinline__ void load_block(double* dst, const double* M, int64_t ldm, int row0,
                                           int col0, int rows, int cols) {
  if (V16) {
    for (int x = threadIdx.x; x < TB * TB / 2; x += NT) {
      const int r = x >> 5, c2 = (x & 31) * 2;
      const bool ok = r < rows && c2 < cols;
      const double* src = ok ? M + (int64_t)(row0 + r) * ldm + col0 + c2 : M;
      cp_async16_zfill(dst + r * OLD + c2, src, ok);
    }
  } else {
    for (int x = threadIdx.x; x < TB * TB; x += NT) {
      const int r = x >> 6, c = x & 63;
      const bool ok = r < rows && c < cols;
      const double* src = ok ? M + (int64_t)(row0 + r) * ldm + col0 + c : M;
      cp_async8_zfill(dst + r * OLD + c, src, ok);
    }
  }
}

// The lower 8x8 blocks (bi >= bj) of Cs -= Xs^T Xs on `nw` warps, one block at a time
// per warp (K = 64 in 16 DMMA steps).  The blocks above the diagonal are not used.
__device__ __forceinline__ void sub_xtx_lower(double* Cs, const double* Xs, int nw) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  for (int x = warp; x < 36; x += nw) {
    int bi = 0;
    while ((bi + 1) * (bi + 2) / 2 <= x) ++bi;
    const int bj = x - bi * (bi + 1) / 2;
    double c0 = 0.0, c1 = 0.0;
#pragma unroll
    for (int kk = 0; kk < TB; kk += 4)
      dmma_m8n8k4(c0, c1, Xs[(kk + t) * OLD + 8 * bi + g], Xs[(kk + t) * OLD + 8 * bj + g]);
    double* c = Cs + (8 * bi + g) * OLD + 8 * bj + 2 * t;
    c[0] -= c0;
    c[1] -= c1;
  }
}

// Cs -= Xs^T Ys (64x64, K = 64) on 4 warps, warp w owning the quadrant (w>>1, w&1);
// `warp` is the warp's index inside the group.
__device__ __forceinline__ void sub_xty_4w(double* Cs, const double* Xs, const double* Ys,
                                           int warp) {
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int wr = (warp >> 1) * 32, wc = (warp & 1) * 32;
  double acc[4][4][2] = {};
#pragma unroll 4
  for (int kk = 0; kk < TB; kk += 4) {
    double a[4], b[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = Xs[(kk + t) * OLD + wr + i * 8 + g];
#pragma unroll
    for (int j = 0; j < 4; ++j) b[j] = Ys[(kk + t) * OLD + wc + j * 8 + g];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) dmma_m8n8k4(acc[i][j][0], acc[i][j][1], a[i], b[j]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      double* c = Cs + (wr + i * 8 + g) * OLD + wc + j * 8 + 2 * t;
      c[0] -= acc[i][j][0];
      c[1] -= acc[i][j][1];
    }
}

__device__ __forceinline__ void factor_group_sync() {
  asm volatile("bar.sync 1, %0;\n" ::"n"(FACTOR_THREADS) : "memory");
}

constexpr int PANEL_SMEM = 6 * TB * OLD * (int)sizeof(double);

// Reverse Cholesky of the 8x8 block D = A[R0..R0+8)^2 of the shared tile A into
// registers: L (lower) = M_D and inv[p] = 1/M_D[p][p].  Every calling thread
// computes the same factor; nothing is shared, so no barrier is needed between
// the factor and its use.  Returns the first bad pivot (elimination order,
// local index) or -1.
__device__ __forceinline__ int factor_diag8_regs(const double* A, int R0, double (&L)[8][8],
                                                 double (&inv)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j <= i; ++j) L[i][j] = A[(R0 + i) * OLD + R0 + j];
  int bad = -1;
#pragma unroll
  for (int p = 7; p >= 0; --p) {
    const double piv = L[p][p];
    const bool ok = piv > 0.0 && isfinite(piv);
    if (!ok && bad < 0) bad = p;
    const double r = ok ? rsqrt(piv) : 0.0;
    const double r2 = r * r;
#pragma unroll
    for (int i = p - 1; i >= 0; --i) {  // row p-1 first: it carries the next pivot
      const double mi = L[p][i] * r2;
#pragma unroll
      for (int j = 0; j <= i; ++j) L[i][j] = fma(-mi, L[p][j], L[i][j]);
    }
#pragma unroll
    for (int j = 0; j <= p; ++j) L[p][j] *= r;
    inv[p] = r;
  }
  return bad;
}

// X <- M_D^{-T} X for the 8 rows R0..R0+8 of column c of the shared tile X,
// with M_D the 8x8 diagonal block of the shared factor F (back substitution).
__device__ __forceinline__ void solve_col8(double* X, const double* F, const double* invd, int R0,
                                           int c) {
  double x[8];
#pragma unroll
  for (int a = 0; a < 8; ++a) x[a] = X[(R0 + a) * OLD + c];
#pragma unroll
  for (int p = 7; p >= 0; --p) {
    x[p] *= invd[R0 + p];
#pragma unroll
    for (int i = 0; i < p; ++i) x[i] = fma(-F[(R0 + p) * OLD + R0 + i], x[p], x[i]);
  }
#pragma unroll
  for (int a = 0; a < 8; ++a) X[(R0 + a) * OLD + c] = x[a];
}

// The same with the factor in registers.
__device__ __forceinline__ void solve_col8_regs(double* X, const double (&L)[8][8],
                                                const double (&inv)[8], int R0, int c) {
  double x[8];
#pragma unroll
  for (int a = 0; a < 8; ++a) x[a] = X[(R0 + a) * OLD + c];
#pragma unroll
  for (int p = 7; p >= 0; --p) {
    x[p] *= inv[p];
#pragma unroll
    for (int i = 0; i < p; ++i) x[i] = fma(-L[p][i], x[p], x[i]);
  }
#pragma unroll
  for (int a = 0; a < 8; ++a) X[(R0 + a) * OLD + c] = x[a];
}

// C[8bi.., 8bj..] -= sum_{a<8} S[R0+a][8bi + r] T[R0+a][8bj + c] for the 8x8 block
// (bi, bj) of shared tile C, on one warp (two m8n8k4 DMMA steps).
__device__ __forceinline__ void rank8_block(double* C, const double* S, const double* T, int R0,
                                            int bi, int bj) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  double c0 = 0.0, c1 = 0.0;
#pragma unroll
  for (int kk = 0; kk < 8; kk += 4)
    dmma_m8n8k4(c0, c1, S[(R0 + kk + t) * OLD + 8 * bi + g], T[(R0 + kk + t) * OLD + 8 * bj + g]);
  double* dst = C + (8 * bi + g) * OLD + 8 * bj + 2 * t;
  dst[0] -= c0;
  dst[1] -= c1;
}

// One launch per block row K.  CTA K factors the diagonal block; CTAs b < K
// factor the same block redundantly (cheaper than a separate launch) and solve
// their block M_Kb = M_KK^{-T} A_Kb.  Those CTAs read A_KK from M, and the order in
// which the CTAs of a launch are dispatched is not fixed, so CTA K must not
// overwrite A_KK in this launch: it leaves M_KK in the block above the diagonal,
// (K-1, K), which is zero and read by no step of the factorization, and CTA K-1 of
// the next launch moves it to (K, K) and zeroes (K-1, K) again.  The last launch
// (K = 0) has one CTA and writes its block in place.  Each CTA first applies, left-
// looking, the updates of the factored block rows j = K+1 .. whi (the window that
// the trailing updates have not applied) to the blocks it reads:
// A_KK -= M_jK^T M_jK and A_Kb -= M_jK^T M_jb, streaming the window's blocks
// through a double buffer; the last row's update of A_Kb runs beside the
// factorization of the diagonal block.
//
// The 64x64 factorization runs in 8-row strips from the bottom: warp 0 factors
// the strip's 8x8 diagonal block (factor_diag8); one thread per column solves
// the strip left of it (solve_col8); the strip's rank-8 update of the leading
// block runs on the DMMA units of all warps (rank8_block).  The solve of A_Kb
// goes the same way.  Rows beyond a ragged edge get a unit diagonal, which
// leaves the factor of the leading part unchanged.
template <bool V16>
__global__ void __launch_bounds__(PANEL_THREADS) panel_kernel(double* __restrict__ M, int64_t ldm,
                                                              int k, int K, int whi,
                                                              long long* info) {
  if (*(volatile long long*)info >= 0) return;
  extern __shared__ __align__(128) double sm[];
  double* Ad = sm;              // A_KK, then M_KK
  double* Ab = Ad + TB * OLD;   // A_Kb, then M_Kb
  // window row j in stage (j - K - 1) & 1: M_jK, then M_jb
  auto mn = [&](int st) { return Ab + (1 + 2 * st) * (TB * OLD); };
  auto mb = [&](int st) { return Ab + (2 + 2 * st) * (TB * OLD); };
  __shared__ double invd[TB];
  __shared__ int bad;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int rb = K * TB, nb = min(TB, k - rb);
  const int b = blockIdx.x;
  if (tid == 0) bad = -1;
  if (b == K && rb + TB < k) {
    // the previous launch's diagonal factor, from (K, K + 1) to (K + 1, K + 1);
    // no CTA of this launch reads either block
    const int r1 = rb + TB, n1 = min(TB, k - r1);
    for (int e = tid; e < n1 * TB; e += PANEL_THREADS) {
      const int r = e >> 6, c = e & 63;
      if (c < n1) {
        double* src = M + (int64_t)(rb + r) * ldm + r1 + c;
        M[(int64_t)(r1 + r) * ldm + r1 + c] = *src;
        *src = 0.0;
      }
    }
  }
  auto load_row = [&](int j, int st) {  // window row j (only the last block row is ragged)
    const int rj = j * TB, nj = min(TB, k - rj);
    load_block<V16, PANEL_THREADS>(mn(st), M, ldm, rj, rb, nj, nb);
    if (b < K) load_block<V16, PANEL_THREADS>(mb(st), M, ldm, rj, b * TB, nj, TB);
  };

  load_block<V16, PANEL_THREADS>(Ad, M, ldm, rb, rb, nb, nb);
  if (b < K) load_block<V16, PANEL_THREADS>(Ab, M, ldm, rb, b * TB, nb, TB);
  if (whi > K) load_row(K + 1, 0);
  cp_async_commit_group();
  // every window row but the last: A_KK on warps 0..7, A_Kb on warps 8..11
#pragma unroll 1
  for (int j = K + 1; j < whi; ++j) {
    const int st = (j - K - 1) & 1;
    load_row(j + 1, st ^ 1);
    cp_async_commit_group();
    cp_async_wait_group<1>();
    __syncthreads();
    if (warp < FACTOR_THREADS / 32) sub_xtx_lower(Ad, mn(st), FACTOR_THREADS / 32);
    else if (b < K) sub_xty_4w(Ab, mn(st), mb(st), warp - FACTOR_THREADS / 32);
    __syncthreads();
  }
  cp_async_wait_group<0>();
  __syncthreads();
  const int st_last = (whi - K - 1) & 1;
  if (whi > K) sub_xtx_lower(Ad, mn(st_last), PANEL_THREADS / 32);  // the factor needs it first
  // unit diagonal past a ragged edge (only the last block row is ragged, and it
  // has no window, so no other thread writes these elements)
  if (tid < TB && tid >= nb) Ad[tid * OLD + tid] = 1.0;
  __syncthreads();

  if (warp >= FACTOR_THREADS / 32) {
    // warps 8..11: the last window row's A_Kb -= M_jK^T M_jb, needed only by the
    // solve below, while warps 0..7 factor the diagonal block
    if (whi > K && b < K) sub_xty_4w(Ab, mn(st_last), mb(st_last), warp - FACTOR_THREADS / 32);
  } else {
  // factor A_KK in place, strips s = 7..0.  Threads <= 8s factor strip s's 8x8
  // diagonal block in registers; threads < 8s then solve one column of the strip
  // each, and thread 8s stores the block.
  auto factor_strip = [&](int s) {
    const int R0 = 8 * s;
    double L[8][8], inv[8];
    const int bp = factor_diag8_regs(Ad, R0, L, inv);
    if (tid < R0) {
      solve_col8_regs(Ad, L, inv, R0, tid);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        invd[R0 + i] = inv[i];
#pragma unroll
        for (int j = 0; j < 8; ++j) Ad[(R0 + i) * OLD + R0 + j] = j <= i ? L[i][j] : 0.0;
      }
      if (bp >= 0 && bad < 0) bad = rb + R0 + bp;
    }
  };
  if (tid <= TB - 8) factor_strip(TB / 8 - 1);
  factor_group_sync();
#pragma unroll 1
  for (int s = TB / 8 - 1; s >= 1; --s) {
    // strip s is done.  First its update of the next strip's row of blocks
    // (s-1, 0..s-1), one block per warp ...
    if (warp < s) rank8_block(Ad, Ad, Ad, 8 * s, s - 1, warp);
    factor_group_sync();
    // ... then strip s-1 is factored on warps 0..1 while warps 2..7 apply strip s's
    // update to the rows above it: A[i][j] -= sum_a M[8s+a][i] M[8s+a][j], lower
    // 8x8 blocks (bi >= bj) with bi < s-1
    if (tid <= 8 * (s - 1)) {
      factor_strip(s - 1);
    } else if (warp >= 2) {
      const int nblk = (s - 1) * s / 2;
      for (int x = warp - 2; x < nblk; x += FACTOR_THREADS / 32 - 2) {
        int bi = 0;
        while ((bi + 1) * (bi + 2) / 2 <= x) ++bi;
        rank8_block(Ad, Ad, Ad, 8 * s, bi, x - bi * (bi + 1) / 2);
      }
    }
    factor_group_sync();
  }
  }
  __syncthreads();
  if (bad >= 0) {  // uniform: read after the barrier
    if (tid == 0) *info = bad;
    return;
  }
  // zero the strict upper part of the 8x8 blocks above the diagonal blocks
  for (int e = tid; e < TB * TB; e += PANEL_THREADS) {
    const int r = e >> 6, c = e & 63;
    if (c > r) Ad[r * OLD + c] = 0.0;
  }
  __syncthreads();
  if (b == K) {  // in place for K = 0, else parked in (K - 1, K)
    const int r0 = K > 0 ? rb - TB : rb;
    for (int e = tid; e < nb * TB; e += PANEL_THREADS) {
      const int r = e >> 6, c = e & 63;
      if (c < nb) M[(int64_t)(r0 + r) * ldm + rb + c] = Ad[r * OLD + c];
    }
    return;
  }

  // X <- M_KK^{-T} X in strips from the bottom
#pragma unroll 1
  for (int s = TB / 8 - 1; s >= 0; --s) {
    const int R0 = 8 * s;
    if (tid < TB) solve_col8(Ab, Ad, invd, R0, tid);
    __syncthreads();
    // X[i][c] -= sum_a M[R0+a][i] X[R0+a][c] for rows i < R0
    for (int x = warp; x < s * 8; x += PANEL_THREADS / 32) rank8_block(Ab, Ad, Ab, R0, x >> 3, x & 7);
    __syncthreads();
  }
  for (int e = tid; e < nb * TB; e += PANEL_THREADS) {
    const int r = e >> 6, c = e & 63;
    M[(int64_t)(rb + r) * ldm + (int64_t)b * TB + c] = Ab[r * OLD + c];
  }
}

constexpr int MAX_STRIP = 4;  // block rows per strip (rank of a trailing update: 64 x strip)

struct TrailPlan {
  int k0, nk;    // the strip: factored block rows k0 .. k0 + nk - 1
  int rows;      // block rows I = 0 .. rows - 1 are updated (J <= I)
  int per_cta;   // block pairs per CTA
};

constexpr int TR_STAGE = 8 * 40;  // per warp: one 8x32 strip of the product (row stride 40)
// Shared memory of a trailing CTA of nw warps for a strip of nk rows: the strip's
// blocks of column I, two stream buffers, one staging strip per warp.
constexpr int tr_smem(int nk, int nw) { return ((nk + 2) * TB * OLD + nw * TR_STAGE) * (int)sizeof(double); }

// A_IJ -= sum_{q < nk} M_{k0+q,I}^T M_{k0+q,J} for J <= I: the rank-64 nk update of
// one strip.  The block pairs (I, J) are numbered row by row and every CTA takes an
// equal run of them (no CTA waits for a longer one at the end of the launch).  A
// CTA keeps the strip's blocks of its current column I in shared memory (reloaded
// when its run enters the next row) and streams the blocks M_{k0+q,J} through a
// double buffer (q fastest); the sum over the strip stays in registers, and goes
// into A_IJ by reductions in L2 (no read of the block), one whole 256-byte row at a
// time through a shared strip.  NW warps (4: two CTAs per SM, for strips of one row;
// 8: one CTA per SM with room for four rows), warp w owning rows (64 / (NW/2)) (w>>1)..
// and columns 32 (w&1).. of the 64x64 block.  Only the lower part of A_II is touched.
template <bool V16, int NW>
__global__ void __launch_bounds__(NW * 32, NW == 4 ? 2 : 1) trailing_kernel(double* __restrict__ M,
                                                                 int64_t ldm, int k,
                                                                 const long long* info,
                                                                 TrailPlan pl) {
  constexpr int NT = NW * 32;
  constexpr int RF = 64 / (NW / 2) / 8;  // 8-row fragments per warp
  if (*(volatile const long long*)info >= 0) return;
  extern __shared__ __align__(128) double sm[];
  double* const Xs = sm;                        // Xs[q][r][i] = M[64 (k0+q) + r][64 I + i]
  double* const Y0 = sm + pl.nk * TB * OLD;     // two stream buffers
  double* const stage = Y0 + 2 * TB * OLD;
  auto ybuf = [&](int bsel) { return Y0 + bsel * (TB * OLD); };
  const long long total = (long long)pl.rows * (pl.rows + 1) / 2;
  const long long p0 = (long long)blockIdx.x * pl.per_cta;
  const long long p1 = min(p0 + pl.per_cta, total);
  if (p0 >= p1) return;
  const int nk = pl.nk;
  auto rows_of = [&](int q) { return min(TB, k - (pl.k0 + q) * TB); };  // only the last block row is ragged
  // (I, J) of the first pair: row I holds pairs I (I + 1) / 2 .. I (I + 1) / 2 + I
  int I = (int)((sqrt(8.0 * (double)p0 + 1.0) - 1.0) * 0.5);
  while ((long long)(I + 1) * (I + 2) / 2 <= p0) ++I;
  while ((long long)I * (I + 1) / 2 > p0) --I;
  int J = (int)(p0 - (long long)I * (I + 1) / 2);
  auto load_x = [&](int col) {
    for (int q = 0; q < nk; ++q)
      load_block<V16, NT>(Xs + q * (TB * OLD), M, ldm, (pl.k0 + q) * TB, col * TB, rows_of(q), TB);
  };
  load_x(I);
  load_block<V16, NT>(ybuf(0), M, ldm, pl.k0 * TB, J * TB, rows_of(0), TB);
  cp_async_commit_group();

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5, g8 = lane >> 2, t4 = lane & 3;
  const int wr = (warp >> 1) * (8 * RF), wc = (warp & 1) * 32;
  const long long nsteps = (p1 - p0) * nk;
  double acc[RF][4][2] = {};
  int Jn = J, In = I;  // the pair of the next step's block
  for (long long step = 0; step < nsteps; ++step) {
    const int q = (int)(step % nk);
    if (q == 0 && step > 0) {
      // next pair; entering a new row reloads the strip's blocks of column I (every
      // warp finished with the old ones at the end of the previous step)
      const int Iprev = I;
      I = In;
      J = Jn;
      if (I != Iprev) {
        load_x(I);
        cp_async_commit_group();
      }
    }
    const int bsel = (int)(step & 1);
    if (step + 1 < nsteps) {
      const int q1 = (int)((step + 1) % nk);
      if (q1 == 0) {  // the following pair
        Jn = J + 1;
        In = I;
        if (Jn > In) {
          ++In;
          Jn = 0;
        }
      }
      load_block<V16, NT>(ybuf(bsel ^ 1), M, ldm, (pl.k0 + q1) * TB, (q1 == 0 ? Jn : J) * TB, rows_of(q1), TB);
      cp_async_commit_group();
      cp_async_wait_group<1>();
    } else {
      cp_async_wait_group<0>();
    }
    __syncthreads();
    const double* Xq = Xs + q * (TB * OLD);
    const double* Ys = ybuf(bsel);
#pragma unroll 4
    for (int kk = 0; kk < TB; kk += 4) {
      double a[RF], bv[4];
#pragma unroll
      for (int i = 0; i < RF; ++i) a[i] = Xq[(kk + t4) * OLD + wr + i * 8 + g8];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Ys[(kk + t4) * OLD + wc + j * 8 + g8];
#pragma unroll
      for (int i = 0; i < RF; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) dmma_m8n8k4(acc[i][j][0], acc[i][j][1], a[i], bv[j]);
    }
    if (q == nk - 1) {
      // A_IJ -= the strip's product by reductions in L2 (each element of the block
      // gets exactly one contribution per launch): whole 256-byte rows through a
      // shared strip
      double* st = stage + warp * TR_STAGE;
      double* Cw = M + (int64_t)(I * TB + wr) * ldm + (int64_t)J * TB + wc;
#pragma unroll
      for (int i = 0; i < RF; ++i) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          *reinterpret_cast<double2*>(st + g8 * 40 + j * 8 + 2 * t4) =
              make_double2(-acc[i][j][0], -acc[i][j][1]);
          acc[i][j][0] = acc[i][j][1] = 0.0;
        }
        __syncwarp();
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const int row = wr + i * 8 + r, col = wc + lane;
          if (I != J || col <= row) red_add(Cw + (int64_t)(i * 8 + r) * ldm + lane, st[r * 40 + lane]);
        }
        __syncwarp();
      }
    }
    __syncthreads();
  }
}

std::atomic<uint64_t> g_trailing_smem_set[4];
std::atomic<uint64_t> g_panel_smem_set[2];


// One factor's enqueue state: panels on `ps`, trailing updates on `us`.
struct FactorJob {
  const void* H;
  int h_dtype, k, T;
  int64_t ldh, ldm;
  double* M;
  long long* info;
  bool v16;
  cudaStream_t ps, us;
  cudaEvent_t ready;        // H is in place once this has completed (may be null)
  cudaEvent_t* panel_done;  // [RING]
  cudaEvent_t* rest_done;   // [RING]
};

int enqueue_convert(const FactorJob& f, int sms) {
  const int cblocks = (int)std::min<int64_t>(((int64_t)f.k * f.k + 255) / 256, (int64_t)sms * 16);
  if (f.h_dtype == GPTQ2D_F32)
    GPTQ2D_LAUNCH(KC_OTHER, f.ps,
                  convert_lower_kernel<float><<<cblocks, 256, 0, f.ps>>>(
                      static_cast<const float*>(f.H), f.ldh, f.k, f.M, f.ldm, f.info));
  else
    GPTQ2D_LAUNCH(KC_OTHER, f.ps,
                  convert_lower_kernel<double><<<cblocks, 256, 0, f.ps>>>(
                      static_cast<const double*>(f.H), f.ldh, f.k, f.M, f.ldm, f.info));
  return cudaGetLastError() == cudaSuccess ? GPTQ2D_OK : GPTQ2D_ERR_CUDA;
}

// Block rows per strip: one row (a lookahead of one row, as in the classic
// right-looking scheme) up to 128 block rows, where the panels set the pace; four
// beyond, where the trailing updates dominate: each pass over the trailing matrix
// then carries a rank-256 update, with a quarter of the launches (measured on a
// B200: 16384^2 in 82 ms instead of 103, 28672^2 in 418 ms instead of 502; two
// equal factors at once gain nothing, the GPU being full either way).
inline int strip_rows(int T) { return T <= 128 ? 1 : MAX_STRIP; }

// Step K of one factor.  The block rows are grouped into strips of r rows from the
// bottom (strip s: rows lo_s .. hi_s, hi_s = T-1 - s r).  panel(K) applies the rows
// K+1 .. hi_{s-1} (its own strip and the one below it) left-looking; the strip's
// trailing update, launched after its last panel, applies it to the rows below the
// next strip (I < lo_s - r).  So every row K sees each factored row exactly once,
// and the first panel of strip s waits only for the trailing update of strip s-2,
// which leaves strip s-1's trailing update running beside strip s's panels.  The
// trailing updates of one factor run in order on one stream (a fixed order of the
// reductions into each block: deterministic).
int enqueue_step(const FactorJob& f, int K, int sms) {
  const int r = strip_rows(f.T);
  const int sidx = (f.T - 1 - K) / r;
  const int hi_s = f.T - 1 - sidx * r, lo_s = std::max(0, hi_s - r + 1);
  const int whi = std::min(f.T - 1, hi_s + r);
  bool ok = true;
  if (K == hi_s && sidx >= 2)
    ok = cudaStreamWaitEvent(f.ps, f.rest_done[(sidx - 2) % RING], 0) == cudaSuccess;
  if (f.v16)
    GPTQ2D_LAUNCH(KC_PREP_PANEL, f.ps,
                  panel_kernel<true><<<K + 1, PANEL_THREADS, PANEL_SMEM, f.ps>>>(f.M, f.ldm, f.k,
                                                                                   K, whi, f.info));
  else
    GPTQ2D_LAUNCH(KC_PREP_PANEL, f.ps,
                  panel_kernel<false><<<K + 1, PANEL_THREADS, PANEL_SMEM, f.ps>>>(f.M, f.ldm, f.k,
                                                                                    K, whi, f.info));
  const int rows = lo_s - r;  // block rows I = 0 .. lo_s - r - 1
  if (K != lo_s || rows <= 0)
    return ok && cudaGetLastError() == cudaSuccess ? GPTQ2D_OK : GPTQ2D_ERR_CUDA;
  ok = ok && cudaEventRecord(f.panel_done[sidx % RING], f.ps) == cudaSuccess &&
       cudaStreamWaitEvent(f.us, f.panel_done[sidx % RING], 0) == cudaSuccess;
  const long long total = (long long)rows * (rows + 1) / 2;
  const int nk = hi_s - lo_s + 1;
  const bool wide = nk > 1;  // 8 warps, one CTA per SM; else 4 warps, two per SM
  const int smem = tr_smem(nk, wide ? 8 : 4);
  const int target = (wide ? 1 : 2) * sms;  // one wave of CTAs
  TrailPlan pl;
  pl.k0 = lo_s;
  pl.nk = nk;
  pl.rows = rows;
  pl.per_cta = (int)std::max<long long>(1, (total + target - 1) / target);
  const int ctas = (int)((total + pl.per_cta - 1) / pl.per_cta);
  auto kern = f.v16 ? (wide ? trailing_kernel<true, 8> : trailing_kernel<true, 4>)
                    : (wide ? trailing_kernel<false, 8> : trailing_kernel<false, 4>);
  GPTQ2D_LAUNCH(KC_PREP_TRAILING, f.us,
                kern<<<ctas, wide ? 256 : 128, smem, f.us>>>(f.M, f.ldm, f.k, f.info, pl));
  ok = ok && cudaEventRecord(f.rest_done[sidx % RING], f.us) == cudaSuccess;
  return ok && cudaGetLastError() == cudaSuccess ? GPTQ2D_OK : GPTQ2D_ERR_CUDA;
}

int ensure_prepare_smem() {
  if (ensure_smem(trailing_kernel<true, 8>, tr_smem(MAX_STRIP, 8), g_trailing_smem_set[0]) != cudaSuccess ||
      ensure_smem(trailing_kernel<false, 8>, tr_smem(MAX_STRIP, 8), g_trailing_smem_set[1]) != cudaSuccess ||
      ensure_smem(trailing_kernel<true, 4>, tr_smem(1, 4), g_trailing_smem_set[2]) != cudaSuccess ||
      ensure_smem(trailing_kernel<false, 4>, tr_smem(1, 4), g_trailing_smem_set[3]) != cudaSuccess ||
      ensure_smem(panel_kernel<true>, PANEL_SMEM, g_panel_smem_set[0]) != cudaSuccess ||
      ensure_smem(panel_kernel<false>, PANEL_SMEM, g_panel_smem_set[1]) != cudaSuccess)
    return GPTQ2D_ERR_CUDA;
  return GPTQ2D_OK;
}

FactorJob make_job(const void* H, int h_dtype, int k, int64_t ldh, double* M, int64_t ldm,
                   void* ws, cudaStream_t ps, cudaStream_t us, cudaEvent_t* pd, cudaEvent_t* rd) {
  FactorJob f;
  f.H = H;
  f.h_dtype = h_dtype;
  f.k = k;
  f.T = (k + TB - 1) / TB;
  f.ldh = ldh;
  f.ldm = ldm;
  f.M = M;
  f.info = static_cast<long long*>(ws);
  // 16-byte copies need aligned row starts and even block widths
  f.v16 = (ldm % 2 == 0) && (k % 2 == 0) && ((reinterpret_cast<uintptr_t>(M) & 15u) == 0);
  f.ps = ps;
  f.us = us;
  f.panel_done = pd;
  f.rest_done = rd;
  f.ready = nullptr;
  return f;
}

// Enqueues the factorizations of `jobs` (1 or 2), forked from and joined back to s.
// alt: the jobs run on hi2/lo2 and hi3/lo3 (join events to match).
int enqueue_factors(FactorJob* jobs, int nj, cudaStream_t s, DevStreams* ds, bool alt = false) {
  int rc = ensure_prepare_smem();
  if (rc != GPTQ2D_OK) return rc;
  bool ok = cudaEventRecord(ds->fork, s) == cudaSuccess;
  for (int j = 0; j < nj && ok; ++j) {
    ok = cudaStreamWaitEvent(jobs[j].ps, ds->fork, 0) == cudaSuccess &&
         cudaStreamWaitEvent(jobs[j].us, ds->fork, 0) == cudaSuccess;
    if (ok && jobs[j].ready)
      ok = cudaStreamWaitEvent(jobs[j].ps, jobs[j].ready, 0) == cudaSuccess;
  }
  if (!ok) return GPTQ2D_ERR_CUDA;
  for (int j = 0; j < nj && rc == GPTQ2D_OK; ++j) rc = enqueue_convert(jobs[j], ds->sms);
  int steps = 0;
  for (int j = 0; j < nj; ++j) steps = std::max(steps, jobs[j].T);
  for (int st = 0; st < steps && rc == GPTQ2D_OK; ++st)
    for (int j = 0; j < nj && rc == GPTQ2D_OK; ++j)
      if (st < jobs[j].T) rc = enqueue_step(jobs[j], jobs[j].T - 1 - st, ds->sms);
  cudaEvent_t joins[4] = {alt ? ds->join_hi3 : ds->join_hi, alt ? ds->join_lo3 : ds->join_lo,
                          ds->join_hi2, ds->join_lo2};
  for (int j = 0; j < nj && ok; ++j)
    ok = cudaEventRecord(joins[2 * j], jobs[j].ps) == cudaSuccess &&
         cudaEventRecord(joins[2 * j + 1], jobs[j].us) == cudaSuccess &&
         cudaStreamWaitEvent(s, joins[2 * j], 0) == cudaSuccess &&
         cudaStreamWaitEvent(s, joins[2 * j + 1], 0) == cudaSuccess;
  if (rc != GPTQ2D_OK) return rc;
  return ok ? GPTQ2D_OK : GPTQ2D_ERR_CUDA;
}

}  // namespace

size_t prepare_ws_bytes(int64_t) { return 256; }

int prepare_launch(const void* H, int h_dtype, int k, int64_t ldh, double* M, int64_t ldm,
                   void* ws, cudaStream_t s) {
  DevStreams* ds = nullptr;
  int rc = dev_streams(&ds);
  if (rc != GPTQ2D_OK) return rc;
  std::lock_guard<std::recursive_mutex> lk(ds->mu);
  FactorJob f = make_job(H, h_dtype, k, ldh, M, ldm, ws, ds->hi, ds->lo, ds->panel_done[0],
                         ds->rest_done[0]);
  return enqueue_factors(&f, 1, s, ds);
}

int prepare_pair_launch(const void* H_L, int64_t m, int64_t ldhl, const void* H_R, int64_t n,
                        int64_t ldhr, int h_dtype, double* M_L, int64_t ldml, double* M_R,
                        int64_t ldmr, void* ws_l, void* ws_r, cudaStream_t s,
                        cudaEvent_t ready_l, cudaEvent_t ready_r, bool alt) {
  DevStreams* ds = nullptr;
  int rc = dev_streams(&ds);
  if (rc != GPTQ2D_OK) return rc;
  std::lock_guard<std::recursive_mutex> lk(ds->mu);
  // stream pairs: (hi, lo) then (hi2, lo2); alt: (hi3, lo3) then (hi2, lo2)
  cudaStream_t ph[2] = {alt ? ds->hi3 : ds->hi, ds->hi2};
  cudaStream_t pl[2] = {alt ? ds->lo3 : ds->lo, ds->lo2};
  FactorJob jobs[2];
  int nj = 0;
  if (m > 0) {
    jobs[nj] = make_job(H_L, h_dtype, (int)m, ldhl, M_L, ldml, ws_l, ph[0], pl[0],
                        ds->panel_done[0], ds->rest_done[0]);
    jobs[nj++].ready = ready_l;
  }
  if (n > 0) {
    jobs[nj] = make_job(H_R, h_dtype, (int)n, ldhr, M_R, ldmr, ws_r, ph[nj], pl[nj],
                        ds->panel_done[nj], ds->rest_done[nj]);
    jobs[nj++].ready = ready_r;
  }
  if (nj == 0) return GPTQ2D_OK;
  return enqueue_factors(jobs, nj, s, ds, alt);
}

}  // namespace gptq2d

// GPTQ-2D rounding on sm_100a.
//
// What is computed (arxivlens "GPTQ-2D: Cubic-Time Two-Sided Adaptive
// Rounding", Abstract and Analysis > Results / Methodology; mind-verse.de
// "Neue Ansätze ... durch GPTQ-2D", "Die algorithmische Neuerung"):
// with lower factors M_L, M_R (M^T M = H) and their row-normalised forms
// Lh = diag(M_L)^-1 M_L, Rh = diag(M_R)^-1 M_R (unit diagonal), entry (i,j)
// rounds
//     y_ij = W_ij + sum_{i'<=i, j'<=j, (i',j') != (i,j)} Lh[i,i'] dW[i',j'] Rh[j,j']
//     q_ij = clamp(rint(y_ij / s_i)),   dW_ij = W_ij - s_i q_ij,
// the row (i,j) of the Kronecker triangular factor applied to the errors made
// so far.  y_ij depends only on the dominated quadrant, so all entries of one
// anti-diagonal are independent.
//
// Data layout in HBM (workspace, row-major, padded to whole 64 x 64 tiles):
//   Lh (mp x mp), Rh (np x np)  normalised factors, strictly lower (diagonal
//                               stored as 0), zero padding
//   P  (mp x np)  right feedback  P[i,j] = sum_{done j'<=j} dW[i,j'] Rh[j,j']
//   E  (mp x np)  down feedback   E[i,j] = sum_{i' in tile rows <= I-2} Lh[i,i'] P[i',j]
//   Dl (mp x np)  errors dW of finished tiles
//
// Schedule: 64 x 64 tiles, one tile wavefront D (tile row + tile column = D)
// at a time, on two internal streams forked from the caller's stream:
//   high priority  sweep_kernel(D): one CTA per tile.  It first pulls the
//                  contributions of its left and upper neighbours (wavefront
//                  D-1) with two FP64 tensor-core products run side by side,
//                  then sweeps the tile as 8 x 8 sub-tiles: the sub-tiles of one
//                  sub-wavefront go to one warp each, which walks the 15 local
//                  anti-diagonals warp-synchronously (row and column pushes by
//                  shuffles); between sub-wavefronts the finished sub-tiles push
//                  to their neighbours with 8x8x8 DMMA products, and the pushes
//                  two or more sub-tiles away run on helper warps during the
//                  next sub-wavefront.
//   low priority   far_kernel(D): the band products that carry the tiles of
//                  wavefront D to tiles two or more tiles away (to the right:
//                  P += dW Rh^T; below: E += Lh P), 64x64x64 DMMA tasks
//                  claimed one at a time per group.  One launch runs beside
//                  sweep_kernel(D+1) on the SMs that sweep leaves free; when the
//                  work outlasts that sweep a second launch on the high-priority
//                  stream, after sweep_kernel(D+1), takes the rest on the SMs the
//                  sweep frees.
// sweep_kernel(D) waits for far_kernel(D-2) only.  Exactness: every
// contribution to a tile comes from earlier wavefronts (far: through P and E,
// near: pulled by the sweep) or from the tile itself (the sweep).
#include <algorithm>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "pipeline.cuh"

namespace gptq2d {

namespace {

constexpr int SLD = TB + 4;  // 68 doubles: [row][k] tiles (conflict-free DMMA fragments)
constexpr int SWEEP_THREADS = 512;

// The right factor given per mode (k-way rounding): R^ = Lh_0 (x) ... (x) Lh_{nf-1},
// Lh_f = diag(M_f)^-1 M_f, generated where it is used.  A column j has the mixed-
// radix digits d_f(j) = (j / stride_f) % dim_f (last factor fastest).  The last
// nf - nout factors form the inner group of size m_in (dividing the tile width), so
// a tile holds a = TB / m_in consecutive outer indices u = j / m_in, and a block of
// R^ between tiles is (a x a outer block of Ah) (x) Lin, with Ah the outer factors'
// product and Lin the inner one's.
constexpr int KMAXF = 8;
constexpr int KMAXA = 8;  // a = TB / m_in with m_in >= 8
struct KronDesc {
  int nf, nout;
  int m_in, a;
  int lg;                   // log2 m_in (m_in is a power of two: it divides 64)
  int U;                    // outer extent n / m_in
  int dim[KMAXF];
  int ustride[KMAXF];       // stride_f / m_in for the outer factors
  int vstride[KMAXF];       // stride_f for the inner factors
  const double* M[KMAXF];   // the factors as given (lower, fp64)
  int64_t ld[KMAXF];
  const double* lin;        // Lin, m_in x m_in, unit diagonal, zero above (workspace)
};

struct QArgs {
  const void* W;
  int64_t ldw;
  int m, n;
  const double* ML;
  int64_t ldl;
  const double* MR;
  int64_t ldr;
  const float* scales;
  int64_t lds;           // row stride of scales / zero in groups
  int64_t group;         // columns per scale group; 0: one scale per row
  const uint8_t* zero;   // integer zero points (asymmetric grid), or null
  double lo, hi;         // symmetric grid range (infinite without clamp)
  double top;            // 2^bits - 1: top of the asymmetric code range
  double code_off;       // added to q + z for the stored code (offset binary when packed)
  int clamp;
  int packed;            // two 4-bit codes per byte
  uint8_t* Q;
  int64_t ldq;           // bytes
  int* err;       // nonzero: a bounded wait in a kernel timed out
  double* Lh;     // mp x mp
  double* Rh;     // np x np
  double* P;      // mp x np
  double* E;      // mp x np
  double* Dl;     // mp x np
  int64_t mp, np;
  double* dL;     // M_L[i,i] (mp)
  double* dR;     // M_R[j,j] (np)
  TileStat* part; // Tm x Tn
  int Tm, Tn;
  int kron;       // 1: the right factor is kd (Rh is not formed)
  KronDesc kd;
};

// One normalised factor entry Lh_f[r][c]: 1 on the diagonal, M_f[r][c] / M_f[r][r]
// below it, 0 above.
__device__ __forceinline__ double kron_factor_entry(const KronDesc& k, int f, int r, int c) {
  if (r == c) return 1.0;
  if (c > r) return 0.0;
  const double* Mf = k.M[f] + (int64_t)r * k.ld[f];
  return Mf[c] / Mf[r];
}
// Ah[u][u'] (outer indices u, u' < U).
__device__ __forceinline__ double kron_outer(const KronDesc& k, int u, int up) {
  double v = 1.0;
  for (int f = 0; f < k.nout && v != 0.0; ++f) {
    const int r = (u / k.ustride[f]) % k.dim[f], c = (up / k.ustride[f]) % k.dim[f];
    v *= kron_factor_entry(k, f, r, c);
  }
  return v;
}

// ---------------------------------------------------------------------------
// small PTX helpers
// ---------------------------------------------------------------------------
// The bounded wait above on an mbarrier that nothing completes: the check behind
// gptq2d_check_wait_timeout.  *status = GPTQ2D_ERR_TIMEOUT once the wait has
// given up (GPTQ2D_OK would mean the barrier completed).
__global__ void wait_timeout_kernel(unsigned long long limit_ns, int* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) mbar_init(&bar, 1);
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  __syncthreads();
  const bool done = mbar_wait(&bar, 0, limit_ns);
  __syncwarp();
  if (threadIdx.x == 0) *status = done ? GPTQ2D_OK : GPTQ2D_ERR_TIMEOUT;
}

// ---------------------------------------------------------------------------
// set-up: normalised, tile-padded factors and their diagonals
// ---------------------------------------------------------------------------
// Normalised factors Lh = diag(M_L)^-1 M_L and Rh = diag(M_R)^-1 M_R, strictly
// lower (the unit diagonal is implied), and the diagonals dL, dR.  Only the blocks
// on or below the 64-block diagonal are written: no kernel reads the others.  One
// CTA per row i (rows of Lh first, then rows of Rh); the threads take the columns
// k < 64 (i / 64 + 1), two at a time.
__global__ void __launch_bounds__(256) normalize_kernel(QArgs a) {
  const bool left = blockIdx.x < a.mp;
  const int i = left ? blockIdx.x : blockIdx.x - (int)a.mp;
  const int64_t ldo = left ? a.mp : a.np;
  const int dim = left ? a.m : a.n;
  const double* Mrow = (left ? a.ML + (int64_t)i * a.ldl : a.MR + (int64_t)i * a.ldr);
  double* out = (left ? a.Lh : a.Rh) + (int64_t)i * ldo;
  const double d = i < dim ? Mrow[i] : 0.0;
  if (threadIdx.x == 0) (left ? a.dL : a.dR)[i] = d;
  const int kend = (i / TB + 1) * TB;  // end of the diagonal block
  for (int k = 2 * threadIdx.x; k < kend; k += 2 * blockDim.x) {
    double2 v;
    v.x = (i < dim && k < i) ? Mrow[k] / d : 0.0;
    v.y = (i < dim && k + 1 < i) ? Mrow[k + 1] / d : 0.0;
    *reinterpret_cast<double2*>(out + k) = v;
  }
}

// The per-mode right factor's set-up: Lin (the inner group's normalised factor,
// m_in x m_in, into the workspace) and dR[j] = M_R[j][j] = prod_f M_f[d_f(j)][d_f(j)]
// (zero on the padding columns).  Grid-stride over m_in^2 + np entries.
__global__ void __launch_bounds__(256) kron_setup_kernel(QArgs a) {
  const KronDesc& k = a.kd;
  const int64_t nlin = (int64_t)k.m_in * k.m_in, total = nlin + a.np;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    if (e < nlin) {
      const int v = (int)(e / k.m_in), vp = (int)(e % k.m_in);
      double x = 1.0;
      for (int f = k.nout; f < k.nf && x != 0.0; ++f)
        x *= kron_factor_entry(k, f, (v / k.vstride[f]) % k.dim[f], (vp / k.vstride[f]) % k.dim[f]);
      const_cast<double*>(k.lin)[e] = x;
    } else {
      const int64_t j = e - nlin;
      double d = 0.0;
      if (j < a.n) {
        d = 1.0;
        const int u = (int)(j / k.m_in), v = (int)(j % k.m_in);
        for (int f = 0; f < k.nf; ++f) {
          const int r = f < k.nout ? (u / k.ustride[f]) % k.dim[f] : (v / k.vstride[f]) % k.dim[f];
          d *= k.M[f][(int64_t)r * k.ld[f] + r];
        }
      }
      a.dR[j] = d;
    }
  }
}

// ---------------------------------------------------------------------------
// the tile sweep
// ---------------------------------------------------------------------------
template <typename TW>
struct WStore { using T = float; };          // f32 and bf16 are exact in f32
template <>
struct WStore<__nv_bfloat16> { using T = __nv_bfloat16; };
template <>
struct WStore<double> { using T = double; };

// Shared memory of the sweep: six 64 x SLD fp64 tiles: P, V, W-then-dW, the
// diagonal blocks of Rh and Lh, and t = y / s of every rounded entry.
template <typename TW>
constexpr int sweep_smem_bytes() {
  return 6 * TB * SLD * (int)sizeof(double);
}

constexpr int SUB = 8;             // sub-tile edge
constexpr int NSUB = TB / SUB;     // sub-tiles per tile edge

// One CTA per tile (I, J) with I = I0 + blockIdx.x, J = D - I.
//
// The tile is swept as 8 x 8 sub-tiles, one sub-tile wavefront (p + q = w) at a
// time.  A sub-tile's 15 local anti-diagonals run in one warp, warp-
// synchronously: lane (a = lane/4, cq = lane%4) holds row a, columns cq and
// cq + 4 of P (right feedback), V (down feedback) and W / dW in registers; the
// rank-one updates of each rounded entry inside the sub-tile go through warp
// shuffles (dW along its row, P_final down its column).  After each sub-tile
// wavefront, every finished sub-tile (p, q) pushes its errors to the sub-tiles
// right of it (P[p][q'] += dW[p][q] Rh[q'][q]^T) and its final P below it
// (V[p'][q] += Lh[p'][p] P[p][q]) as 8x8x8 FP64 tensor-core products, one warp
// per target sub-tile.
// KRON: the right factor is given per mode (a.kron); a separate instantiation, so
// that the dense route's code is not touched by it.
template <typename TW, bool KRON>
__global__ void __launch_bounds__(SWEEP_THREADS, 1) sweep_kernel(QArgs a, int D, int I0) {
  extern __shared__ __align__(128) double sm[];
  double* Pt = sm;                 // P of the tile
  double* Vt = Pt + TB * SLD;      // V of the tile
  double* Dt = Vt + TB * SLD;      // W, overwritten by dW entry by entry
  double* Rt = Dt + TB * SLD;      // Rt[c'][c] = Rh[c0+c'][c0+c] (strictly lower)
  double* Lt = Rt + TB * SLD;      // Lt[a'][a] = Lh[r0+a'][r0+a]
  double* Tq = Lt + TB * SLD;      // t = y / s of each rounded entry (Q and statistics come from it)

  const int I = I0 + blockIdx.x, J = D - I;
  const int r0 = I * TB, c0 = J * TB;
  const int rows = min(TB, a.m - r0), cols = min(TB, a.n - c0);
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5, g = lane >> 2, t4 = lane & 3;
  const int64_t np = a.np;
  const int64_t ts = (int64_t)r0 * np + c0;  // tile origin in the workspace matrices

  // ---- near-neighbour feedback, pulled from the tiles finished one wavefront ago:
  //   right: P += dW[I,J-1] Rh[J,J-1]^T      (warps 0..7)
  //   down:  V += Lh[I,I-1] P_final[I-1,J]   (warps 8..15)
  // All operand tiles and the tile's own P and E arrive in two async batches; the
  // two products run side by side on the DMMA units.
  //   With the right factor given per mode, P holds the far-field sum before the
  //   inner factor (see kron_push_kernel) and the right product is
  //   P = (P + dW[I,J-1] mixed by the outer block Ah[J,J-1]) (I_a (x) Lin)^T.
  const bool has_r = J > 0, has_d = I > 0;
  constexpr bool kron = KRON;
  __shared__ double KN[KRON ? KMAXA : 1][KMAXA], KA[KRON ? KMAXA : 1][KMAXA];  // Ah[J,J-1], Ah[J,J]
  if constexpr (KRON) {
    if (tid < 2 * KMAXA * KMAXA) {
      const KronDesc& k = a.kd;
      const bool diag = tid >= KMAXA * KMAXA;
      const int x = (tid % (KMAXA * KMAXA)) / KMAXA, y = tid % KMAXA;
      const int u = J * k.a + x, up = (J - (diag ? 0 : 1)) * k.a + y;
      const double v =
          (x < k.a && y < k.a && u < k.U && up >= 0 && up < k.U) ? kron_outer(k, u, up) : 0.0;
      (diag ? KA : KN)[x][y] = v;
    }
  }
  for (int x = tid; x < TB * TB / 2; x += SWEEP_THREADS) {
    const int r = x >> 5, c2 = (x & 31) * 2;
    if (has_r) {
      cp_async16_zfill(Dt + r * SLD + c2, a.Dl + ts - TB + (int64_t)r * np + c2, true);
      if (kron && a.kd.a == 1) {  // I_a (x) Lin = Lin, [target column][source column]
        cp_async16_zfill(Rt + r * SLD + c2, a.kd.lin + r * TB + c2, c0 + r < a.n);
      } else if (kron) {
        const int lg = a.kd.lg, mk = a.kd.m_in - 1;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int c = c2 + e;
          Rt[r * SLD + c] = ((r >> lg) == (c >> lg) && c0 + r < a.n)
                                ? a.kd.lin[((r & mk) << lg) + (c & mk)]
                                : 0.0;
        }
      } else {
        cp_async16_zfill(Rt + r * SLD + c2, a.Rh + (int64_t)(c0 + r) * np + c0 - TB + c2, true);
      }
    }
    if (has_d) {
      cp_async16_zfill(Lt + r * SLD + c2, a.Lh + (int64_t)(r0 + r) * a.mp + r0 - TB + c2, true);
      cp_async16_zfill(Tq + r * SLD + c2, a.P + ts - (int64_t)TB * np + (int64_t)r * np + c2, true);
    }
  }
  cp_async_commit_group();
  // far-field feedback reaches a tile only from two or more tiles away: P needs
  // J >= 2 and E needs I >= 2 (else zero; those buffers may not be zeroed yet)
  // (with the right factor per mode, P is an operand of the right product: it goes
  // with the first batch)
  if constexpr (KRON) {
    for (int x = tid; x < TB * TB / 2; x += SWEEP_THREADS) {
      const int r = x >> 5, c2 = (x & 31) * 2;
      cp_async16_zfill(Pt + r * SLD + c2, J >= 2 ? a.P + ts + (int64_t)r * np + c2 : a.P, J >= 2);
    }
    cp_async_commit_group();
  }
  for (int x = tid; x < TB * TB / 2; x += SWEEP_THREADS) {
    const int r = x >> 5, c2 = (x & 31) * 2;
    if (!kron)
      cp_async16_zfill(Pt + r * SLD + c2, J >= 2 ? a.P + ts + (int64_t)r * np + c2 : a.P, J >= 2);
    cp_async16_zfill(Vt + r * SLD + c2, I >= 2 ? a.E + ts + (int64_t)r * np + c2 : a.E, I >= 2);
  }
  cp_async_commit_group();
  // grid of every (row, 8-column sub-tile): step, its reciprocal, integer zero point
  // (a scale group holds a multiple of 8 columns, so a sub-tile lies in one group);
  // the factor diagonals of the tile
  __shared__ double Ss[TB][NSUB], Si[TB][NSUB];
  __shared__ float Sz[TB][NSUB];
  __shared__ double Sdl[TB], Sdr[TB];
  static_assert(SWEEP_THREADS == TB * NSUB, "one thread per (row, sub-tile column)");
  {
    const int r = tid / NSUB, qs = tid % NSUB;
    const int64_t col = c0 + SUB * qs;
    double sv = 1.0;
    float z = 0.f;
    if (r < rows && col < a.n) {
      const int64_t gi = (int64_t)(r0 + r) * a.lds + (a.group ? col / a.group : 0);
      sv = (double)a.scales[gi];
      if (a.zero) z = (float)a.zero[gi];
    }
    Ss[r][qs] = sv;
    Si[r][qs] = 1.0 / sv;
    Sz[r][qs] = z;
    if (tid < TB) {
      Sdl[tid] = a.dL[r0 + tid];
      Sdr[tid] = a.dR[c0 + tid];
    }
  }
  // W of the tile (zero outside the matrix)
  constexpr int WPT = TB * TB / SWEEP_THREADS;
  double wv[WPT];
#pragma unroll
  for (int u = 0; u < WPT; ++u) {
    const int x = tid + u * SWEEP_THREADS, r = x >> 6, c = x & 63;
    wv[u] = (r < rows && c < cols)
                ? to_f64(static_cast<const TW*>(a.W)[(int64_t)(r0 + r) * a.ldw + c0 + c])
                : 0.0;
  }
  if (kron) {
    // P += dW[I,J-1] mixed by Ah[J,J-1]: column (x, v) of the tile takes
    // sum_y Ah[Ja+x][(J-1)a+y] dW[I,J-1][., (y, v)]
    cp_async_wait_group<1>();
    __syncthreads();
    if (has_r) {
      const int lg = a.kd.lg, v_mask = a.kd.m_in - 1, na = a.kd.a;
      for (int e = tid; e < TB * TB; e += SWEEP_THREADS) {
        const int r = e >> 6, c = e & 63, xq = c >> lg, v = c & v_mask;
        double sacc = Pt[r * SLD + c];
        for (int y = 0; y < na; ++y) sacc = fma(KN[xq][y], Dt[r * SLD + (y << lg) + v], sacc);
        Pt[r * SLD + c] = sacc;
      }
    }
  } else {
    cp_async_wait_group<1>();
  }
  __syncthreads();
  {
    // warp w8 = warp % 8 owns rows (w8>>1)*16..+16, columns (w8&1)*32..+32
    const int w8 = warp & 7, nr = (w8 >> 1) * 16, nc = (w8 & 1) * 32;
    const bool right = warp < 8;
    const double* Ar = kron ? Pt : Dt;  // the right product's A operand
    double acc[2][4][2] = {};
    if (right ? has_r : has_d) {
#pragma unroll 4
      for (int kk = 0; kk < TB; kk += 4) {
        double av[2], bv[4];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int r = nr + i * 8 + g;
          av[i] = right ? Ar[r * SLD + kk + t4] : Lt[r * SLD + kk + t4];
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int c = nc + j * 8 + g;
          bv[j] = right ? Rt[c * SLD + kk + t4] : Tq[(kk + t4) * SLD + c];
        }
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) dmma_m8n8k4(acc[i][j][0], acc[i][j][1], av[i], bv[j]);
      }
    }
    cp_async_wait_group<0>();
    __syncthreads();
    double* C = right ? Pt : Vt;
    const bool overwrite = right && kron;  // the mixed sum was the product's operand
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        double* c = C + (nr + i * 8 + g) * SLD + nc + j * 8 + 2 * t4;
        c[0] = overwrite ? acc[i][j][0] : c[0] + acc[i][j][0];
        c[1] = overwrite ? acc[i][j][1] : c[1] + acc[i][j][1];
      }
  }
  __syncthreads();
  // ---- W -> Dt, V += W; diagonal blocks of the normalised factors -> Rt, Lt
  for (int x = tid; x < TB * TB / 2; x += SWEEP_THREADS) {
    const int r = x >> 5, c2 = (x & 31) * 2;
    if (kron && a.kd.a == 1) {
      // Rh[J,J] = Lin; the sweep reads only its strictly lower part
      cp_async16_zfill(Rt + r * SLD + c2, a.kd.lin + r * TB + c2, c0 + r < a.n);
    } else if (kron) {  // Rh[J,J] = Ah[J,J] (x) Lin, strictly lower
      const int lg = a.kd.lg, mk = a.kd.m_in - 1;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int c = c2 + e;
        Rt[r * SLD + c] = (c < r && c0 + r < a.n)
                              ? KA[r >> lg][c >> lg] * a.kd.lin[((r & mk) << lg) + (c & mk)]
                              : 0.0;
      }
    } else {
      cp_async16_zfill(Rt + r * SLD + c2, a.Rh + (int64_t)(c0 + r) * np + c0 + c2, true);
    }
    cp_async16_zfill(Lt + r * SLD + c2, a.Lh + (int64_t)(r0 + r) * a.mp + r0 + c2, true);
  }
  cp_async_commit_group();
#pragma unroll
  for (int u = 0; u < WPT; ++u) {
    const int x = tid + u * SWEEP_THREADS, r = x >> 6, c = x & 63;
    Dt[r * SLD + c] = wv[u];
    Vt[r * SLD + c] += wv[u];
  }
  cp_async_wait_group<0>();
  __syncthreads();

  // One 8x8x8 FP64 tensor-core product: the finished sub-tile (p, q) pushes to
  //   right (p, tgt):  P[p][tgt] += dW[p][q] Rh[tgt][q]^T
  //   down  (tgt, q):  V[tgt][q] += Lh[tgt][p] P_final[p][q]
  auto sub_update = [&](int p, int q, bool right, int tgt) {
    const int R0 = SUB * p, C0 = SUB * q, T0 = SUB * tgt;
    double* C = right ? Pt + (R0 + g) * SLD + T0 + 2 * t4 : Vt + (T0 + g) * SLD + C0 + 2 * t4;
    double c0v = C[0], c1v = C[1];
#pragma unroll
    for (int kk = 0; kk < SUB; kk += 4) {
      const double av = right ? Dt[(R0 + g) * SLD + C0 + kk + t4] : Lt[(T0 + g) * SLD + R0 + kk + t4];
      const double bv = right ? Rt[(T0 + g) * SLD + C0 + kk + t4] : Pt[(R0 + kk + t4) * SLD + C0 + g];
      dmma_m8n8k4(c0v, c1v, av, bv);
    }
    C[0] = c0v;
    C[1] = c1v;
  };

  double loss = 0.0;
  long long ncl = 0, nnt = 0, nnf = 0, nor = 0;
  const int sa = lane >> 2, cq = lane & 3;  // row inside a sub-tile, column group (cq, cq + 4)
  for (int w = 0; w < 2 * NSUB - 1; ++w) {
    const int p0 = w - (NSUB - 1) > 0 ? w - (NSUB - 1) : 0;
    const int p1 = w < NSUB - 1 ? w : NSUB - 1;
    const int nsub = p1 - p0 + 1;

    // ---- sweep: warp i takes sub-tile (p0 + i, w - p0 - i)
    if (warp < nsub) {
      const int p = p0 + warp, q = w - p;
      const int R0 = SUB * p, C0 = SUB * q;
      if (R0 < rows && C0 < cols) {
        const int ar = R0 + sa;
        const bool rok = ar < rows;
        const double s = Ss[ar][q], inv_s = Si[ar][q];
        // admissible range of this sub-tile's entries: the symmetric grid, or the
        // codes [0, 2^bits - 1] shifted by the zero point
        const double zq = Sz[ar][q];
        const double lo = a.zero ? (a.clamp ? -zq : -HUGE_VAL) : a.lo;
        const double hi = a.zero ? (a.clamp ? a.top - zq : HUGE_VAL) : a.hi;
        double P[2], V[2], Wd[2];
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
          const int cc = C0 + cq + 4 * sl;
          P[sl] = Pt[ar * SLD + cc];
          V[sl] = Vt[ar * SLD + cc];
          Wd[sl] = Dt[ar * SLD + cc];
        }
#pragma unroll
        for (int t = 0; t < 2 * SUB - 1; ++t) {
          // The entry of this lane on local anti-diagonal t, if any: at most one of
          // its two slots lies on it.  One branch-free chain for all owner lanes.
          const bool o1 = sa + cq + 4 == t;
          const bool mine = (sa + cq == t || o1) && rok && C0 + cq + (o1 ? 4 : 0) < cols;
          const double Px = o1 ? P[1] : P[0];
          const double y = (o1 ? V[1] : V[0]) + Px;
          const double tq = y * inv_s;
          const double qr = (tq + 6755399441055744.0) - 6755399441055744.0;  // rint, |t| <= 2^51
          const double qv = qr < lo ? lo : (qr > hi ? hi : qr);  // lo/hi infinite: no clamp
          const double delta = fma(-s, qv, o1 ? Wd[1] : Wd[0]);
          const double pf = Px + delta;
          const double dO = mine ? delta : 0.0, pO = mine ? pf : 0.0;
          if (mine && !o1) { P[0] = pf; Wd[0] = delta; }
          if (mine && o1) { P[1] = pf; Wd[1] = delta; }
          // dW of this row's entry (column t - sa) and P_final of each column's entry (row t - col)
          const int cl = t - sa;
          const double dRow = __shfl_sync(0xffffffffu, dO, (sa << 2) | (cl & 3));
          double pCol[2];
#pragma unroll
          for (int sl = 0; sl < 2; ++sl)
            pCol[sl] = __shfl_sync(0xffffffffu, pO, (((t - cq - 4 * sl) & 7) << 2) | cq);
#pragma unroll
          for (int sl = 0; sl < 2; ++sl) {
            const int col = cq + 4 * sl, ae = t - col;
            if (cl >= 0 && cl < col)  // row push: P[sa][col] += dW[sa][cl] Rh[col][cl]
              P[sl] = fma(dRow, Rt[(C0 + col) * SLD + C0 + cl], P[sl]);
            if (ae >= 0 && ae < sa)   // column push: V[sa][col] += Lh[sa][ae] P_final[ae][col]
              V[sl] = fma(pCol[sl], Lt[(R0 + sa) * SLD + R0 + ae], V[sl]);
          }
          if (mine) Tq[ar * SLD + C0 + cq + (o1 ? 4 : 0)] = tq;  // off the chain
        }
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
          const int cc = C0 + cq + 4 * sl;
          Pt[ar * SLD + cc] = P[sl];
          Dt[ar * SLD + cc] = Wd[sl];
        }
      }
    }
    // ---- meanwhile, warps NSUB.. apply the updates of sub-wavefront w-1 that are not
    // needed before sub-wavefront w+2 (targets two or more sub-tiles away); they
    // touch sub-tiles no sweep of wave w reads or writes
    if (warp >= NSUB && w >= 1) {
      const int wp = w - 1;
      const int pp0 = wp - (NSUB - 1) > 0 ? wp - (NSUB - 1) : 0;
      const int pp1 = wp < NSUB - 1 ? wp : NSUB - 1;
      int x = warp - NSUB;
      for (int pp = pp0; pp <= pp1; ++pp) {
        const int qq = wp - pp;
        const int nr = NSUB - 2 - qq > 0 ? NSUB - 2 - qq : 0;  // right targets qq+2 ..
        const int nd = NSUB - 2 - pp > 0 ? NSUB - 2 - pp : 0;  // down targets pp+2 ..
        for (; x < nr + nd; x += SWEEP_THREADS / 32 - NSUB) {
          if (x < nr) sub_update(pp, qq, true, qq + 2 + x);
          else sub_update(pp, qq, false, pp + 2 + (x - nr));
        }
        x -= nr + nd;
      }
    }
    __syncthreads();
    if (w == 2 * NSUB - 2) break;

    // ---- the urgent updates of sub-wavefront w: its right and lower neighbours
    if (warp < 2 * nsub) {
      const int p = p0 + (warp >> 1), q = w - p;
      if ((warp & 1) == 0) {
        if (q + 1 < NSUB) sub_update(p, q, true, q + 1);
      } else {
        if (p + 1 < NSUB) sub_update(p, q, false, p + 1);
      }
    }
    __syncthreads();
  }

  // ---- outputs: final P and dW of the tile (whole tile, padding included), Q
  for (int x = tid; x < TB * TB / 2; x += SWEEP_THREADS) {
    const int r = x >> 5, c2 = (x & 31) * 2;
    *reinterpret_cast<double2*>(a.P + ts + (int64_t)r * np + c2) =
        make_double2(Pt[r * SLD + c2], Pt[r * SLD + c2 + 1]);
    *reinterpret_cast<double2*>(a.Dl + ts + (int64_t)r * np + c2) =
        make_double2(Dt[r * SLD + c2], Dt[r * SLD + c2 + 1]);
  }
  // Q and the statistics of every rounded entry, from its t = y / s:
  // loss term (M_L[i,i] M_R[j,j] s (t - q))^2 (the nearest-plane residual identity).
  // Two adjacent columns per thread (one byte of packed output; both in one sub-tile).
  for (int x = tid; x < TB * TB / 2; x += SWEEP_THREADS) {
    const int r = x >> 5, c = (x & 31) * 2;
    if (r >= rows || c >= cols) continue;
    const double sr = Ss[r][c / SUB], zq = Sz[r][c / SUB];
    const double lo = a.zero ? (a.clamp ? -zq : -HUGE_VAL) : a.lo;
    const double hi = a.zero ? (a.clamp ? a.top - zq : HUGE_VAL) : a.hi;
    int code[2] = {0, 0};
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int cc = c + k;
      if (cc >= cols) break;
      const double tq = Tq[r * SLD + cc];
      const double qr = (tq + 6755399441055744.0) - 6755399441055744.0;
      const double qv = qr < lo ? lo : (qr > hi ? hi : qr);
      // an unclamped integer beyond the int8 range is stored saturated and counted
      // (only the symmetric byte output can be unclamped: zero points and packing
      // require clamping, which keeps every code inside its byte)
      const double qs = a.clamp ? qv : fmin(fmax(qv, -128.0), 127.0);
      nor += (qs != qv) && isfinite(tq);
      code[k] = (int)(qs + zq + a.code_off);
      const double res = Sdl[r] * Sdr[cc] * sr * (tq - qv);
      loss += res * res;
      ncl += (qv != qr);
      const double qn = qr + (tq >= qr ? 1.0 : -1.0);
      nnt += (0.5 - fabs(tq - qr) < 1e-6) && (fmin(qr, qn) >= lo) && (fmax(qr, qn) <= hi);
      nnf += !isfinite(tq);
      // a bad step counts once per group (at the group's first column)
      const int64_t col = (int64_t)c0 + cc;
      if ((a.group ? col % a.group == 0 : col == 0) && !(sr > 0.0 && isfinite(sr))) ++nnf;
    }
    uint8_t* qrow = a.Q + (int64_t)(r0 + r) * a.ldq;
    if (a.packed) {
      qrow[(c0 + c) / 2] = (uint8_t)((code[0] & 15) | ((code[1] & 15) << 4));
    } else {
      qrow[c0 + c] = (uint8_t)code[0];
      if (c + 1 < cols) qrow[c0 + c + 1] = (uint8_t)code[1];
    }
  }

  // ---- tile statistics (fixed reduction order: deterministic)
  __shared__ double red_l[SWEEP_THREADS / 32];
  __shared__ long long red_c[SWEEP_THREADS / 32][4];
  for (int o = 16; o > 0; o >>= 1) {
    loss += __shfl_down_sync(0xffffffffu, loss, o);
    ncl += __shfl_down_sync(0xffffffffu, ncl, o);
    nnt += __shfl_down_sync(0xffffffffu, nnt, o);
    nnf += __shfl_down_sync(0xffffffffu, nnf, o);
    nor += __shfl_down_sync(0xffffffffu, nor, o);
  }
  if (lane == 0) {
    red_l[warp] = loss;
    red_c[warp][0] = ncl;
    red_c[warp][1] = nnt;
    red_c[warp][2] = nnf;
    red_c[warp][3] = nor;
  }
  __syncthreads();
  if (tid == 0) {
    TileStat st{0.0, 0, 0, 0, 0};
    for (int w2 = 0; w2 < SWEEP_THREADS / 32; ++w2) {
      st.loss += red_l[w2];
      st.clamped += red_c[w2][0];
      st.near_tie += red_c[w2][1];
      st.nonfinite += red_c[w2][2];
      st.out_of_range += red_c[w2][3];
    }
    a.part[(int64_t)I * a.Tn + J] = st;
  }
}

// ---------------------------------------------------------------------------
// band products to tiles two or more tiles away
// ---------------------------------------------------------------------------
constexpr int MAX_GROUPS = 512;  // 2 groups per tile: 256 tiles per launch
constexpr int MAX_STREAMS = 640;  // task streams of one plan over both of its launches
constexpr int FAR_HELP = 16;      // groups a stream helps once its own run dry
constexpr int FAR_CLAIM = 2;      // tasks a stream claims from a group at a time
// One wavefront's far-field tasks.  Group g < nt holds the right tasks of source
// tile I0+g, group g >= nt its down tasks; the tasks of a group share one
// operand.  Each group has a task counter in the workspace, so the streams on a
// group take its tasks one at a time; stream s works on own[s] (or, when there
// are fewer streams than groups, on every rr-th group from its own index) and
// then helps the groups in help[].
struct FarPlan {
  int D, I0, nt;     // source tiles: I0..I0+nt-1 of wavefront D
  int dist0;         // distance of the first target tile (2: far field)
  int cap;           // most tasks per group
  int* gcnt;         // per-group task counters, zero before the first launch on this plan
  int stream_base;   // index of this launch's first stream
  int nstreams;      // streams planned over both launches
  int rr_a, rr_b;    // nonzero: streams < rr_a take every rr_a-th group, the rest every rr_b-th
  int nhelp;
  short help[FAR_HELP];
  short own[MAX_STREAMS];
};

constexpr int FAR_CONS = 128;                    // consumer threads per task stream (4 warps)
constexpr int FAR_THREADS = 2 * FAR_CONS + 64;   // 2 streams + one producer warp each
constexpr int FAR_SLOTS = 3;                     // 64x64 tile buffers per stream
constexpr int FAR_DQ = 4;                        // task descriptors in flight per stream
constexpr int FAR_TILE_BYTES = TB * TB * (int)sizeof(double);
constexpr int FAR_STREAM_DOUBLES = FAR_SLOTS * TB * SLD;
constexpr int FAR_SMEM = 2 * FAR_STREAM_DOUBLES * (int)sizeof(double);

// One task for the consumers: the slots of its operands and its target tile.
struct FarDesc {
  double* C;      // 64x64 target tile (row stride np)
  int task_slot;  // buffer holding R^[J+d+x, J] ([c][k]) or L^[I+d+x, I] ([a][k])
  int sh_slot;    // buffer holding dW[I,J] ([a][k]) or P_final[I,J] ([k][c])
  int flags;      // FD_* bits
};
constexpr int FD_DOWN = 1, FD_FIRST = 2, FD_LAST = 4, FD_END = 8;

// mbarriers of one stream:
//   full[s]  : producer's expect_tx + the 64 row copies into slot s (count 1)
//   empty[s] : one arrival per consumer warp when it is done with slot s (count 4)
//   dqf[e]   : descriptor e written (count 1); dqe[e]: descriptor e read (count 4)
struct FarSync {
  uint64_t full[FAR_SLOTS], empty[FAR_SLOTS], dqf[FAR_DQ], dqe[FAR_DQ];
  FarDesc desc[FAR_DQ];
};

// Each CTA runs two independent task streams.  A stream is one producer warp and
// four consumer warps.  The producer walks its list of groups (FarPlan), claims
// the group's tasks one at a time from the group's counter (a task is one
// 64x64x64 product; the tasks of a group share one operand, loaded once per
// group and stream) and brings every operand tile in with 512-byte bulk row
// copies (TMA engine) that complete on the slot's mbarrier.  Slots are handed out
// in the order the consumers free them, so the next group's shared operand is
// fetched while the current one runs.  The consumers wait for a descriptor and
// its slots, run the DMMA product, free the slots, and add the product into P or
// E by reductions in L2 (red_add: each element gets one contribution per launch,
// so the sum equals a load, add and store).  Both launches on one plan (one
// beside the next sweep, one on the SMs that sweep frees) share the counters.
// Every wait gives up after kWaitLimitNs, sets *a.err and leaves the kernel (the
// call then reports GPTQ2D_ERR_TIMEOUT); a producer that gives up first waits,
// again bounded, for the copies it has in flight.
__global__ void __launch_bounds__(FAR_THREADS, 1) far_kernel(QArgs a, FarPlan pl) {
  extern __shared__ __align__(128) double sm[];
  __shared__ FarSync sync[2];
  __shared__ __align__(16) double stage[8][8 * 40];  // per consumer warp: one 8x32 strip (row stride 40)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool producer = warp >= 8;
  const int h = producer ? warp - 8 : warp >> 2;  // task stream
  double* const Slot0 = sm + h * FAR_STREAM_DOUBLES;
  auto slot_ptr = [&](int s) { return Slot0 + s * (TB * SLD); };
  FarSync& S = sync[h];
  if (threadIdx.x < 2) {
    FarSync& T = sync[threadIdx.x];
    for (int s = 0; s < FAR_SLOTS; ++s) {
      mbar_init(&T.full[s], 1);
      mbar_init(&T.empty[s], 4);
    }
    for (int e = 0; e < FAR_DQ; ++e) {
      mbar_init(&T.dqf[e], 1);
      mbar_init(&T.dqe[e], 4);
    }
  }
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  __syncthreads();
  const int64_t np = a.np;

  if (producer) {
    const uint64_t keep = policy_evict_last(), stream = policy_evict_first();
    int fills[FAR_SLOTS] = {0, 0, 0};  // fills issued per slot
    int fifo[4] = {0, 1, 2, 0};        // slots in the order the consumers free them
    int fh = 0, ft = FAR_SLOTS, nd = 0;
    bool ok = true;
    // the next slot in release order, once the consumers have freed it
    auto acquire = [&](int& s) -> bool {
      s = fifo[fh & 3];
      ++fh;
      const int k = fills[s];
      if (k > 0 && !mbar_wait(&S.empty[s], (k - 1) & 1)) return false;
      fills[s] = k + 1;
      return true;
    };
    auto release_later = [&](int s) {
      fifo[ft & 3] = s;
      ++ft;
    };
    auto fill = [&](int s, const double* src, int64_t ld, uint64_t pol) {
      if (lane == 0) mbar_arrive_expect_tx(&S.full[s], FAR_TILE_BYTES);
      __syncwarp();
      double* dst = slot_ptr(s);
      for (int r = lane; r < TB; r += 32)
        bulk_g2s(dst + r * SLD, src + (int64_t)r * ld, TB * sizeof(double), &S.full[s], pol);
    };
    auto put_desc = [&](double* C, int ts, int shs, int flags) -> bool {
      const int e = nd % FAR_DQ, k = nd / FAR_DQ;
      if (k > 0 && !mbar_wait(&S.dqe[e], (k - 1) & 1)) return false;
      if (lane == 0) {
        S.desc[e].C = C;
        S.desc[e].task_slot = ts;
        S.desc[e].sh_slot = shs;
        S.desc[e].flags = flags;
        mbar_arrive(&S.dqf[e]);
      }
      __syncwarp();
      ++nd;
      return true;
    };
    const int G = 2 * pl.nt;
    const int sid = pl.stream_base + 2 * blockIdx.x + h;  // this stream
    int own_k = 0;
    // the next group on this stream's own list, -1 when the list is done
    auto next_group = [&]() -> int {
      if (sid < pl.nstreams) {
        if (pl.rr_a > 0) {
          const int base = sid < pl.rr_a ? sid : sid - pl.rr_a;
          const int stride = sid < pl.rr_a ? pl.rr_a : pl.rr_b;
          const int g = base + own_k * stride;
          if (stride > 0 && g < G) {
            ++own_k;
            return g;
          }
        } else if (own_k == 0) {
          ++own_k;
          return pl.own[sid];
        }
      }
      return -1;
    };
    // claims the next FAR_CLAIM tasks of group g for this stream; returns the first
    auto claim = [&](int g) -> int {
      int x = 0;
      if (lane == 0) x = atomicAdd(pl.gcnt + g, FAR_CLAIM);
      return __shfl_sync(0xffffffffu, x, 0);
    };
    auto group_count = [&](int g) -> int {
      const bool dn = g >= pl.nt;
      const int I = pl.I0 + (dn ? g - pl.nt : g), J = pl.D - I;
      // (with the right factor given per mode, kron_push_kernel does the right tasks)
      return min(pl.cap, dn ? a.Tm - I - pl.dist0 : (a.kron ? 0 : a.Tn - J - pl.dist0));
    };
    unsigned help_done = 0;  // help groups found empty
    for (int g = next_group(); ok; g = next_group()) {
      if (g < 0) {
        // own list done: look at every help group at once and join one with tasks left
        bool left = false;
        if (lane < pl.nhelp && !((help_done >> lane) & 1u)) {
          const int hg = pl.help[lane];
          left = *(volatile const int*)(pl.gcnt + hg) < group_count(hg);
        }
        const unsigned m = __ballot_sync(0xffffffffu, left);
        help_done |= ~m & ((pl.nhelp >= 32 ? 0u : (1u << pl.nhelp)) - 1u);
        if (m == 0) break;
        const int q = __ffs(m) - 1;
        help_done |= 1u << q;
        g = pl.help[q];
      }
      const bool down = g >= pl.nt;
      const int I = pl.I0 + (down ? g - pl.nt : g), J = pl.D - I;
      const int count = group_count(g);
      if (count <= 0) continue;
      int x = claim(g), xe = min(x + FAR_CLAIM, count);
      if (x >= count) continue;  // nothing left: no operand load
      // shared operand: right -> dW[I,J] as [a][k]; down -> P_final[I,J] as [k][c]
      int shs;
      ok = acquire(shs);
      if (!ok) break;
      fill(shs, (down ? a.P : a.Dl) + (int64_t)I * TB * np + J * TB, np, stream);
      const int64_t opld = down ? a.mp : np;
      bool first = true;
      while (ok) {
        int xn = xe;
        bool lastx = false;
        if (x + 1 >= xe) {  // last of the claimed run: claim more before publishing it
          xn = claim(g);
          lastx = xn >= count;
        }
        int ts;
        ok = acquire(ts);
        if (!ok) break;
        // right: Rh[(J+d+x) rows][J cols] as [c][k]; down: Lh[(I+d+x) rows][I cols] as [a][k]
        fill(ts,
             down ? a.Lh + (int64_t)(I + pl.dist0 + x) * TB * a.mp + I * TB
                  : a.Rh + (int64_t)(J + pl.dist0 + x) * TB * np + J * TB,
             opld, keep);
        release_later(ts);
        if (lastx) release_later(shs);
        double* C = down ? a.E + (int64_t)(I + pl.dist0 + x) * TB * np + J * TB
                         : a.P + (int64_t)I * TB * np + (J + pl.dist0 + x) * TB;
        ok = put_desc(C, ts, shs,
                      (down ? FD_DOWN : 0) | (first ? FD_FIRST : 0) | (lastx ? FD_LAST : 0));
        first = false;
        if (lastx) break;
        if (x + 1 >= xe) {
          x = xn;
          xe = min(xn + FAR_CLAIM, count);
        } else {
          ++x;
        }
      }
    }
    if (ok) ok = put_desc(nullptr, 0, 0, FD_END);
    if (!ok) {
      if (lane == 0) atomicExch(a.err, 1);
      for (int s = 0; s < FAR_SLOTS; ++s)  // let this warp's copies land before the CTA exits
        if (fills[s] > 0) mbar_wait(&S.full[s], (fills[s] - 1) & 1);
    }
    return;
  }

  // consumers: warp cw of this stream owns the 32x32 quadrant (cw>>1, cw&1)
  const int cw = warp & 3, g8 = lane >> 2, t4 = lane & 3;
  const int wr = (cw >> 1) * 32, wc = (cw & 1) * 32;
  unsigned par = 0;  // bit s: parity of the next phase of full[s] to wait for
  for (int n = 0;; ++n) {
    const int e = n % FAR_DQ;
    if (!mbar_wait(&S.dqf[e], (n / FAR_DQ) & 1)) break;
    const FarDesc d = S.desc[e];
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.dqe[e]);
    if (d.flags & FD_END) return;
    if (d.flags & FD_FIRST) {
      if (!mbar_wait(&S.full[d.sh_slot], (par >> d.sh_slot) & 1)) break;
      par ^= 1u << d.sh_slot;
    }
    if (!mbar_wait(&S.full[d.task_slot], (par >> d.task_slot) & 1)) break;
    par ^= 1u << d.task_slot;
    const bool down = (d.flags & FD_DOWN) != 0;
    const double* Ts = slot_ptr(d.task_slot);
    const double* Hs = slot_ptr(d.sh_slot);
    // A(r, k) = Ap[i * 8 * SLD + kk] for r = wr + 8i + g8, k = kk + t4 (both layouts);
    // B(k, c) for c = wc + 8j + g8: down [k][c] -> Bp[kk * SLD + 8j], right [c][k] ->
    // Bp[8j * SLD + kk].  Two loops with fixed strides, no per-load layout choice.
    const double* Ap = (down ? Ts : Hs) + (wr + g8) * SLD + t4;
    double acc[4][4][2] = {};
    auto product = [&](const double* Bp, int bk, int bj) {
#pragma unroll 4
      for (int kk = 0; kk < TB; kk += 4) {
        double av[4], bv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) av[i] = Ap[i * 8 * SLD + kk];
#pragma unroll
        for (int j = 0; j < 4; ++j) bv[j] = Bp[kk * bk + j * bj];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) dmma_m8n8k4(acc[i][j][0], acc[i][j][1], av[i], bv[j]);
      }
    };
    if (down)
      product(Hs + t4 * SLD + wc + g8, SLD, 8);
    else
      product(Ts + (wc + g8) * SLD + t4, 1, 8 * SLD);
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&S.empty[d.task_slot]);
      if (d.flags & FD_LAST) mbar_arrive(&S.empty[d.sh_slot]);
    }
    // reductions of whole 256-byte rows: each 8x32 strip goes through shared memory
    double* st = stage[warp];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        *reinterpret_cast<double2*>(st + g8 * 40 + j * 8 + 2 * t4) =
            make_double2(acc[i][j][0], acc[i][j][1]);
      __syncwarp();
#pragma unroll
      for (int r = 0; r < 8; ++r)
        red_add(d.C + (int64_t)(wr + i * 8 + r) * np + wc + lane, st[r * 40 + lane]);
      __syncwarp();
    }
  }
  if (lane == 0) atomicExch(a.err, 1);  // a wait gave up
}

// Far-field right feedback with the right factor given per mode.  The product
// dW[I,J] Rh[J',J]^T (J' >= J + 2) factors as (dW[I,J] mixed by the outer block
// Ah[J',J]) (I_a (x) Lin)^T, and the inner factor is common to every source of a
// target, so the sources add only their mixed dW into P[I,J'] (column (x, v) takes
// sum_y Ah[J'a+x][Ja+y] dW[I,J][., (y, v)]: a multiply-adds per entry, no product);
// the target's sweep applies Lin once, with its near neighbour (sweep_kernel).  One
// CTA per source tile of wavefront D and run of KP_RUN targets (one: a late
// wavefront has few sources, and a CTA's targets run one after another), with
// dW[I,J] read into shared memory from L2.  Each entry of P gets one addition per
// launch (one source per tile row on a wavefront), so the sums do not depend on the
// order of the CTAs.
constexpr int KP_RUN = 1;
constexpr int KP_THREADS = 256;
constexpr int KP_SMEM = TB * SLD * (int)sizeof(double);

inline __host__ __device__ int kp_targets(int J, int Tn) { return Tn - J - 2 > 0 ? Tn - J - 2 : 0; }

__global__ void __launch_bounds__(KP_THREADS) kron_push_kernel(QArgs a, int D, int I0, int nt) {
  extern __shared__ __align__(16) double dws[];  // dW[I,J], row stride SLD
  __shared__ double cc[KMAXA][KMAXA];
  const KronDesc& k = a.kd;
  // this CTA's source tile and run of targets
  int b = blockIdx.x, i = 0;
  for (; i < nt; ++i) {
    const int runs = (kp_targets(D - (I0 + i), a.Tn) + KP_RUN - 1) / KP_RUN;
    if (b < runs) break;
    b -= runs;
  }
  if (i >= nt) return;
  const int I = I0 + i, J = D - I;
  const int rows = min(TB, a.m - I * TB);
  const int t0 = J + 2 + b * KP_RUN, t1 = min(a.Tn, t0 + KP_RUN);
  const int64_t np = a.np;
  const double* src = a.Dl + (int64_t)I * TB * np + (int64_t)J * TB;
  for (int x = threadIdx.x; x < TB * TB / 2; x += KP_THREADS) {
    const int r = x >> 5, c2 = (x & 31) * 2;
    cp_async16_zfill(dws + r * SLD + c2, src + (int64_t)r * np + c2, true);
  }
  cp_async_commit_group();
  const int lg = k.lg, v_mask = k.m_in - 1, na = k.a;
  for (int Jt = t0; Jt < t1; ++Jt) {
    if (threadIdx.x < KMAXA * KMAXA) {
      const int x = threadIdx.x / KMAXA, y = threadIdx.x % KMAXA;
      const int u = Jt * na + x, up = J * na + y;
      cc[x][y] = (x < na && y < na && u < k.U && up < k.U) ? kron_outer(k, u, up) : 0.0;
    }
    cp_async_wait_group<0>();
    __syncthreads();
    const int cols = min(TB, a.n - Jt * TB);
    double* dst = a.P + (int64_t)I * TB * np + (int64_t)Jt * TB;
    for (int e = threadIdx.x; e < TB * TB; e += KP_THREADS) {
      const int r = e >> 6, c = e & 63;
      if (r >= rows || c >= cols) continue;
      const int xq = c >> lg, v = c & v_mask;
      double acc = 0.0;
      for (int y = 0; y < na; ++y) acc = fma(cc[xq][y], dws[r * SLD + (y << lg) + v], acc);
      red_add(dst + (int64_t)r * np + c, acc);
    }
    __syncthreads();  // cc is rewritten for the next target
  }
}

// Sums the per-tile statistics in a fixed order into the caller's gptq2d_stats.
__global__ void __launch_bounds__(256) finalize_kernel(const TileStat* part, int ntiles,
                                                       const int* err, gptq2d_stats* out) {
  __shared__ double sl[256];
  __shared__ long long sc[256][4];
  const int tid = threadIdx.x;
  double l = 0.0;
  long long c0 = 0, c1 = 0, c2 = 0, c3 = 0;
  for (int i = tid; i < ntiles; i += 256) {
    l += part[i].loss;
    c0 += part[i].clamped;
    c1 += part[i].near_tie;
    c2 += part[i].nonfinite;
    c3 += part[i].out_of_range;
  }
  sl[tid] = l;
  sc[tid][0] = c0;
  sc[tid][1] = c1;
  sc[tid][2] = c2;
  sc[tid][3] = c3;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (tid < o) {
      sl[tid] += sl[tid + o];
      sc[tid][0] += sc[tid + o][0];
      sc[tid][1] += sc[tid + o][1];
      sc[tid][2] += sc[tid + o][2];
      sc[tid][3] += sc[tid + o][3];
    }
    __syncthreads();
  }
  if (tid == 0) {
    gptq2d_stats st;
    st.proxy_loss = sl[0];
    st.n_clamped = sc[0][0];
    st.n_near_tie = sc[0][1];
    st.n_nonfinite = sc[0][2];
    st.n_out_of_range = sc[0][3];
    st.status = *err != 0 ? GPTQ2D_ERR_TIMEOUT
                : sc[0][2] > 0 ? GPTQ2D_ERR_NONFINITE
                : sc[0][3] > 0 ? GPTQ2D_ERR_RANGE : GPTQ2D_OK;
    *out = st;
  }
}

__global__ void zero_stats_kernel(gptq2d_stats* out) {
  gptq2d_stats st{0.0, 0, 0, 0, GPTQ2D_OK, 0};
  *out = st;
}

// ---------------------------------------------------------------------------
// workspace and streams
// ---------------------------------------------------------------------------
struct WsLayout {
  int64_t mp, np;
  int Tm, Tn;
  size_t off_Lh, off_Rh, off_P, off_E, off_D, off_dL, off_dR, off_lin, off_part, off_cnt, total;
  int n_cnt;  // far-field plans (MAX_GROUPS group counters each)
};

// Tiles of wavefront D, and the first of them.
inline int wave_i0(int D, int Tn) { return D - (Tn - 1) > 0 ? D - (Tn - 1) : 0; }
inline int wave_tiles(int D, int Tm, int Tn) {
  if (D < 0 || D > Tm + Tn - 2) return 0;
  return std::min(D, Tm - 1) - wave_i0(D, Tn) + 1;
}

// m_in > 0: the right factor is given per mode (no Rh; Lin of m_in x m_in instead).
WsLayout layout(int64_t m, int64_t n, int m_in = 0) {
  WsLayout L;
  L.mp = round_up(m, TB);
  L.np = round_up(n, TB);
  L.Tm = (int)(L.mp / TB);
  L.Tn = (int)(L.np / TB);
  const size_t mat = align256((size_t)L.mp * L.np * sizeof(double));
  size_t o = 0;
  L.off_Lh = o; o += align256((size_t)L.mp * L.mp * sizeof(double));
  L.off_Rh = o; o += m_in > 0 ? 0 : align256((size_t)L.np * L.np * sizeof(double));
  L.off_P = o; o += mat;
  L.off_E = o; o += mat;
  L.off_D = o; o += mat;
  L.off_dL = o; o += align256(L.mp * sizeof(double));
  L.off_dR = o; o += align256(L.np * sizeof(double));
  L.off_lin = o; o += align256((size_t)m_in * m_in * sizeof(double));
  L.off_part = o; o += align256((size_t)L.Tm * L.Tn * sizeof(TileStat));
  L.n_cnt = 0;
  for (int D = 0; D < L.Tm + L.Tn - 1; ++D)  // one far-field plan per MAX_GROUPS/2 tiles
    L.n_cnt += (wave_tiles(D, L.Tm, L.Tn) + MAX_GROUPS / 2 - 1) / (MAX_GROUPS / 2);
  L.off_cnt = o; o += align256((1 + (size_t)L.n_cnt * MAX_GROUPS) * sizeof(int));  // error word + group counters
  L.total = o;
  return L;
}

std::atomic<uint64_t> g_sweep_smem_set[6];  // per weight type, dense and per mode
std::atomic<uint64_t> g_far_smem_set{0};

template <typename TW>
int launch_all(QArgs& a, const WsLayout& L, gptq2d_stats* stats, cudaStream_t s, int wslot,
               int n_row_ev, const int* row_tile, cudaEvent_t* row_ev) {
  constexpr int SW_SMEM = sweep_smem_bytes<TW>();
  if (ensure_smem(sweep_kernel<TW, false>, SW_SMEM, g_sweep_smem_set[wslot]) != cudaSuccess ||
      (a.kron &&
       ensure_smem(sweep_kernel<TW, true>, SW_SMEM, g_sweep_smem_set[3 + wslot]) != cudaSuccess) ||
      ensure_smem(far_kernel, FAR_SMEM, g_far_smem_set) != cudaSuccess)
    return GPTQ2D_ERR_CUDA;
  DevStreams* ds = nullptr;
  int rc = dev_streams(&ds);
  if (rc != GPTQ2D_OK) return rc;
  std::lock_guard<std::recursive_mutex> lk(ds->mu);
  cudaStream_t hi = ds->hi, lo = ds->lo;
  bool ok = cudaEventRecord(ds->fork, s) == cudaSuccess &&
            cudaStreamWaitEvent(hi, ds->fork, 0) == cudaSuccess &&
            cudaStreamWaitEvent(lo, ds->fork, 0) == cudaSuccess;
  if (!ok) return GPTQ2D_ERR_CUDA;

  // set-up: normalised factors on the high-priority stream (the first sweeps need
  // them); zero P and E and the counters on the low-priority one, where only the
  // far-field launches, which run after it, write them (the sweeps of tiles with
  // I < 2 or J < 2, which get no far-field feedback, do not read them)
  GPTQ2D_LAUNCH(KC_OTHER, hi,
                normalize_kernel<<<(int)(a.kron ? L.mp : L.mp + L.np), 256, 0, hi>>>(a));
  if (a.kron) {
    const int64_t work = (int64_t)a.kd.m_in * a.kd.m_in + L.np;
    const int blocks = (int)std::min<int64_t>((work + 255) / 256, 4 * (int64_t)ds->sms);
    GPTQ2D_LAUNCH(KC_OTHER, hi, kron_setup_kernel<<<blocks, 256, 0, hi>>>(a));
  }
  ok = ok && cudaMemsetAsync(a.P, 0, (size_t)(L.off_D - L.off_P), lo) == cudaSuccess;
  int* counters = a.err + 1;
  ok = ok && cudaMemsetAsync(a.err, 0, (1 + (size_t)L.n_cnt * MAX_GROUPS) * sizeof(int), lo) ==
                  cudaSuccess;
  ok = ok && cudaEventRecord(ds->setup, hi) == cudaSuccess &&
       cudaStreamWaitEvent(lo, ds->setup, 0) == cudaSuccess;
  const int nd = a.Tm + a.Tn - 1;
  const int sms = ds->sms;
  int next_cnt = 0;
  // far(D) = one launch on the low-priority stream beside sweep(D+1), on the SMs that
  // sweep leaves free, plus (when the work outlasts that sweep) one on the
  // high-priority stream after sweep(D+1), on the SMs it frees; both draw chunks from
  // the same group counters.  sweep(D+2) waits for both.
  std::vector<FarPlan> prev_plans;  // far(D-1), still to get its second launch
  std::vector<int> prev_b;          // and its CTA counts
  bool far_recorded[RING] = {};
  for (int D = 0; D < nd && ok; ++D) {
    const int I0 = wave_i0(D, a.Tn);
    const int nt = wave_tiles(D, a.Tm, a.Tn);
    if (D >= 2 && far_recorded[(D - 2) % RING])
      ok = cudaStreamWaitEvent(hi, ds->far[(D - 2) % RING], 0) == cudaSuccess;
    far_recorded[D % RING] = false;
    GPTQ2D_LAUNCH(KC_SWEEP, hi,
                  (a.kron ? sweep_kernel<TW, true> : sweep_kernel<TW, false>)<<<nt, SWEEP_THREADS,
                                                                               SW_SMEM, hi>>>(a, D, I0));
    // tile row I is final after the sweep of its last tile, on wavefront I + Tn - 1
    for (int k = 0; k < n_row_ev && ok; ++k)
      if (D == row_tile[k] + a.Tn - 1) ok = cudaEventRecord(row_ev[k], hi) == cudaSuccess;
    const bool b_launched = !prev_plans.empty();
    for (size_t q = 0; q < prev_plans.size(); ++q)
      GPTQ2D_LAUNCH(KC_PROPAGATE, hi,
                    far_kernel<<<prev_b[q], FAR_THREADS, FAR_SMEM, hi>>>(a, prev_plans[q]));
    prev_plans.clear();
    prev_b.clear();

    // band products of wavefront D to tiles two or more tiles away (with the right
    // factor given per mode, the right ones are kron_push_kernel's mixed adds)
    long long total = 0, kp_runs = 0;
    for (int i = 0; i < nt; ++i) {
      const int I = I0 + i, J = D - I;
      if (a.kron)
        kp_runs += (kp_targets(J, a.Tn) + KP_RUN - 1) / KP_RUN;
      else
        total += std::max(0, a.Tn - J - 2);
      total += std::max(0, a.Tm - I - 2);
    }
    if (total == 0 && kp_runs == 0) continue;
    const int nt_next = wave_tiles(D + 1, a.Tm, a.Tn);
    const int a_ctas = std::max(sms / 4, sms - nt_next);
    // a second launch pays when the work outlasts the next sweep on a_ctas SMs
    // (about 24 tasks per CTA fit in one sweep's time)
    const bool want_b = nt_next > 0 && total > 24LL * a_ctas;
    ok = ok && cudaEventRecord(b_launched ? ds->farb[(D - 1) % RING] : ds->sw[D % RING], hi) ==
                   cudaSuccess &&
         cudaStreamWaitEvent(lo, b_launched ? ds->farb[(D - 1) % RING] : ds->sw[D % RING], 0) ==
             cudaSuccess;
    for (int tb = 0; tb < nt && ok; tb += MAX_GROUPS / 2) {  // tiles per plan
      FarPlan pl;
      pl.D = D;
      pl.I0 = I0 + tb;
      pl.nt = std::min(nt - tb, MAX_GROUPS / 2);
      pl.dist0 = 2;
      pl.cap = 1 << 30;
      pl.gcnt = counters + (size_t)(next_cnt++) * MAX_GROUPS;
      const int G = 2 * pl.nt;
      int cnt[MAX_GROUPS];
      long long tasks = 0;
      int nonempty = 0;
      for (int gidx = 0; gidx < G; ++gidx) {
        const int I = pl.I0 + (gidx < pl.nt ? gidx : gidx - pl.nt), J = D - I;
        cnt[gidx] = gidx < pl.nt ? (a.kron ? 0 : std::max(0, a.Tn - J - 2))
                                 : std::max(0, a.Tm - I - 2);
        tasks += cnt[gidx];
        nonempty += cnt[gidx] > 0;
      }
      if (tasks == 0) continue;
      const int ctas = (int)std::min<long long>(std::min(a_ctas, MAX_STREAMS / 4), (tasks + 1) / 2);
      const int b_ctas = want_b ? std::min(nt_next, MAX_STREAMS / 2 - ctas) : 0;
      const int sa = 2 * ctas, sb = 2 * b_ctas;
      pl.stream_base = 0;
      pl.nstreams = sa + sb;
      // streams of the first launch cover every group; the others join the groups
      // with the most tasks per stream (those of the second launch arrive later)
      if (sa >= nonempty) {
        pl.rr_a = pl.rr_b = 0;
        int k[MAX_GROUPS];
        int s2 = 0;
        for (int gidx = 0; gidx < G; ++gidx) {
          k[gidx] = 0;
          if (cnt[gidx] > 0) {
            pl.own[s2++] = (short)gidx;
            k[gidx] = 1;
          }
        }
        for (; s2 < sa + sb; ++s2) {
          int best = -1;
          for (int gidx = 0; gidx < G; ++gidx)
            if (cnt[gidx] > 0 && (best < 0 || (long long)cnt[gidx] * k[best] >
                                                  (long long)cnt[best] * k[gidx]))
              best = gidx;
          pl.own[s2] = (short)best;
          ++k[best];
        }
      } else {
        pl.rr_a = sa;
        pl.rr_b = sb;
      }
      // idle streams help the largest groups
      int order[MAX_GROUPS];
      for (int gidx = 0; gidx < G; ++gidx) order[gidx] = gidx;
      std::stable_sort(order, order + G, [&](int x, int y) { return cnt[x] > cnt[y]; });
      pl.nhelp = 0;
      for (int q = 0; q < G && pl.nhelp < FAR_HELP && cnt[order[q]] > 0; ++q)
        pl.help[pl.nhelp++] = (short)order[q];
      GPTQ2D_LAUNCH(KC_PROPAGATE, lo, far_kernel<<<ctas, FAR_THREADS, FAR_SMEM, lo>>>(a, pl));
      if (b_ctas > 0) {
        pl.stream_base = sa;
        prev_plans.push_back(pl);
        prev_b.push_back(b_ctas);
      }
    }
    if (kp_runs > 0)
      GPTQ2D_LAUNCH(KC_PROPAGATE, lo,
                    kron_push_kernel<<<(int)kp_runs, KP_THREADS, KP_SMEM, lo>>>(a, D, I0, nt));
    ok = ok && cudaEventRecord(ds->far[D % RING], lo) == cudaSuccess;
    far_recorded[D % RING] = true;
  }
  GPTQ2D_LAUNCH(KC_OTHER, hi, finalize_kernel<<<1, 256, 0, hi>>>(a.part, a.Tm * a.Tn, a.err, stats));
  ok = ok && cudaEventRecord(ds->join_hi, hi) == cudaSuccess &&
       cudaEventRecord(ds->join_lo, lo) == cudaSuccess &&
       cudaStreamWaitEvent(s, ds->join_hi, 0) == cudaSuccess &&
       cudaStreamWaitEvent(s, ds->join_lo, 0) == cudaSuccess;
  return ok ? GPTQ2D_OK : GPTQ2D_ERR_CUDA;
}

}  // namespace

size_t quantize_ws_bytes(int64_t m, int64_t n) { return layout(m, n).total; }

int kron_inner(int nf, const int64_t* dims, int* nin) {
  int64_t p = 1;
  int best = 0, cnt = 0;
  for (int f = nf - 1; f >= 0; --f) {
    if (dims[f] < 1 || p * dims[f] > TB || TB % (p * dims[f]) != 0) break;
    p *= dims[f];
    ++cnt;
    if (p >= 8) {
      best = (int)p;
      *nin = cnt;
    }
  }
  return best;
}

size_t quantize_kron_ws_bytes(int64_t m, int nf, const int64_t* dims) {
  int nin = 0;
  const int m_in = kron_inner(nf, dims, &nin);
  if (m_in == 0) return 0;
  int64_t n = 1;
  for (int f = 0; f < nf; ++f) n *= dims[f];
  return layout(m, n, m_in).total;
}

namespace {
__device__ int g_wait_status;
}  // namespace

int check_wait_timeout(long long limit_ns, cudaStream_t s) {
  int* st = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&st), g_wait_status) != cudaSuccess)
    return GPTQ2D_ERR_CUDA;
  GPTQ2D_LAUNCH(KC_OTHER, s,
                wait_timeout_kernel<<<1, 32, 0, s>>>((unsigned long long)limit_ns, st));
  int host = GPTQ2D_ERR_CUDA;
  if (cudaGetLastError() != cudaSuccess ||
      cudaMemcpyAsync(&host, st, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return GPTQ2D_ERR_CUDA;
  return host;
}

int quantize_launch(const void* W, int w_dtype, int m, int n, int64_t ldw, const double* ML,
                    int64_t ldl, const double* MR, int64_t ldr, const float* scales, int bits,
                    int clamp, int8_t* Q, int64_t ldq, gptq2d_stats* stats, void* ws,
                    cudaStream_t s, int n_row_ev, const int* row_tile, cudaEvent_t* row_ev,
                    const GridSpec* grid, const KronSpec* kron) {
  if (m == 0 || n == 0) {
    GPTQ2D_LAUNCH(KC_OTHER, s, zero_stats_kernel<<<1, 1, 0, s>>>(stats));
    return cudaGetLastError() == cudaSuccess ? GPTQ2D_OK : GPTQ2D_ERR_CUDA;
  }
  int nin = 0;
  const int m_in = kron ? kron_inner(kron->nf, kron->dims, &nin) : 0;
  if (kron && (m_in == 0 || kron->nf > KMAXF)) return GPTQ2D_ERR_INVALID_ARG;
  const WsLayout L = layout(m, n, m_in);
  char* base = static_cast<char*>(ws);
  QArgs a;
  a.W = W;
  a.ldw = ldw;
  a.m = m;
  a.n = n;
  a.ML = ML;
  a.ldl = ldl;
  a.MR = MR;
  a.ldr = ldr;
  const GridSpec gs = grid ? *grid : GridSpec{};
  a.scales = scales;
  a.lds = gs.lds;
  a.group = gs.group >= n ? 0 : gs.group;  // one group per row
  a.zero = gs.zero;
  a.lo = clamp ? -(double)(1 << (bits - 1)) : -HUGE_VAL;
  a.hi = clamp ? (double)((1 << (bits - 1)) - 1) : HUGE_VAL;
  a.top = (double)((1 << bits) - 1);
  a.code_off = (gs.packed && !gs.zero) ? (double)(1 << (bits - 1)) : 0.0;
  a.clamp = clamp;
  a.packed = gs.packed;
  a.Q = reinterpret_cast<uint8_t*>(Q);
  a.ldq = ldq;
  a.Lh = reinterpret_cast<double*>(base + L.off_Lh);
  a.Rh = reinterpret_cast<double*>(base + L.off_Rh);
  a.P = reinterpret_cast<double*>(base + L.off_P);
  a.E = reinterpret_cast<double*>(base + L.off_E);
  a.Dl = reinterpret_cast<double*>(base + L.off_D);
  a.mp = L.mp;
  a.np = L.np;
  a.dL = reinterpret_cast<double*>(base + L.off_dL);
  a.dR = reinterpret_cast<double*>(base + L.off_dR);
  a.part = reinterpret_cast<TileStat*>(base + L.off_part);
  a.err = reinterpret_cast<int*>(base + L.off_cnt);
  a.Tm = L.Tm;
  a.Tn = L.Tn;
  a.kron = kron ? 1 : 0;
  a.kd = KronDesc{};
  if (kron) {
    KronDesc& k = a.kd;
    k.nf = kron->nf;
    k.nout = kron->nf - nin;
    k.m_in = m_in;
    k.a = TB / m_in;
    k.lg = 0;
    while ((1 << k.lg) < m_in) ++k.lg;
    k.U = n / m_in;
    int64_t stride = 1;
    for (int f = k.nf - 1; f >= 0; --f) {
      k.dim[f] = (int)kron->dims[f];
      k.M[f] = kron->M[f];
      k.ld[f] = kron->ldm[f];
      k.vstride[f] = f >= k.nout ? (int)stride : 1;
      k.ustride[f] = f < k.nout ? (int)(stride / m_in) : 1;
      stride *= kron->dims[f];
    }
    k.lin = reinterpret_cast<const double*>(base + L.off_lin);
  }
  int rc;
  switch (w_dtype) {
    case GPTQ2D_F32: rc = launch_all<float>(a, L, stats, s, 0, n_row_ev, row_tile, row_ev); break;
    case GPTQ2D_BF16:
      rc = launch_all<__nv_bfloat16>(a, L, stats, s, 1, n_row_ev, row_tile, row_ev);
      break;
    default: rc = launch_all<double>(a, L, stats, s, 2, n_row_ev, row_tile, row_ev); break;
  }
  if (rc != GPTQ2D_OK) return rc;
  return cudaGetLastError() == cudaSuccess ? GPTQ2D_OK : GPTQ2D_ERR_CUDA;
}

}  // namespace gptq2d

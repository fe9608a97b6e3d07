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
// Data layout in HBM (workspace, row-major, padded to 64 x 64 tiles):
//   P  (mp x np)  right feedback  P[i,j]  = sum_{done j'<=j} dW[i,j'] Rh[j,j']
//   E  (mp x np)  down feedback   E[i,j]  = sum_{i' < tile row of i} Lh[i,i'] P[i',j]
//   Dl (mp x np)  errors dW of finished tiles
// Schedule: 64 x 64 tiles, one tile wavefront (tile row + tile column = D) at a time:
//   sweep_kernel      one CTA per tile of the wavefront; the tile's 127 local
//                     anti-diagonals run in shared memory with the rank-one,
//                     separable updates applied as a row push (along Rh) and
//                     a column push (along Lh)
//   propagate_kernel  the band products that carry a finished tile's errors to
//                     the tiles right of it (P += dW Rh^T) and its final P to
//                     the tiles below it (E += Lh P); 64x64x64 FP64 tensor-core
//                     (DMMA) tiles
// Exactness: every contribution to a tile comes from tiles on earlier
// wavefronts (through P and E) or from the tile itself (through the sweep).
#include "common.cuh"

namespace gptq2d {

namespace {

constexpr int SLD = TB + 4;    // 68 doubles: shared tiles accessed along rows and anti-diagonals
constexpr int KLD = TB + 8;    // 72 doubles: [k][n] operand tiles of the band products
constexpr int SWEEP_THREADS = 256;  // 4 threads per tile row

struct QArgs {
  const void* W;
  int64_t ldw;
  int m, n;
  const double* ML;
  int64_t ldl;
  const double* MR;
  int64_t ldr;
  const float* scales;
  double lo, hi;
  int clamp;
  int8_t* Q;
  int64_t ldq;
  double* P;
  double* E;
  double* Dl;
  int64_t lds;  // leading dimension of P, E, Dl (np)
  const double* dL;     // M_L[i,i]   (mp, zero-padded)
  const double* dR;     // M_R[j,j]   (np)
  const double* invdL;  // 1/M_L[i,i] (mp)
  const double* invdR;  // 1/M_R[j,j] (np)
  TileStat* part;       // Tm x Tn
  int Tm, Tn;
};

template <typename TW>
__device__ __forceinline__ double load_w(const QArgs& a, int64_t idx) {
  return to_f64(static_cast<const TW*>(a.W)[idx]);
}

// Diagonals of both factors and their reciprocals, zero beyond m / n.
__global__ void diag_kernel(QArgs a, int mp, int np) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < mp + np; i += gridDim.x * blockDim.x) {
    if (i < mp) {
      const double d = (i < a.m) ? a.ML[(int64_t)i * a.ldl + i] : 0.0;
      const_cast<double*>(a.dL)[i] = d;
      const_cast<double*>(a.invdL)[i] = (i < a.m) ? 1.0 / d : 0.0;
    } else {
      const int j = i - mp;
      const double d = (j < a.n) ? a.MR[(int64_t)j * a.ldr + j] : 0.0;
      const_cast<double*>(a.dR)[j] = d;
      const_cast<double*>(a.invdR)[j] = (j < a.n) ? 1.0 / d : 0.0;
    }
  }
}

// One CTA per tile (I, J) with I = I0 + blockIdx.x, J = D - I.
template <typename TW>
__global__ void __launch_bounds__(SWEEP_THREADS) sweep_kernel(QArgs a, int D, int I0) {
  extern __shared__ double sm[];
  double* Ws = sm;                // W, overwritten by dW as entries are rounded
  double* V = Ws + TB * SLD;      // W + E + in-tile column feedback
  double* Pt = V + TB * SLD;      // P of the tile (left feedback + in-tile row feedback)
  double* Lh = Pt + TB * SLD;     // Lh[a][a'] = M_L[r0+a][r0+a'] / M_L[r0+a][r0+a], a' < a
  double* Rh = Lh + TB * SLD;     // Rh[c'][c] = M_R[c0+c'][c0+c] / M_R[c0+c'][c0+c'], c < c'
  signed char* Qs = reinterpret_cast<signed char*>(Rh + TB * SLD);  // TB x TB

  const int I = I0 + blockIdx.x, J = D - I;
  const int r0 = I * TB, c0 = J * TB;
  const int rows = min(TB, a.m - r0), cols = min(TB, a.n - c0);
  const int tid = threadIdx.x;

  for (int e = tid; e < TB * TB; e += SWEEP_THREADS) {
    const int r = e >> 6, c = e & 63;
    const int64_t wi = (int64_t)(r0 + r) * a.lds + c0 + c;
    const double w = (r < rows && c < cols) ? load_w<TW>(a, (int64_t)(r0 + r) * a.ldw + c0 + c) : 0.0;
    Ws[r * SLD + c] = w;
    V[r * SLD + c] = w + a.E[wi];
    Pt[r * SLD + c] = a.P[wi];
    Lh[r * SLD + c] =
        (r < rows && c < r) ? a.ML[(int64_t)(r0 + r) * a.ldl + r0 + c] * a.invdL[r0 + r] : 0.0;
    Rh[r * SLD + c] =
        (r < cols && c < r) ? a.MR[(int64_t)(c0 + r) * a.ldr + c0 + c] * a.invdR[c0 + r] : 0.0;
  }
  __syncthreads();

  const int ra = tid >> 2, k4 = tid & 3;
  const bool row_ok = ra < rows;
  const double s = row_ok ? (double)a.scales[r0 + ra] : 1.0;
  const double dl = a.dL[r0 + ra];
  const bool s_bad = row_ok && !(s > 0.0 && isfinite(s));
  double loss = 0.0;
  long long ncl = 0, nnt = 0, nnf = 0;

  const int steps = rows + cols - 1;
  for (int t = 0; t < steps; ++t) {
    const int c = t - ra;
    const bool act = row_ok && c >= 0 && c < cols;
    double delta = 0.0, pf = 0.0, q = 0.0;
    if (act) {
      const double w = Ws[ra * SLD + c];
      const double p = Pt[ra * SLD + c];
      const double y = V[ra * SLD + c] + p;
      const double tq = y / s;
      const double qr = rint(tq);
      q = a.clamp ? fmin(fmax(qr, a.lo), a.hi) : qr;
      delta = w - s * q;
      pf = p + delta;
      if (k4 == 0) {
        const double res = (dl * a.dR[c0 + c]) * (y - s * q);
        loss += res * res;
        ncl += (q != qr);
        const double h = floor(tq) + 0.5;
        nnt += (fabs(tq - h) < 1e-6) && (h - 0.5 >= a.lo) && (h + 0.5 <= a.hi);
        nnf += !isfinite(y);
      }
    }
    __syncwarp();
    if (act) {
      if (k4 == 0) {
        Pt[ra * SLD + c] = pf;
        Ws[ra * SLD + c] = delta;
        Qs[ra * TB + c] = (signed char)(int)q;
      }
      // row push: P[ra][c'] += dW * Rh[c'][c], c' > c
      for (int cc = c + 1 + k4; cc < cols; cc += 4)
        Pt[ra * SLD + cc] = fma(delta, Rh[cc * SLD + c], Pt[ra * SLD + cc]);
      // column push: V[a'][c] += Lh[a'][ra] * P_final[ra][c], a' > ra
      for (int aa = ra + 1 + k4; aa < rows; aa += 4)
        V[aa * SLD + c] = fma(pf, Lh[aa * SLD + ra], V[aa * SLD + c]);
    }
    __syncthreads();
  }

  // write back Q, dW, final P of the tile
  for (int e = tid; e < TB * TB; e += SWEEP_THREADS) {
    const int r = e >> 6, c = e & 63;
    const int64_t wi = (int64_t)(r0 + r) * a.lds + c0 + c;
    a.Dl[wi] = Ws[r * SLD + c];
    a.P[wi] = Pt[r * SLD + c];
    if (r < rows && c < cols) a.Q[(int64_t)(r0 + r) * a.ldq + c0 + c] = Qs[r * TB + c];
  }

  // tile statistics (fixed reduction order: deterministic)
  if (k4 == 0 && c0 == 0 && s_bad) ++nnf;
  __shared__ double red_l[SWEEP_THREADS / 32];
  __shared__ long long red_c[SWEEP_THREADS / 32][3];
  for (int o = 16; o > 0; o >>= 1) {
    loss += __shfl_down_sync(0xffffffffu, loss, o);
    ncl += __shfl_down_sync(0xffffffffu, ncl, o);
    nnt += __shfl_down_sync(0xffffffffu, nnt, o);
    nnf += __shfl_down_sync(0xffffffffu, nnf, o);
  }
  if ((tid & 31) == 0) {
    red_l[tid >> 5] = loss;
    red_c[tid >> 5][0] = ncl;
    red_c[tid >> 5][1] = nnt;
    red_c[tid >> 5][2] = nnf;
  }
  __syncthreads();
  if (tid == 0) {
    TileStat st{0.0, 0, 0, 0};
    for (int w = 0; w < SWEEP_THREADS / 32; ++w) {
      st.loss += red_l[w];
      st.clamped += red_c[w][0];
      st.near_tie += red_c[w][1];
      st.nonfinite += red_c[w][2];
    }
    a.part[(int64_t)I * a.Tn + J] = st;
  }
}

// Band products of the tiles of wavefront D.  blockIdx.y = tile, blockIdx.z:
//   0: right,  P[I, J+1+x] += (dW[I,J] M_R[J+1+x, J]^T) * diag(1/M_R)   (columns scaled)
//   1: down,   E[I+1+x, J] += diag(1/M_L) (M_L[I+1+x, I] P[I,J])        (rows scaled)
__global__ void __launch_bounds__(128) propagate_kernel(QArgs a, int D, int I0) {
  extern __shared__ double sm[];
  double* As = sm;             // [64][SLD]: A[row][k]
  double* Bs = sm + TB * SLD;  // right: [n][k] with SLD; down: [k][n] with KLD
  const int I = I0 + blockIdx.y, J = D - I;
  const int x = blockIdx.x;
  const bool down = blockIdx.z == 1;
  const int tid = threadIdx.x;
  int R0, C0;  // output tile origin in the workspace
  if (!down) {
    const int Jp = J + 1 + x;
    if (Jp >= a.Tn) return;
    R0 = I * TB;
    C0 = Jp * TB;
    for (int e = tid; e < TB * TB; e += blockDim.x) {
      const int r = e >> 6, c = e & 63;
      As[r * SLD + c] = a.Dl[(int64_t)(I * TB + r) * a.lds + J * TB + c];
      const int jr = Jp * TB + r, jc = J * TB + c;  // M_R[jr][jc], jr > jc always
      Bs[r * SLD + c] = (jr < a.n && jc < a.n) ? a.MR[(int64_t)jr * a.ldr + jc] : 0.0;
    }
  } else {
    const int Ip = I + 1 + x;
    if (Ip >= a.Tm) return;
    R0 = Ip * TB;
    C0 = J * TB;
    for (int e = tid; e < TB * TB; e += blockDim.x) {
      const int r = e >> 6, c = e & 63;
      const int ir = Ip * TB + r, ic = I * TB + c;
      As[r * SLD + c] = (ir < a.m && ic < a.m) ? a.ML[(int64_t)ir * a.ldl + ic] : 0.0;
      Bs[r * KLD + c] = a.P[(int64_t)(I * TB + r) * a.lds + J * TB + c];
    }
  }
  __syncthreads();

  double acc[4][4][2] = {};
  if (!down)
    mma_64x64x64(
        acc, [&](int row, int kk) { return As[row * SLD + kk]; },
        [&](int kk, int col) { return Bs[col * SLD + kk]; });
  else
    mma_64x64x64(
        acc, [&](int row, int kk) { return As[row * SLD + kk]; },
        [&](int kk, int col) { return Bs[kk * KLD + col]; });

  double* C = down ? a.E : a.P;
  const int lane = tid & 31, warp = tid >> 5, g = lane >> 2, t = lane & 3;
  const int wr = (warp >> 1) * 32, wc = (warp & 1) * 32;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = R0 + wr + i * 8 + g, c = C0 + wc + j * 8 + 2 * t;
      double2* dst = reinterpret_cast<double2*>(C + (int64_t)r * a.lds + c);
      double2 v = *dst;
      if (down) {
        const double sc = a.invdL[r];
        v.x = fma(sc, acc[i][j][0], v.x);
        v.y = fma(sc, acc[i][j][1], v.y);
      } else {
        v.x = fma(a.invdR[c], acc[i][j][0], v.x);
        v.y = fma(a.invdR[c + 1], acc[i][j][1], v.y);
      }
      *dst = v;
    }
}

// Sums the per-tile statistics in a fixed order into the caller's gptq2d_stats.
__global__ void __launch_bounds__(256) finalize_kernel(const TileStat* part, int ntiles,
                                                       gptq2d_stats* out) {
  __shared__ double sl[256];
  __shared__ long long sc[256][3];
  const int tid = threadIdx.x;
  double l = 0.0;
  long long c0 = 0, c1 = 0, c2 = 0;
  for (int i = tid; i < ntiles; i += 256) {
    l += part[i].loss;
    c0 += part[i].clamped;
    c1 += part[i].near_tie;
    c2 += part[i].nonfinite;
  }
  sl[tid] = l;
  sc[tid][0] = c0;
  sc[tid][1] = c1;
  sc[tid][2] = c2;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (tid < o) {
      sl[tid] += sl[tid + o];
      sc[tid][0] += sc[tid + o][0];
      sc[tid][1] += sc[tid + o][1];
      sc[tid][2] += sc[tid + o][2];
    }
    __syncthreads();
  }
  if (tid == 0) {
    gptq2d_stats st;
    st.proxy_loss = sl[0];
    st.n_clamped = sc[0][0];
    st.n_near_tie = sc[0][1];
    st.n_nonfinite = sc[0][2];
    st.status = sc[0][2] > 0 ? GPTQ2D_ERR_NONFINITE : GPTQ2D_OK;
    *out = st;
  }
}

__global__ void zero_stats_kernel(gptq2d_stats* out) {
  gptq2d_stats st{0.0, 0, 0, 0, GPTQ2D_OK};
  *out = st;
}

struct WsLayout {
  int64_t mp, np;
  int Tm, Tn;
  size_t off_P, off_E, off_D, off_dL, off_dR, off_idL, off_idR, off_part, total;
};

WsLayout layout(int64_t m, int64_t n) {
  WsLayout L;
  L.mp = round_up(m, TB);
  L.np = round_up(n, TB);
  L.Tm = (int)(L.mp / TB);
  L.Tn = (int)(L.np / TB);
  const size_t mat = align256((size_t)L.mp * L.np * sizeof(double));
  size_t o = 0;
  L.off_P = o; o += mat;
  L.off_E = o; o += mat;
  L.off_D = o; o += mat;
  L.off_dL = o; o += align256(L.mp * sizeof(double));
  L.off_dR = o; o += align256(L.np * sizeof(double));
  L.off_idL = o; o += align256(L.mp * sizeof(double));
  L.off_idR = o; o += align256(L.np * sizeof(double));
  L.off_part = o; o += align256((size_t)L.Tm * L.Tn * sizeof(TileStat));
  L.total = o;
  return L;
}

std::atomic<uint64_t> g_sweep_smem_set[3];
std::atomic<uint64_t> g_prop_smem_set{0};

constexpr int SWEEP_SMEM = 5 * TB * SLD * (int)sizeof(double) + TB * TB;
constexpr int PROP_SMEM = (TB * SLD + TB * KLD) * (int)sizeof(double);

template <typename TW>
int launch_all(QArgs& a, const WsLayout& L, gptq2d_stats* stats, cudaStream_t s, int wslot) {
  if (ensure_smem(sweep_kernel<TW>, SWEEP_SMEM, g_sweep_smem_set[wslot]) != cudaSuccess ||
      ensure_smem(propagate_kernel, PROP_SMEM, g_prop_smem_set) != cudaSuccess)
    return GPTQ2D_ERR_CUDA;
  const int nd = a.Tm + a.Tn - 1;
  const int gx = (a.Tm > a.Tn ? a.Tm : a.Tn) - 1;
  for (int D = 0; D < nd; ++D) {
    const int I0 = D - (a.Tn - 1) > 0 ? D - (a.Tn - 1) : 0;
    const int I1 = D < a.Tm - 1 ? D : a.Tm - 1;
    const int nt = I1 - I0 + 1;
    GPTQ2D_LAUNCH(KC_SWEEP, s, sweep_kernel<TW><<<nt, SWEEP_THREADS, SWEEP_SMEM, s>>>(a, D, I0));
    if (D < nd - 1 && gx > 0)
      GPTQ2D_LAUNCH(KC_PROPAGATE, s,
                    propagate_kernel<<<dim3(gx, nt, 2), 128, PROP_SMEM, s>>>(a, D, I0));
  }
  GPTQ2D_LAUNCH(KC_OTHER, s, finalize_kernel<<<1, 256, 0, s>>>(a.part, a.Tm * a.Tn, stats));
  return GPTQ2D_OK;
}

}  // namespace

size_t quantize_ws_bytes(int64_t m, int64_t n) { return layout(m, n).total; }

int quantize_launch(const void* W, int w_dtype, int m, int n, int64_t ldw, const double* ML,
                    int64_t ldl, const double* MR, int64_t ldr, const float* scales, int bits,
                    int clamp, int8_t* Q, int64_t ldq, gptq2d_stats* stats, void* ws,
                    cudaStream_t s) {
  if (m == 0 || n == 0) {
    GPTQ2D_LAUNCH(KC_OTHER, s, zero_stats_kernel<<<1, 1, 0, s>>>(stats));
    return cudaGetLastError() == cudaSuccess ? GPTQ2D_OK : GPTQ2D_ERR_CUDA;
  }
  const WsLayout L = layout(m, n);
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
  a.scales = scales;
  a.lo = clamp ? -(double)(1 << (bits - 1)) : -HUGE_VAL;
  a.hi = clamp ? (double)((1 << (bits - 1)) - 1) : HUGE_VAL;
  a.clamp = clamp;
  a.Q = Q;
  a.ldq = ldq;
  a.P = reinterpret_cast<double*>(base + L.off_P);
  a.E = reinterpret_cast<double*>(base + L.off_E);
  a.Dl = reinterpret_cast<double*>(base + L.off_D);
  a.lds = L.np;
  a.dL = reinterpret_cast<double*>(base + L.off_dL);
  a.dR = reinterpret_cast<double*>(base + L.off_dR);
  a.invdL = reinterpret_cast<double*>(base + L.off_idL);
  a.invdR = reinterpret_cast<double*>(base + L.off_idR);
  a.part = reinterpret_cast<TileStat*>(base + L.off_part);
  a.Tm = L.Tm;
  a.Tn = L.Tn;

  // P and E start at zero (E and P are contiguous).
  if (cudaMemsetAsync(a.P, 0, L.off_D - L.off_P, s) != cudaSuccess) return GPTQ2D_ERR_CUDA;
  GPTQ2D_LAUNCH(KC_OTHER, s, diag_kernel<<<64, 256, 0, s>>>(a, (int)L.mp, (int)L.np));
  int rc;
  switch (w_dtype) {
    case GPTQ2D_F32: rc = launch_all<float>(a, L, stats, s, 0); break;
    case GPTQ2D_BF16: rc = launch_all<__nv_bfloat16>(a, L, stats, s, 1); break;
    default: rc = launch_all<double>(a, L, stats, s, 2); break;
  }
  if (rc != GPTQ2D_OK) return rc;
  return cudaGetLastError() == cudaSuccess ? GPTQ2D_OK : GPTQ2D_ERR_CUDA;
}

}  // namespace gptq2d

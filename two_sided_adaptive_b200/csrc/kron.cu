// Kronecker product of lower-triangular factors, for Hessians with more than two
// Kronecker factors (arxivlens "GPTQ-2D: Cubic-Time Two-Sided Adaptive
// Rounding", Abstract: the algorithm extends to any number of Kronecker factors).
//
// A k-way tensor W of shape (m_1, ..., m_k) with H = H_1 (x) ... (x) H_k (H_j on
// mode j) is the 2-D problem with rows = mode 1 (H_L = H_1) and columns = modes
// 2..k flattened in C order (H_R = H_2 (x) ... (x) H_k).  The reverse Cholesky
// factor of a Kronecker product is the Kronecker product of the factors
// ((A (x) B)^T (A (x) B) = A^T A (x) B^T B, and it is lower with a positive
// diagonal), so M_R = M_2 (x) ... (x) M_k: one factorization per mode plus this
// product, instead of a factorization of the n x n Gram.  M_R is nonzero only
// where every mode index of the column is <= that of the row (the k-way product
// order), so the anti-diagonal sweep, which visits the entries in a linear
// extension of that order, computes the k-way rounding.
//
// The kernel writes every entry of out (n x n, n = prod dims): the product of
// the factors' entries where every mode index of the column is <= that of the
// row, exact zero elsewhere (the factors' strict upper triangles are not read).
// One CTA per row (grid-stride over rows), threads over the columns up to the
// diagonal; the rest of the row is a plain zero fill.  HBM-bound: 8 n^2 bytes
// written, the factors (sum of dims^2 entries) stay in L1/L2.
#include "common.cuh"

namespace gptq2d {

namespace {

struct KronArgs {
  const double* M[GPTQ2D_MAX_KRON_FACTORS];
  int64_t ld[GPTQ2D_MAX_KRON_FACTORS];
  int dim[GPTQ2D_MAX_KRON_FACTORS];
  int nf;
  int n;
  double* out;
  int64_t ldo;
};

__global__ void __launch_bounds__(256) kron_lower_kernel(KronArgs a) {
  __shared__ int rdig[GPTQ2D_MAX_KRON_FACTORS];
  for (int r = blockIdx.x; r < a.n; r += gridDim.x) {
    __syncthreads();  // the previous row's digits are no longer read
    if (threadIdx.x == 0) {
      int x = r;
      for (int f = a.nf - 1; f >= 0; --f) {  // last factor on the fastest index
        rdig[f] = x % a.dim[f];
        x /= a.dim[f];
      }
    }
    __syncthreads();
    double* orow = a.out + (int64_t)r * a.ldo;
    for (int c = threadIdx.x; c < a.n; c += blockDim.x) {
      double v = 0.0;
      if (c <= r) {
        v = 1.0;
        int x = c;
        for (int f = a.nf - 1; f >= 0; --f) {
          const int cd = x % a.dim[f];
          x /= a.dim[f];
          const int rd = rdig[f];
          v = cd <= rd ? v * a.M[f][(int64_t)rd * a.ld[f] + cd] : 0.0;
        }
      }
      orow[c] = v;
    }
  }
}

}  // namespace

int kron_factor_launch(int nf, const double* const* M, const int64_t* dims, const int64_t* ldm,
                       double* out, int64_t ldo, cudaStream_t s) {
  KronArgs a{};
  int64_t n = 1;
  for (int f = 0; f < nf; ++f) {
    a.M[f] = M[f];
    a.ld[f] = ldm[f];
    a.dim[f] = (int)dims[f];
    n *= dims[f];
  }
  a.nf = nf;
  a.n = (int)n;
  a.out = out;
  a.ldo = ldo;
  if (n == 0) return GPTQ2D_OK;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t blocks = n < (int64_t)sms * 16 ? n : (int64_t)sms * 16;
  GPTQ2D_LAUNCH(KC_OTHER, s, kron_lower_kernel<<<(int)blocks, 256, 0, s>>>(a));
  return cudaGetLastError() == cudaSuccess ? GPTQ2D_OK : GPTQ2D_ERR_CUDA;
}

}  // namespace gptq2d

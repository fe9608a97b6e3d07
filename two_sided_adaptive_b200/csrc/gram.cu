// The Kronecker factors from calibration activations, on the 5th-generation tensor
// cores (tcgen05): H = X^T X / N + damping, the step before the path (arxivlens
// "GPTQ-2D: Cubic-Time Two-Sided Adaptive Rounding", Analysis > Limitations and
// Future work: the fixed bases' Grams are formed and factored once).  A factor is
// the Gram of its basis; with A = X / sqrt(N) for N rows of activations X (N x k),
// H = A^T A.  The damping (a fraction of the mean diagonal added to the diagonal)
// is GPTQ's usual one; the pages give none.
//
// gram_kernel: one CTA per pair of 128 x 128 blocks (bi, 2c), (bi, 2c + 1) of the
// lower block triangle of H, or per diagonal block (bi, bi) of an even block row
// (then 2c = bi).  The product is D = X[:, I]^T X[:, J] over all rows, 128 x 256 (or
// 128 x 128), accumulated in fp32 in tensor memory by tcgen05.mma (kind::f16, bf16
// operands, M = 128, N = 256 or 128, K = 16 per instruction): the wide tile reads
// 12 KB of shared memory per 2^20 flops where two 128 x 128 tiles read 16 KB.  Both
// operands are chunks of 64 rows of X, and X is row-major (features contiguous), so
// A (128 features x 64 rows) and B (256 or 128 features) are "MN-major".  Each
// operand is a run of TMA boxes of 64 features x 64 rows (cp.async.bulk.tensor,
// 128-byte swizzle; zero fill past the last row or column): a box holds the rows
// as 128-byte lines, swizzled in groups of 8 lines, which is the canonical
// 128B-swizzled MN-major layout of the operand descriptor (stride byte offset 1024
// between 8-row groups, leading byte offset 8192 between 64-feature boxes).
//   warp 1, one thread  fills a 4-stage ring: it waits for the stage's empty
//                       barrier, arms the full barrier with the stage's bytes and
//                       issues the 2 (diagonal block: B = A) or 6 box loads;
//   warp 0              allocates 256 columns of tensor memory; its elected thread
//                       waits for a full stage, issues the stage's four MMAs and
//                       frees the stage with tcgen05.commit on its empty barrier.
//                       A last commit signals the end.
// Then each warp reads its 32 lanes (rows) of the accumulator with tcgen05.ld and
// writes (or adds) the fp32 block into H.  Every wait is bounded (%globaltimer);
// a wait that gives up sets the error word, and the CTA still waits (bounded) for
// its copies and MMAs and frees its tensor memory before it exits.
//
// gram_diag_kernel + gram_finalize_kernel: the diagonal's sum (one CTA, fixed order:
// deterministic) into the workspace, then H <- H / N on the lower block triangle
// and H_ii += damp * mean_i(H_ii / N).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "pipeline.cuh"

namespace gptq2d {

namespace {

constexpr int GB = 128;                      // block edge (MMA M; N is one or two blocks)
constexpr int GK = 64;                       // rows of X per stage
constexpr int GSTAGES = 4;
constexpr int GTHREADS = 128;
constexpr int G_BOX = 64 * GK * 2;           // one TMA box: 64 features x 64 rows, 8 KB
constexpr int G_TILE = 2 * G_BOX;            // one bf16 operand tile of 128 features: 16 KB
constexpr int G_STAGE = 3 * G_TILE;          // A (128 features) and B (up to 256)
constexpr int G_SMEM = GSTAGES * G_STAGE + 1024;  // + room to align the ring to 1024 bytes
constexpr uint32_t G_SBO = 1024;             // between 8-row groups
constexpr uint32_t G_LBO = G_BOX;            // between the two 64-feature boxes
constexpr uint32_t G_TMEM_COLS = 2 * GB;     // fp32 accumulator: 128 lanes x up to 256 columns

// Shared-memory operand descriptor: start address, leading and stride byte offsets
// (all in 16-byte units), descriptor version 1, 128-byte swizzle (layout type 2).
__device__ __forceinline__ uint64_t g_desc(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((G_LBO >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((G_SBO >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// One TMA box (x = feature, y = row) into shared memory, completing on `bar`.
// x is a multiple of 64 (a 128-byte boundary of a row).  No multicast.
__device__ __forceinline__ void tma_box(void* dst, const CUtensorMap* map, int x, int y,
                                        uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];\n" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Instruction descriptor (kind::f16): fp32 accumulator (bit 4), bf16 A (bit 7) and
// B (bit 10), both MN-major (bits 15, 16), N / 8 at bit 17, M / 16 at bit 24.
__host__ __device__ constexpr uint32_t g_idesc(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(GB >> 4) << 24);
}

// CTAs of block rows 0 .. B - 1: row bi holds ceil((bi + 1) / 2) of them.
__host__ __device__ inline int g_ctas_before(int B) { return (B + 1) * (B + 1) / 4; }

// CTA order.  Block rows are taken in bands of GBAND; within a band the CTAs go
// column pair by column pair (all the band's rows of pair c, then of c + 1), so the
// CTAs resident at one time share a few row blocks and a few column blocks of X and
// read them from L2, where a row-by-row order would stream a whole block row's
// columns from HBM once per wave.
constexpr int GBAND = 16;

// CTA t -> (block row bi, column pair c) for nb block rows.
__host__ __device__ inline void g_cta_block(int t, int nb, int& bi, int& c) {
  // the band is the one holding t's block row in row-by-row order
  int r = (int)(2.0f * sqrtf((float)t)) - 1;
  if (r < 0) r = 0;
  while (g_ctas_before(r + 1) <= t) ++r;
  while (r > 0 && g_ctas_before(r) > t) --r;
  const int b0 = r - r % GBAND;
  const int gb = min(GBAND, nb - b0);  // rows in the band
  int u = t - g_ctas_before(b0);
  const int c_full = b0 / 2 + 1;       // pairs c with 2c <= b0: present in every row
  if (u < c_full * gb) {
    c = u / gb;
    bi = b0 + u % gb;
    return;
  }
  u -= c_full * gb;
  for (c = c_full;; ++c) {             // pair c is in rows 2c .. b0 + gb - 1
    const int nc = b0 + gb - 2 * c;
    if (u < nc) {
      bi = 2 * c + u;
      return;
    }
    u -= nc;
  }
}

__device__ __forceinline__ void tc_mma(uint32_t tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}

struct GramArgs {
  const __nv_bfloat16* X;
  int64_t N;     // rows
  int k;         // columns (features), a multiple of 8
  int64_t ldx;   // a multiple of 8
  float* H;
  int64_t ldh;
  int beta;      // 1: add to H, 0: overwrite
  int* err;
};

__global__ void __launch_bounds__(GTHREADS, 1) gram_kernel(GramArgs a,
                                                          const __grid_constant__ CUtensorMap tmap) {
  extern __shared__ __align__(1024) uint8_t gsm_raw[];
  // the 128-byte swizzle repeats every 1024 bytes: align the ring to that
  uint8_t* gsm = gsm_raw + ((1024u - (smem_u32(gsm_raw) & 1023u)) & 1023u);
  __shared__ __align__(8) uint64_t full_bar[GSTAGES], empty_bar[GSTAGES], done_bar;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  __shared__ long long issued;  // chunks whose loads were issued
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // blocks (bi, bj0) and (bi, bj0 + 1) of the lower block triangle, bj0 = 2c (one
  // block when bj0 = bi): a 128 x 256 (or 128 x 128) product
  int bi, cp;
  g_cta_block(blockIdx.x, (a.k + GB - 1) / GB, bi, cp);
  const int bj0 = 2 * cp;
  const int nbj = bj0 + 1 <= bi ? 2 : 1;
  const int nw = nbj * GB;  // output columns
  const int i0 = bi * GB, j0 = bj0 * GB;

  if (tid == 0) {
    for (int s = 0; s < GSTAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&done_bar, 1);
    abort_flag = 0;
    issued = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     smem_u32(&tmem_base)),
                 "r"(G_TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  const int64_t nchunks = (a.N + GK - 1) / GK;

  if (warp == 1 && lane == 0) {
    // ---- producer: chunk c into stage c % GSTAGES, after the MMAs of chunk c - GSTAGES
    const bool diag = nbj == 1;  // the one-block tile is a diagonal block: B = A
    const unsigned bytes = (diag ? 1 : 3) * G_TILE;
    long long c = 0;
    for (; c < nchunks; ++c) {
      const int st = (int)(c % GSTAGES);
      if (c >= GSTAGES &&
          !mbar_wait(&empty_bar[st], (uint32_t)(((c / GSTAGES) - 1) & 1))) {
        atomicExch(&abort_flag, 1);
        break;
      }
      if (*(volatile int*)&abort_flag) break;
      uint8_t* sA = gsm + st * G_STAGE;
      const int y = (int)(c * GK);
      mbar_arrive_expect_tx(&full_bar[st], bytes);
      tma_box(sA, &tmap, i0, y, &full_bar[st]);
      tma_box(sA + G_BOX, &tmap, i0 + 64, y, &full_bar[st]);
      if (!diag)
        for (int q = 0; q < 4; ++q)  // B: 64-feature boxes, LBO = G_BOX apart
          tma_box(sA + G_TILE + q * G_BOX, &tmap, j0 + 64 * q, y, &full_bar[st]);
    }
    issued = c;
  } else if (warp == 0 && lane == 0) {
    // ---- MMA issuer (one thread)
    for (int64_t c = 0; c < nchunks; ++c) {
      const int st = (int)(c % GSTAGES);
      if (!mbar_wait(&full_bar[st], (uint32_t)((c / GSTAGES) & 1))) {
        atomicExch(&abort_flag, 1);
        break;
      }
      if (*(volatile int*)&abort_flag) break;
      tc_fence_after();
      const uint32_t aaddr = smem_u32(gsm + st * G_STAGE);
      const uint32_t baddr = nbj == 1 ? aaddr : aaddr + G_TILE;
      const uint32_t idesc = g_idesc(nw);
      // K step s16 = rows 16 s16 .. 16 s16 + 15: two 8-row groups further (2 * SBO)
#pragma unroll
      for (int s16 = 0; s16 < GK / 16; ++s16)
        tc_mma(tmem, g_desc(aaddr + s16 * 2 * G_SBO), g_desc(baddr + s16 * 2 * G_SBO), idesc,
               (c > 0 || s16 > 0) ? 1u : 0u);
      tc_commit(&empty_bar[st]);
    }
    tc_commit(&done_bar);  // completes once every MMA issued above has
  }
  __syncwarp();
  __syncthreads();
  if (abort_flag && warp == 1 && lane == 0) {
    // a wait gave up: let the box loads still in flight land before the CTA exits
    for (long long c = issued - GSTAGES > 0 ? issued - GSTAGES : 0; c < issued; ++c)
      mbar_wait(&full_bar[c % GSTAGES], (uint32_t)((c / GSTAGES) & 1));
  }
  // every thread: the accumulator is final once done_bar completes
  const bool done = mbar_wait(&done_bar, 0);
  if (!done) atomicExch(&abort_flag, 1);
  tc_fence_after();
  __syncthreads();
  const bool good = !abort_flag;
  const bool empty = nchunks == 0;  // no rows: the block is zero
  // ---- epilogue: warp w reads rows 32 w .. 32 w + 31 (its tensor-memory lanes)
  const int row = warp * 32 + lane;
  const int gi = i0 + row;
#pragma unroll 1
  for (int cb = 0; cb < nw / 32; ++cb) {
    uint32_t v[32];
    const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(cb * 32);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
          "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
          "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
          "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
    if (good && gi < a.k) {
      float* hrow = a.H + (int64_t)gi * a.ldh + j0 + cb * 32;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        if (j0 + cb * 32 + c < a.k) {
          const float x = empty ? 0.f : __uint_as_float(v[c]);
          hrow[c] = a.beta ? hrow[c] + x : x;
        }
      }
    }
  }
  if (!good && tid == 0) atomicExch(a.err, 1);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem),
                 "r"(G_TMEM_COLS)
                 : "memory");
  }
}

// sum_i H_ii into *diag_sum (one CTA; a fixed reduction order).
__global__ void __launch_bounds__(256) gram_diag_kernel(const float* H, int k, int64_t ldh,
                                                        double* diag_sum) {
  __shared__ double part[256];
  double s = 0.0;
  for (int i = threadIdx.x; i < k; i += 256) s += (double)H[(int64_t)i * ldh + i];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) part[threadIdx.x] += part[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) *diag_sum = part[0];
}

// H <- H / N on the lower block triangle (blocks of 128), H_ii += damp * mean(H_ii / N).
// One CTA per row; row r covers columns 0 .. end of its diagonal block, read and
// written once (coalesced, four independent loads in flight per thread).
__global__ void __launch_bounds__(256) gram_finalize_kernel(float* H, int k, int64_t ldh,
                                                            double inv_n, double damp,
                                                            const double* diag_sum) {
  const double shift = damp * (*diag_sum) * inv_n / (double)k;
  const int r = blockIdx.x;
  const int cend = min(k, (r / GB + 1) * GB);  // end of the row's diagonal block
  float* hr = H + (int64_t)r * ldh;
#pragma unroll 4
  for (int c = threadIdx.x; c < cend; c += 256) {
    double v = (double)hr[c] * inv_n;
    if (c == r) v += shift;
    hr[c] = (float)v;
  }
}

std::atomic<uint64_t> g_gram_smem_set{0};


// cuTensorMapEncodeTiled through the runtime's driver entry point (no link to libcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::atomic<void*> fn{nullptr};
  void* p = fn.load(std::memory_order_acquire);
  if (!p) {
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn.store(p, std::memory_order_release);
  }
  return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
}

}  // namespace

int gram_accumulate_launch(const void* X, int64_t N, int k, int64_t ldx, float* H, int64_t ldh,
                           int beta, int* err, cudaStream_t s) {
  if (ensure_smem(gram_kernel, G_SMEM, g_gram_smem_set) != cudaSuccess) return GPTQ2D_ERR_CUDA;
  const int nb = (k + GB - 1) / GB;
  GramArgs a{static_cast<const __nv_bfloat16*>(X), N, k, ldx, H, ldh, beta, err};
  // X as a 2-D tensor (features fastest) in boxes of 64 x 64, 128-byte swizzle, zero
  // fill outside; not built when there are no rows (the kernel then loads nothing)
  CUtensorMap tmap;
  memset(&tmap, 0, sizeof(tmap));
  if (N > 0) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return GPTQ2D_ERR_CUDA;
    cuuint64_t dims[2] = {(cuuint64_t)k, (cuuint64_t)N};
    cuuint64_t strides[1] = {(cuuint64_t)ldx * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)GK};
    cuuint32_t estr[2] = {1, 1};
    if (enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(X), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return GPTQ2D_ERR_CUDA;
  }
  const int blocks = g_ctas_before(nb);
  GPTQ2D_LAUNCH(KC_OTHER, s, gram_kernel<<<blocks, GTHREADS, G_SMEM, s>>>(a, tmap));
  return cudaGetLastError() == cudaSuccess ? GPTQ2D_OK : GPTQ2D_ERR_CUDA;
}

int gram_finalize_launch(float* H, int k, int64_t ldh, int64_t total_rows, double damp,
                         double* diag_sum, cudaStream_t s) {
  GPTQ2D_LAUNCH(KC_OTHER, s, gram_diag_kernel<<<1, 256, 0, s>>>(H, k, ldh, diag_sum));
  GPTQ2D_LAUNCH(KC_OTHER, s,
                gram_finalize_kernel<<<k, 256, 0, s>>>(H, k, ldh, 1.0 / (double)total_rows, damp,
                                                       diag_sum));
  return cudaGetLastError() == cudaSuccess ? GPTQ2D_OK : GPTQ2D_ERR_CUDA;
}

}  // namespace gptq2d

// The Kronecker factors from calibration activations, on the 5th-generation tensor
// cores (tcgen05): H = X^T X / N + damping, the step before the path (arxivlens
// "GPTQ-2D: Cubic-Time Two-Sided Adaptive Rounding", Analysis > Limitations and
// Future work: the fixed bases' Grams are formed and factored once).  A factor is
// the Gram of its basis; with A = X / sqrt(N) for N rows of activations X (N x k),
// H = A^T A.  The damping (a fraction of the mean diagonal added to the diagonal)
// is GPTQ's usual one; the pages give none.
//
// gram_kernel: one CTA per 128 x 128 block (bi, bj), bj <= bi, of the lower block
// triangle of H.  The block is D = X[:, I]^T X[:, J] over all rows, accumulated in
// fp32 in tensor memory by tcgen05.mma (kind::f16, bf16 operands, M = N = 128,
// K = 16 per instruction).  Both operands are chunks of 64 rows of X, and X is
// row-major (features contiguous), so A (128 features x 64 rows) and B are
// "MN-major": element (feature f, row r) of a chunk sits at byte
//     (f / 8) * 128 + (r / 8) * 2048 + (r % 8) * 16 + (f % 8) * 2
// of its shared-memory tile: 8 x 8 core matrices of 128 contiguous bytes, the
// canonical layout without swizzle of the operand descriptor (stride byte offset
// 128 between feature groups, leading byte offset 2048 between row groups).
//   warps 1..3  fill a 4-stage ring with 16-byte cp.async copies (zero past the
//               last row or column) and signal each stage's full barrier with
//               cp.async.mbarrier.arrive.noinc;
//   warp 0      allocates 128 columns of tensor memory; its elected thread waits
//               for a full stage, fences the copies into the async proxy, issues
//               the stage's four MMAs and frees the stage with tcgen05.commit on
//               its empty barrier.  A last commit signals the end.
// Then each warp reads its 32 lanes (rows) of the accumulator with tcgen05.ld and
// writes (or adds) the fp32 block into H.  Every wait is bounded (%globaltimer);
// a wait that gives up sets the error word, and the CTA still waits (bounded) for
// its copies and MMAs and frees its tensor memory before it exits.
//
// gram_diag_kernel + gram_finalize_kernel: the diagonal's sum (one CTA, fixed order:
// deterministic) into the workspace, then H <- H / N on the lower block triangle
// and H_ii += damp * mean_i(H_ii / N).
#include "common.cuh"
#include "pipeline.cuh"

namespace gptq2d {

namespace {

constexpr int GB = 128;                      // block edge (MMA M = N)
constexpr int GK = 64;                       // rows of X per stage
constexpr int GSTAGES = 4;
constexpr int GTHREADS = 128;
constexpr int GPRODUCERS = GTHREADS - 32;    // warps 1..3
constexpr int G_TILE = GB * GK * 2;          // one bf16 operand tile: 16 KB
constexpr int G_STAGE = 2 * G_TILE;          // A and B
constexpr int G_SMEM = GSTAGES * G_STAGE;
constexpr uint32_t G_SBO = 128;              // between 8-feature groups
constexpr uint32_t G_LBO = 2048;             // between 8-row groups
constexpr uint32_t G_TMEM_COLS = GB;         // fp32 accumulator: 128 lanes x 128 columns

// Shared-memory operand descriptor: start address, leading and stride byte offsets
// (all in 16-byte units), descriptor version 1, no swizzle.
__device__ __forceinline__ uint64_t g_desc(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((G_LBO >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((G_SBO >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  return d;
}

// Instruction descriptor (kind::f16): fp32 accumulator (bit 4), bf16 A (bit 7) and
// B (bit 10), both MN-major (bits 15, 16), N / 8 at bit 17, M / 16 at bit 24.
constexpr uint32_t G_IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                             ((uint32_t)(GB >> 3) << 17) | ((uint32_t)(GB >> 4) << 24);

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
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(smem_u32(bar))
               : "memory");
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

__global__ void __launch_bounds__(GTHREADS, 1) gram_kernel(GramArgs a) {
  extern __shared__ __align__(128) uint8_t gsm[];
  __shared__ __align__(8) uint64_t full_bar[GSTAGES], empty_bar[GSTAGES], done_bar;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // block (bi, bj), bj <= bi, of the lower block triangle
  const int t = blockIdx.x;
  int bi = (int)((sqrtf(8.0f * (float)t + 1.0f) - 1.0f) * 0.5f);
  while ((bi + 1) * (bi + 2) / 2 <= t) ++bi;
  while (bi * (bi + 1) / 2 > t) --bi;
  const int bj = t - bi * (bi + 1) / 2;
  const int i0 = bi * GB, j0 = bj * GB;
  const bool diag = bi == bj;

  if (tid == 0) {
    for (int s = 0; s < GSTAGES; ++s) {
      mbar_init(&full_bar[s], GPRODUCERS);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&done_bar, 1);
    abort_flag = 0;
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

  if (warp >= 1) {
    // ---- producers: chunk c into stage c % GSTAGES, after the MMAs of chunk c - GSTAGES
    const int ptid = tid - 32;
    const int pieces = (diag ? 1 : 2) * (GB * GK / 8);  // 16-byte pieces per stage
    for (int64_t c = 0; c < nchunks; ++c) {
      const int st = (int)(c % GSTAGES);
      if (c >= GSTAGES &&
          !mbar_wait(&empty_bar[st], (uint32_t)(((c / GSTAGES) - 1) & 1))) {
        atomicExch(&abort_flag, 1);
        break;
      }
      if (*(volatile int*)&abort_flag) break;
      uint8_t* sA = gsm + st * G_STAGE;
      const int64_t r0 = c * GK;
      for (int p = ptid; p < pieces; p += GPRODUCERS) {
        const int op = p / (GB * GK / 8), q = p % (GB * GK / 8);
        const int r8 = q & 7, fg = (q >> 3) & 15, rg = q >> 7;  // row % 8, feature group, row group
        const int64_t row = r0 + rg * 8 + r8;
        const int f = (op ? j0 : i0) + fg * 8;
        const bool ok = row < a.N && f < a.k;
        const void* src = ok ? (const void*)(a.X + row * a.ldx + f) : (const void*)a.X;
        cp_async16_zfill(sA + op * G_TILE + fg * 128 + rg * 2048 + r8 * 16, src, ok);
      }
      cp_async_arrive_noinc(&full_bar[st]);
    }
    cp_async_wait_group<0>();
    asm volatile("cp.async.wait_all;\n" ::: "memory");
  } else if (lane == 0) {
    // ---- MMA issuer
    for (int64_t c = 0; c < nchunks; ++c) {
      const int st = (int)(c % GSTAGES);
      if (!mbar_wait(&full_bar[st], (uint32_t)((c / GSTAGES) & 1))) {
        atomicExch(&abort_flag, 1);
        break;
      }
      if (*(volatile int*)&abort_flag) break;
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      tc_fence_after();
      const uint32_t aaddr = smem_u32(gsm + st * G_STAGE);
      const uint32_t baddr = diag ? aaddr : aaddr + G_TILE;
#pragma unroll
      for (int s16 = 0; s16 < GK / 16; ++s16)
        tc_mma(tmem, g_desc(aaddr + s16 * 2 * G_LBO), g_desc(baddr + s16 * 2 * G_LBO), G_IDESC,
               (c > 0 || s16 > 0) ? 1u : 0u);
      tc_commit(&empty_bar[st]);
    }
    tc_commit(&done_bar);  // completes once every MMA issued above has
  }
  __syncwarp();
  __syncthreads();
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
  for (int cb = 0; cb < GB / 32; ++cb) {
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
// One CTA per 128-row stripe.
__global__ void __launch_bounds__(256) gram_finalize_kernel(float* H, int k, int64_t ldh,
                                                            double inv_n, double damp,
                                                            const double* diag_sum) {
  const double shift = damp * (*diag_sum) * inv_n / (double)k;
  const int r0 = blockIdx.x * GB;
  const int cend = min(k, r0 + GB);  // end of the stripe's diagonal block
  for (int r = r0; r < min(k, r0 + GB); ++r) {
    float* hr = H + (int64_t)r * ldh;
    for (int c = threadIdx.x; c < cend; c += 256) {
      double v = (double)hr[c] * inv_n;
      if (c == r) v += shift;
      hr[c] = (float)v;
    }
  }
}

std::atomic<uint64_t> g_gram_smem_set{0};

}  // namespace

int gram_accumulate_launch(const void* X, int64_t N, int k, int64_t ldx, float* H, int64_t ldh,
                           int beta, int* err, cudaStream_t s) {
  if (ensure_smem(gram_kernel, G_SMEM, g_gram_smem_set) != cudaSuccess) return GPTQ2D_ERR_CUDA;
  const int nb = (k + GB - 1) / GB;
  GramArgs a{static_cast<const __nv_bfloat16*>(X), N, k, ldx, H, ldh, beta, err};
  const int blocks = nb * (nb + 1) / 2;
  GPTQ2D_LAUNCH(KC_OTHER, s, gram_kernel<<<blocks, GTHREADS, G_SMEM, s>>>(a));
  return cudaGetLastError() == cudaSuccess ? GPTQ2D_OK : GPTQ2D_ERR_CUDA;
}

int gram_finalize_launch(float* H, int k, int64_t ldh, int64_t total_rows, double damp,
                         double* diag_sum, cudaStream_t s) {
  const int nb = (k + GB - 1) / GB;
  GPTQ2D_LAUNCH(KC_OTHER, s, gram_diag_kernel<<<1, 256, 0, s>>>(H, k, ldh, diag_sum));
  GPTQ2D_LAUNCH(KC_OTHER, s,
                gram_finalize_kernel<<<nb, 256, 0, s>>>(H, k, ldh, 1.0 / (double)total_rows, damp,
                                                        diag_sum));
  return cudaGetLastError() == cudaSuccess ? GPTQ2D_OK : GPTQ2D_ERR_CUDA;
}

}  // namespace gptq2d

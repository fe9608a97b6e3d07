// The Kronecker factors from calibration activations, on the 5th-generation tensor
// cores (tcgen05): H = X^T X / N + damping, the step before the path (arxivlens
// "GPTQ-2D: Cubic-Time Two-Sided Adaptive Rounding", Analysis > Limitations and
// Future work: the fixed bases' Grams are formed and factored once).  A factor is
// the Gram of its basis; with A = X / sqrt(N) for N rows of activations X (N x k),
// H = A^T A.  The damping (a fraction of the mean diagonal added to the diagonal)
// is GPTQ's usual one; the pages give none.
//
// gram_kernel: persistent CTA pairs (clusters of two CTAs on neighbouring SMs, one
// pair per two SMs) over the 256 x 512 tiles (BI, C) of the lower triangle of H:
// rows 256 BI .. 256 BI + 255 and columns 512 C .. 512 C + 511, 2C <= BI; pair p
// takes tiles p, p + pairs, ... of the order below.  A tile is D = X[:, I]^T X[:, J]
// over all rows, accumulated in fp32 in tensor memory by two
// tcgen05.mma.cta_group::2 products per 16 rows (kind::f16, bf16 operands, M = N =
// 256, K = 16 per instruction), one per 256-column half, sharing A: CTA r of the
// pair holds rows 128 r .. 128 r + 127 of A (features 256 BI + 128 r ..) and
// columns 128 r .. of each half of B in its own shared memory, and receives rows
// 128 r .. of D (all 512 columns, the whole tensor memory) in its own tensor memory.
// Per 2^20 flops each SM loads 6 KB of operands from L2 (8 KB for a 256 x 256 tile,
// 12 KB for a one-SM 128 x 256 one).  Both operands are chunks of 64 rows of X, and
// X is row-major (features contiguous), so A and B are "MN-major".  Each operand
// half is two TMA boxes of 64 features x 64 rows (cp.async.bulk.tensor, 128-byte
// swizzle; zero fill past the last row or column): a box holds the rows as 128-byte
// lines, swizzled in groups of 8 lines, which is the canonical 128B-swizzled
// MN-major layout of the operand descriptor (stride byte offset 1024 between 8-row
// groups, leading byte offset 8192 between the two 64-feature boxes).  When the
// first half of B is A's own block (2C = BI) it is not loaded again; when the
// second half lies above the diagonal (2C + 1 > BI) it is neither loaded nor
// multiplied.
//   warp 1, one thread  (both CTAs) fills a 4-stage ring, chunk after chunk, tile
//                       after tile: it waits for the stage's empty barrier and
//                       issues its CTA's box loads, which complete on the
//                       LEADER's full barrier (.cta_group::2); the leader's thread
//                       first arms that barrier with both CTAs' bytes;
//   warp 0              (both CTAs) allocates all 512 columns of tensor memory for
//                       the pair.  In the leader (rank 0) one thread waits until
//                       both CTAs' epilogues have read the previous tile, then, per
//                       full stage, issues the stage's MMAs and frees the stage in
//                       both CTAs with a multicast tcgen05.commit; after a tile's
//                       last chunk a multicast commit marks the accumulator full in
//                       both CTAs;
//   warps 2..5          (both CTAs, the epilogue) wait for the full accumulator,
//                       read their 32 lanes (rows) of it with tcgen05.ld, 32 columns
//                       at a time, tell the leader it is read, and write (or add)
//                       the rows into H, each 32 x 32 chunk turned around in shared
//                       memory so that a store writes 32 consecutive floats of one
//                       row; 128 x 128 blocks above the diagonal are skipped.  The
//                       next tile's loads run meanwhile; its MMAs wait for the read.
// Every wait is bounded (%globaltimer); a wait that gives up sets the error word and
// stops the pair (H is then unspecified); the pair lets copies in flight land (a
// fixed 200 us) and exchanges the outcome across the cluster before either frees
// its tensor memory.
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

constexpr int GB = 128;                      // block edge of H's lower block triangle
constexpr int GT = 2 * GB;                   // tile edge of a CTA pair (MMA M = N)
constexpr int GK = 64;                       // rows of X per stage
constexpr int GSTAGES = 4;
constexpr int GTHREADS = 192;                // warp 0 MMA, warp 1 loads, warps 2..5 epilogue
constexpr int G_BOX = 64 * GK * 2;           // one TMA box: 64 features x 64 rows, 8 KB
constexpr int G_TILE = 2 * G_BOX;            // one CTA's operand half, 128 features: 16 KB
constexpr int G_STAGE = 3 * G_TILE;          // A half and two B halves
constexpr int G_TR = 4 * 32 * 33 * 4;       // the epilogue warps' 32 x 32 transposes
constexpr int G_SMEM = GSTAGES * G_STAGE + G_TR + 1024;  // + room to align the ring to 1024 bytes
constexpr uint32_t G_SBO = 1024;             // between 8-row groups
constexpr uint32_t G_LBO = G_BOX;            // between the two 64-feature boxes
constexpr uint32_t G_TMEM_COLS = 2 * GT;     // fp32 accumulator: 128 lanes x 512 columns
constexpr unsigned long long G_DRAIN_NS = 200000;  // copies in flight after a timeout

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

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
  return r;
}
// The shared::cluster address of `p` (a shared variable) in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
  return a;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

// One TMA box (x = feature, y = row) into this CTA's shared memory, completing on
// the mbarrier at shared::cluster address `bar` (this CTA's or its pair peer's).
// x is a multiple of 64 (a 128-byte boundary of a row).  No multicast.
__device__ __forceinline__ void tma_box(void* dst, const CUtensorMap* map, int x, int y,
                                        uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];\n" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// Instruction descriptor (kind::f16): fp32 accumulator (bit 4), bf16 A (bit 7) and
// B (bit 10), both MN-major (bits 15, 16), N / 8 at bit 17, M / 16 at bit 24; M and N
// of the pair's product.
constexpr uint32_t G_IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                             ((uint32_t)(GT >> 3) << 17) | ((uint32_t)(GT >> 4) << 24);

// Tiles of tile rows 0 .. B - 1: row BI holds the column pairs C with 2C <= BI.
__host__ __device__ inline int g_tiles_before(int B) { return (B + 1) * (B + 1) / 4; }

// Tile order.  Tile rows are taken in bands of GBAND; within a band the pairs go
// column pair by column pair (all the band's rows of pair C, then of C + 1), so the
// CTA pairs resident at one time share a few row blocks and a few column blocks of
// X and read them from L2, where a row-by-row order would stream a whole tile row's
// columns from HBM once per wave.
constexpr int GBAND = 8;

// Pair t -> tile (BI, C) for NB tile rows: rows 256 BI .., columns 512 C ...
__host__ __device__ inline void g_pair_tile(int t, int NB, int& BI, int& C) {
  // the band is the one holding t's tile row in row-by-row order
  int r = (int)(2.0f * sqrtf((float)t)) - 1;
  if (r < 0) r = 0;
  while (g_tiles_before(r + 1) <= t) ++r;
  while (r > 0 && g_tiles_before(r) > t) --r;
  const int b0 = r - r % GBAND;
  const int gb = min(GBAND, NB - b0);  // rows in the band
  int u = t - g_tiles_before(b0);
  const int c_full = b0 / 2 + 1;       // pairs C with 2C <= b0: present in every row
  if (u < c_full * gb) {
    C = u / gb;
    BI = b0 + u % gb;
    return;
  }
  u -= c_full * gb;
  for (C = c_full;; ++C) {             // pair C is in rows 2C .. b0 + gb - 1
    const int nc = b0 + gb - 2 * C;
    if (u < nc) {
      BI = 2 * C + u;
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
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
// Arrives once on the mbarrier at `bar`'s offset in both CTAs of the pair when every
// tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
      "[%0], m;\n\t}\n" ::"r"(smem_u32(bar))
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

__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];\n" ::"r"(cluster_bar)
               : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GTHREADS, 1)
    gram_kernel(GramArgs a, const __grid_constant__ CUtensorMap tmap) {
  extern __shared__ __align__(1024) uint8_t gsm_raw[];
  // the 128-byte swizzle repeats every 1024 bytes: align the ring to that (the
  // offset is the same in both CTAs, which the pair's descriptors rely on)
  uint8_t* gsm = gsm_raw + ((1024u - (smem_u32(gsm_raw) & 1023u)) & 1023u);
  float* trs = reinterpret_cast<float*>(gsm + GSTAGES * G_STAGE);
  __shared__ __align__(8) uint64_t full_bar[GSTAGES], empty_bar[GSTAGES];
  __shared__ __align__(8) uint64_t acc_full, acc_empty;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();  // 0: the leader, which issues the MMAs
  const bool leader = rank == 0;
  const int NB = (a.k + GT - 1) / GT;
  const int ntiles = g_tiles_before(NB);
  const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);
  const int64_t nchunks = (a.N + GK - 1) / GK;

  if (tid == 0) {
    for (int s = 0; s < GSTAGES; ++s) {
      mbar_init(&full_bar[s], 1);   // the leader's arm; both CTAs' bytes
      mbar_init(&empty_bar[s], 1);  // the leader's commit
    }
    mbar_init(&acc_full, 1);   // the leader's commit
    mbar_init(&acc_empty, 8);  // one lane of each epilogue warp of both CTAs
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     smem_u32(&tmem_base)),
                 "r"(G_TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers and tensor memory exist
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (warp == 1) {
    if (lane == 0) {
      // ---- producer (both CTAs): chunk g (counted over all tiles) into stage
      // g % GSTAGES, after the MMAs of chunk g - GSTAGES; its loads complete on the
      // leader's full barrier
      const uint32_t full0 = cluster_addr(&full_bar[0], 0);
      long long g = 0;
      for (int t = pair; t < ntiles && !*(volatile int*)&abort_flag; t += npairs) {
        int BI, C;
        g_pair_tile(t, NB, BI, C);
        const bool diag = 2 * C == BI;      // B0 = A
        const bool wide = 2 * C + 1 <= BI;  // B1 (the second 256 columns) below the diagonal
        const int ia = BI * GT + (int)rank * GB;
        const int jb0 = 2 * C * GT + (int)rank * GB, jb1 = jb0 + GT;
        const unsigned bytes = (1 + (diag ? 0 : 1) + (wide ? 1 : 0)) * G_TILE;  // per CTA
        for (long long c = 0; c < nchunks; ++c, ++g) {
          const int st = (int)(g % GSTAGES);
          if (g >= GSTAGES &&
              !mbar_wait(&empty_bar[st], (uint32_t)(((g / GSTAGES) - 1) & 1))) {
            atomicExch(&abort_flag, 1);
            break;
          }
          if (*(volatile int*)&abort_flag) break;
          uint8_t* sA = gsm + st * G_STAGE;
          const int y = (int)(c * GK);
          const uint32_t fb = full0 + (uint32_t)(st * sizeof(uint64_t));
          if (leader) mbar_arrive_expect_tx(&full_bar[st], 2 * bytes);
          tma_box(sA, &tmap, ia, y, fb);
          tma_box(sA + G_BOX, &tmap, ia + 64, y, fb);
          if (!diag) {
            tma_box(sA + G_TILE, &tmap, jb0, y, fb);
            tma_box(sA + G_TILE + G_BOX, &tmap, jb0 + 64, y, fb);
          }
          if (wide) {
            tma_box(sA + 2 * G_TILE, &tmap, jb1, y, fb);
            tma_box(sA + 2 * G_TILE + G_BOX, &tmap, jb1 + 64, y, fb);
          }
        }
      }
    }
  } else if (warp == 0) {
    if (lane == 0 && leader) {
      // ---- MMA issuer (one thread of the leader)
      long long g = 0;
      int it = 0;  // this pair's tile count
      for (int t = pair; t < ntiles && !*(volatile int*)&abort_flag; t += npairs, ++it) {
        int BI, C;
        g_pair_tile(t, NB, BI, C);
        const bool diag = 2 * C == BI, wide = 2 * C + 1 <= BI;
        // the accumulator was last used by tile it - 1: both epilogues must have read it
        if (it >= 1 && !mbar_wait(&acc_empty, (uint32_t)((it - 1) & 1))) {
          atomicExch(&abort_flag, 1);
          break;
        }
        tc_fence_after();
        bool ok = true;
        for (int64_t c = 0; c < nchunks; ++c, ++g) {
          const int st = (int)(g % GSTAGES);
          if (!mbar_wait(&full_bar[st], (uint32_t)((g / GSTAGES) & 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t aaddr = smem_u32(gsm + st * G_STAGE);
          const uint32_t b0addr = diag ? aaddr : aaddr + G_TILE, b1addr = aaddr + 2 * G_TILE;
          // K step s16 = rows 16 s16 .. 16 s16 + 15: two 8-row groups further (2 * SBO);
          // columns 0..255 of the tile into accumulator columns 0..255, 256..511 into
          // 256..511
#pragma unroll
          for (int s16 = 0; s16 < GK / 16; ++s16) {
            const uint64_t ad = g_desc(aaddr + s16 * 2 * G_SBO);
            const uint32_t acc = (c > 0 || s16 > 0) ? 1u : 0u;
            tc_mma(tmem, ad, g_desc(b0addr + s16 * 2 * G_SBO), G_IDESC, acc);
            if (wide) tc_mma(tmem + (uint32_t)GT, ad, g_desc(b1addr + s16 * 2 * G_SBO), G_IDESC, acc);
          }
          tc_commit_pair(&empty_bar[st]);
        }
        if (!ok) {
          atomicExch(&abort_flag, 1);
          break;
        }
        tc_commit_pair(&acc_full);  // the tile's MMAs are complete in both CTAs
      }
    }
  } else {
    // ---- epilogue (warps 2..5 of both CTAs): warp w reads tensor-memory lanes
    // 32 (w % 4) .. + 31, i.e. rows 32 (w % 4) .. of this CTA's half of the tile
    const int q = warp & 3;
    float* tr = trs + (warp - 2) * 32 * 33;
    const uint32_t empty0 = cluster_addr(&acc_empty, 0);
    // (every decision below is taken by the whole warp: tcgen05.ld is warp-wide)
    int it = 0;
    for (int t = pair; t < ntiles && !__any_sync(0xffffffffu, *(volatile int*)&abort_flag);
         t += npairs, ++it) {
      int BI, C;
      g_pair_tile(t, NB, BI, C);
      const int ia = BI * GT + (int)rank * GB, j0 = 2 * C * GT;
      // 32-column chunks in the tile's 128-blocks 4C .. 4C + 3 at or left of this
      // CTA's diagonal block 2 BI + rank (a prefix of them)
      const int ncb = min(4, 2 * BI + (int)rank - 4 * C + 1) * (GB / 32);
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full, (uint32_t)(it & 1)))) {
        if (lane == 0) atomicExch(&abort_flag, 1);
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
      for (int cb = 0; cb < ncb; ++cb) {
        uint32_t v[32];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
            "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
              "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
              "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
              "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
              "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
              "=r"(v[31])
            : "r"(tbase + (uint32_t)(cb * 32)));
        asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
        if (cb == ncb - 1) {
          // the accumulator is read: hand it back to the leader's MMA thread
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(empty0);
        }
        // turn the 32 x 32 chunk around so that each store writes 32 consecutive
        // floats of one row
#pragma unroll
        for (int c = 0; c < 32; ++c)
          tr[lane * 33 + c] = nchunks == 0 ? 0.f : __uint_as_float(v[c]);
        __syncwarp();
        const int col = j0 + cb * 32 + lane;
#pragma unroll 4
        for (int r = 0; r < 32; ++r) {
          const int gr = ia + q * 32 + r;
          if (gr < a.k && col < a.k) {
            float* h = a.H + (int64_t)gr * a.ldh + col;
            const float x = tr[r * 33 + lane];
            *h = a.beta ? *h + x : x;
          }
        }
        __syncwarp();
      }
    }
  }
  __syncwarp();
  __syncthreads();
  // a wait gave up: let the box loads and MMAs still in flight land before the
  // pair's flags are exchanged and its memory is freed
  if (*(volatile int*)&abort_flag) {
    const unsigned long long t0 = global_ns();
    while (global_ns() - t0 < G_DRAIN_NS) {
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' outcomes are final
  int peer_abort;
  asm volatile("ld.shared::cluster.u32 %0, [%1];\n"
               : "=r"(peer_abort)
               : "r"(cluster_addr(&abort_flag, rank ^ 1u)));
  if ((abort_flag || peer_abort) && tid == 0) atomicExch(a.err, 1);
  cluster_sync();  // neither CTA frees its memory while the other may read it
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;\n" ::"r"(tmem),
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
  const int NB = (k + GT - 1) / GT;
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
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int pairs = std::max(1, std::min(sms / 2, g_tiles_before(NB)));  // one per two SMs
  GPTQ2D_LAUNCH(KC_OTHER, s, gram_kernel<<<2 * pairs, GTHREADS, G_SMEM, s>>>(a, tmap));
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

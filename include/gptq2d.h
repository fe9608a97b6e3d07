/*
 * gptq2d.h -- C ABI of the B200 (sm_100a) GPTQ-2D two-sided adaptive rounding library.
 *
 * The operation (mind-verse.de "Neue Ansätze zur Effizienzsteigerung von Large
 * Language Models durch GPTQ-2D", sections "GPTQ-2D: Eine Weiterentwicklung der
 * adaptiven Rundung" and "Geometrische Grundlagen ..."; arxivlens "GPTQ-2D:
 * Cubic-Time Two-Sided Adaptive Rounding", Abstract and Analysis):
 *
 *   Round a real matrix W (m x n) onto per-row integer grids s_i * Z so that the
 *   rounding follows, entry for entry, the sequential nearest-plane (1-D GPTQ)
 *   sweep over vec(W) under the Kronecker Gram H = H_R (x) H_L, where H_L (m x m)
 *   acts on rows and H_R (n x n) on columns.  The proxy loss is
 *   L(Q) = tr(dW^T H_L dW H_R), dW = W - diag(s) Q.  Entries are rounded anti-
 *   diagonal by anti-diagonal (entry (0,0) first); every entry of one anti-
 *   diagonal is rounded in parallel; the rounding error of entry (i,j) feeds
 *   back as a rank-one, separable update built from column j of the right
 *   factor and column i of the left factor.  Total work is mn(m + n) flops.
 *
 * Conventions shared by every entry point:
 *   - Matrices are row-major; every leading dimension (ld*) counts ELEMENTS and
 *     must be >= the row length.
 *   - All data pointers are DEVICE pointers owned by the caller (except the
 *     *_host entry point, which takes host pointers).  The library never
 *     allocates or frees device memory; scratch space is the caller's
 *     workspace `ws` of at least the size returned by the matching
 *     *_workspace_size query, aligned to 256 bytes.
 *   - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is the
 *     legacy default stream).  Calls are asynchronous unless stated otherwise.
 *   - Return value: a gptq2d_status.  Arguments are checked on the host before
 *     anything is enqueued; an invalid argument returns GPTQ2D_ERR_INVALID_ARG
 *     and enqueues nothing.  A failed launch returns GPTQ2D_ERR_CUDA.  No C++
 *     exception crosses the ABI.
 *   - All floating-point arithmetic on the path is IEEE fp64.
 *   - Results are deterministic: identical inputs on the same device give a
 *     bitwise identical Q and statistics.
 *   - Every pointer a device entry point dereferences on the GPU must belong to
 *     the CURRENT device (cudaSetDevice) or be managed or page-locked host
 *     memory; another device's memory or pageable host memory is refused with
 *     GPTQ2D_ERR_INVALID_ARG before anything is enqueued.
 *   - The library keeps per-device state, created on a device's first call:
 *     internal streams and events, and the address of the no-allocation
 *     scratch.  A cudaDeviceReset invalidates that state; do not call the
 *     library on a device after resetting it in the same process.
 */
#ifndef GPTQ2D_H_
#define GPTQ2D_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GPTQ2D_OK = 0,
  GPTQ2D_ERR_INVALID_ARG = 1, /* null pointer, bad size, ld, dtype, bits or clamp */
  GPTQ2D_ERR_NOT_SPD = 2,     /* a Kronecker factor is not symmetric positive definite */
  GPTQ2D_ERR_NONFINITE = 3,   /* NaN/Inf in W or a scale <= 0 / non-finite (reported in stats) */
  GPTQ2D_ERR_WORKSPACE = 4,   /* workspace too small or misaligned */
  GPTQ2D_ERR_TIMEOUT = 5,     /* a bounded device-side wait gave up */
  GPTQ2D_ERR_CUDA = 6,        /* a CUDA runtime call or kernel launch failed */
  GPTQ2D_ERR_RANGE = 7        /* an unclamped integer does not fit its output byte (reported in
                                 stats; the byte holds the integer saturated to [-128, 127]) */
} gptq2d_status;

typedef enum {
  GPTQ2D_F32 = 0,  /* IEEE binary32 */
  GPTQ2D_BF16 = 1, /* bfloat16 */
  GPTQ2D_F64 = 2   /* IEEE binary64 */
} gptq2d_dtype;

/* Statistics written by gptq2d_quantize on the DEVICE (read them after the
 * stream has reached the end of the call). */
typedef struct {
  double proxy_loss;   /* tr(dW^T H_L dW H_R), accumulated as sum_ij d_ij^2 (y_ij - s_i q_ij)^2
                          with d_ij = M_L[i,i] M_R[j,j] and y_ij the value rounded at (i,j)
                          (the nearest-plane residual identity) */
  int64_t n_clamped;   /* entries where clamping changed rint(y/s) */
  int64_t n_near_tie;  /* entries whose y/s lies within 1e-6 of a boundary k + 1/2
                          between two admissible integers */
  int64_t n_nonfinite; /* entries with non-finite W or y, or rows with an invalid scale */
  int64_t status;      /* GPTQ2D_OK; else, in this order of precedence, GPTQ2D_ERR_TIMEOUT
                          (a bounded device wait gave up), GPTQ2D_ERR_NONFINITE
                          (n_nonfinite > 0), GPTQ2D_ERR_RANGE (n_out_of_range > 0) */
  int64_t n_out_of_range; /* clamp = 0 only: entries whose integer lies outside [-128, 127]
                             and so does not fit its int8 byte; the byte is saturated */
} gptq2d_stats;

/* Human-readable name of a status code (static string, never NULL). */
const char* gptq2d_status_string(int status);

/* Library version, (major << 16) | minor. */
int gptq2d_version(void);

/* Number of kernels this library has launched in this process so far (all
 * devices, all threads).  Lets a caller count launches inside a timed region. */
int64_t gptq2d_launch_count(void);

/* Self-check of the device-side bounded waits: runs the wait the far-field
 * kernel uses on an mbarrier that nothing completes, with a limit of `limit_ns`
 * nanoseconds (1000 .. 10^10), on `stream`, and synchronizes it (no allocation:
 * the status goes through a static device word).  Returns
 * GPTQ2D_ERR_TIMEOUT when the wait gave up as it must (the device stays usable),
 * GPTQ2D_ERR_INVALID_ARG for a limit out of range, GPTQ2D_ERR_CUDA on a launch
 * error; GPTQ2D_OK would mean the wait did not time out. */
int gptq2d_check_wait_timeout(int64_t limit_ns, void* stream);

/* Optional per-launch timing (off by default).  While enabled, every kernel the
 * library launches is bracketed by a pair of CUDA events recorded on the
 * launching stream; events are created on first use and recycled.  Kernel
 * classes: 0 factor panel (diagonal block + block-row solve), 1 factor trailing
 * update, 2 anti-diagonal tile sweep (near feedback included), 3 band products
 * to tiles two or more tiles away (far-field feedback), 4 other (conversion,
 * diagonals, statistics). */
void gptq2d_profile_enable(int on);
/* Number of recorded launches of `kernel_class` and their summed device time
 * in milliseconds (waits for the recorded events).  GPTQ2D_ERR_INVALID_ARG for
 * an unknown class. */
int gptq2d_profile_read(int kernel_class, int64_t* launches, double* total_ms);
/* Timeline of the recorded launches in enqueue order: kernel class and the
 * start / end of each launch in milliseconds after the first recorded event
 * (waits for the events).  Writes min(max_entries, recorded) entries and the
 * number recorded to *n_out. */
int gptq2d_profile_timeline(int64_t max_entries, int32_t* cls, double* start_ms, double* end_ms,
                            int64_t* n_out);
/* Forgets all recorded launches. */
void gptq2d_profile_reset(void);

/* ------------------------------------------------------------------------- */
/* Factor preparation (the fixed bases are factored once: arxivlens, Analysis  */
/* > Limitations, "fixed nonsingular basis matrices"; Future work, "Gram        */
/* factorizations").                                                           */
/* ------------------------------------------------------------------------- */

/* Bytes of workspace gptq2d_prepare needs for a k x k factor (k >= 0). */
size_t gptq2d_prepare_workspace_size(int64_t k);

/* Factor one Kronecker factor H (k x k, symmetric positive definite; only its
 * lower triangle j <= i is read) as H = M^T M with M LOWER triangular with a
 * positive diagonal (a "reverse" Cholesky factor: the last row is eliminated
 * first).  With M_L, M_R of this form, M_R (x) M_L is lower triangular in the
 * column-major order of vec(W), which is the triangular factor of the
 * index-0-first nearest-plane sweep.
 *
 *   H, h_dtype, ldh : device, k x k, GPTQ2D_F32 or GPTQ2D_F64, row-major.
 *   M, ldm          : device fp64 output, k x k row-major; the strict upper
 *                     triangle is written as exact zeros.  May not alias H.
 *   ws, ws_bytes    : device workspace, >= gptq2d_prepare_workspace_size(k).
 *   bad_pivot       : HOST pointer or NULL.  If non-NULL the call synchronizes
 *                     `stream`, writes -1 when H is positive definite, else the
 *                     0-based row index of the first pivot (in elimination
 *                     order, i.e. the largest such index) that was not
 *                     positive and finite, and returns GPTQ2D_ERR_NOT_SPD in
 *                     that case.  If NULL the call is asynchronous and a
 *                     failure is only visible through gptq2d_prepare_info.
 * k == 0 is a no-op. */
int gptq2d_prepare(const void* H, int h_dtype, int64_t k, int64_t ldh,
                   double* M, int64_t ldm, void* ws, size_t ws_bytes,
                   void* stream, int64_t* bad_pivot);

/* Both Kronecker factors in one call: H_L (m x m) -> M_L and H_R (n x n) -> M_R,
 * each exactly as gptq2d_prepare computes it.  The two factorizations run
 * concurrently on two library-internal streams that fork from `stream` and
 * join back to it, so later work on `stream` sees both factors.
 *   ws, ws_bytes : device workspace of at least 512 bytes (256-byte aligned);
 *                  bytes [0,256) hold the left pivot word, [256,512) the right.
 *   bad_pivot, which_factor : HOST pointers or NULL.  If either is non-NULL
 *                  the call synchronizes `stream`; on failure it writes the
 *                  pivot (as gptq2d_prepare does) and 0 for H_L / 1 for H_R
 *                  (H_L reported first) and returns GPTQ2D_ERR_NOT_SPD; else
 *                  it writes -1 to both.  If both are NULL the call is
 *                  asynchronous; gptq2d_prepare_info(ws) and
 *                  gptq2d_prepare_info(ws + 256) read the two pivot words.
 * m == 0 or n == 0 skips that factor. */
int gptq2d_prepare_pair(const void* H_L, int64_t m, int64_t ldhl,
                        const void* H_R, int64_t n, int64_t ldhr, int h_dtype,
                        double* M_L, int64_t ldml, double* M_R, int64_t ldmr,
                        void* ws, size_t ws_bytes, void* stream,
                        int64_t* bad_pivot, int* which_factor);

/* Reads the pivot word a previous asynchronous gptq2d_prepare left in `ws`
 * (synchronizes `stream`).  Writes -1 or the failing pivot to *bad_pivot and
 * returns GPTQ2D_OK or GPTQ2D_ERR_NOT_SPD. */
int gptq2d_prepare_info(const void* ws, void* stream, int64_t* bad_pivot);

/* ------------------------------------------------------------------------- */
/* The Kronecker factors from calibration activations (the step before the     */
/* path; arxivlens "GPTQ-2D: Cubic-Time Two-Sided Adaptive Rounding",          */
/* Analysis > Limitations and Future work: fixed bases whose Grams are formed   */
/* and factored once).  A factor is the Gram of its basis A = X / sqrt(N):      */
/* H = X^T X / N for N rows of activations X, plus GPTQ's usual damping of the  */
/* diagonal (a reading: the pages give none).  Runs on the tcgen05 tensor cores */
/* with bf16 operands and fp32 accumulation.                                    */
/* ------------------------------------------------------------------------- */

/* Bytes of workspace the Gram calls need (a diagonal sum and an error word). */
size_t gptq2d_gram_workspace_size(void);

/* Accumulate the Gram of a batch of activation rows.
 *   X, x_dtype, rows, k, ldx : DEVICE, rows x k, GPTQ2D_BF16 only, row-major;
 *                              k and ldx multiples of 8, X 16-byte aligned;
 *                              rows <= 2^31 - 1 (split larger batches into calls).
 *   H, ldh                   : DEVICE fp32 k x k.  The lower 128-block triangle
 *                              (every 128 x 128 block on or below the diagonal, so
 *                              every j <= i and a few j > i near the diagonal) is
 *                              written: accumulate = 0 sets it to X^T X and clears
 *                              the workspace's error word (a new Gram);
 *                              accumulate = 1 adds X^T X.  Other entries are untouched.
 *   ws, ws_bytes             : DEVICE workspace >= gptq2d_gram_workspace_size(),
 *                              256-byte aligned, kept from the first batch to finalize.
 * Products of bf16 values are exact in fp32; the sums are fp32 (tensor-core order).
 * rows == 0 with accumulate = 0 writes zeros.  k == 0 is a no-op.  A bounded
 * device-side wait that gives up sets the error word (read by gptq2d_gram_finalize
 * when it is given a HOST status pointer); H is then unspecified. */
int gptq2d_gram_accumulate(const void* X, int x_dtype, int64_t rows, int64_t k, int64_t ldx,
                           float* H, int64_t ldh, int accumulate, void* ws, size_t ws_bytes,
                           void* stream);

/* Finish a Gram: H <- H / total_rows on the lower 128-block triangle, then
 * H_ii += damp * mean_i(H_ii), the mean of the scaled diagonal (damp >= 0; GPTQ's
 * usual value is 0.01).  The result is ready for gptq2d_prepare (which reads only
 * the lower triangle).  status (HOST, may be NULL): if non-NULL the call
 * synchronizes `stream` and returns GPTQ2D_ERR_TIMEOUT if a bounded wait of an
 * accumulate call gave up, else GPTQ2D_OK (also written to *status). */
int gptq2d_gram_finalize(float* H, int64_t k, int64_t ldh, int64_t total_rows, double damp,
                         void* ws, size_t ws_bytes, void* stream, int* status);

/* ------------------------------------------------------------------------- */
/* Hessians with more than two Kronecker factors (arxivlens "GPTQ-2D: Cubic-   */
/* Time Two-Sided Adaptive Rounding", Abstract: the algorithm extends to any   */
/* number of Kronecker factors).                                               */
/* ------------------------------------------------------------------------- */

/* Largest number of factors gptq2d_kron_factor combines. */
#define GPTQ2D_MAX_KRON_FACTORS 8

/* Kronecker product of lower factors.  A k-way tensor W of shape (m_1, ..., m_k),
 * row-major (C order), under H = H_1 (x) H_2 (x) ... (x) H_k (H_j acting on mode
 * j) is rounded as the m_1 x (m_2 ... m_k) matrix with H_L = H_1 and
 * H_R = H_2 (x) ... (x) H_k.  The reverse Cholesky factor of that H_R is
 * M_R = M_2 (x) ... (x) M_k (M_j from gptq2d_prepare of H_j), which this call
 * forms; gptq2d_quantize with M_L = M_1 then gives the k-way rounding: every
 * entry sees only its dominated orthant {i' : i'_j <= i_j for all j}, and the
 * result equals the 1-D sweep over the tensor's coordinates in any order that
 * respects that product order.  Scales are per index of mode 1.
 *
 *   nf           : number of factors, 1 <= nf <= GPTQ2D_MAX_KRON_FACTORS.
 *   M, dims, ldm : HOST arrays of nf entries.  M[f] is a DEVICE pointer to a
 *                  dims[f] x dims[f] fp64 lower factor, row-major with leading
 *                  dimension ldm[f] >= dims[f]; its strict upper triangle is not read.
 *   out, ldo     : DEVICE fp64 output, n x n row-major, n = prod dims <= 2^20,
 *                  ldo >= n.  With r = (r_1, ..., r_nf) and c the mixed-radix digits
 *                  of the row and column (last factor fastest),
 *                  out[r][c] = prod_f M[f][r_f][c_f] when every c_f <= r_f, and an
 *                  exact zero otherwise.  Must not overlap a factor.
 * n == 0 (a zero dimension) writes nothing and returns GPTQ2D_OK. */
int gptq2d_kron_factor(int nf, const double* const* M, const int64_t* dims, const int64_t* ldm,
                       double* out, int64_t ldo, void* stream);

/* An order of trailing modes for gptq2d_quantize_kron (host only, no GPU work).  The
 * k-way rounding depends only on each entry's dominated orthant, so reordering modes
 * 2..k permutes the result and nothing else: a caller may permute W's trailing modes
 * (and the factors) by `order`, round, and permute Q back.  The subset of modes whose
 * sizes multiply to the largest of 64, 32, 16, 8 goes last (the inner group), the
 * others keep their order in front; the given order is kept when it already reaches
 * that size.
 *   nf, dims : HOST, the trailing modes' sizes (1 <= nf <= GPTQ2D_MAX_KRON_FACTORS).
 *   order    : HOST, nf entries: order[p] = the given index of the mode placed p-th.
 * Returns the inner size m_in the reordered modes give (8, 16, 32 or 64), or 0 when
 * no subset reaches 8 (order is then the identity); -1 for invalid arguments. */
int gptq2d_per_mode_order(int nf, const int64_t* dims, int* order);

/* Bytes of device workspace gptq2d_quantize_kron needs for an m x prod(dims)
 * rounding with these trailing modes; 0 when the per-mode path does not apply
 * (see gptq2d_quantize_kron) or the arguments are out of range. */
size_t gptq2d_quantize_kron_workspace_size(int64_t m, int nf, const int64_t* dims);

/* The k-way rounding of gptq2d_kron_factor + gptq2d_quantize with the right factor
 * kept per mode: M_R = M[0] (x) ... (x) M[nf-1] is never formed, and the right-hand
 * error feedback is applied mode by mode (the separable feedback of the abstract's
 * extension to several Kronecker factors).  With the normalised factors
 * Lh_f = diag(M_f)^-1 M_f, the last factors whose sizes multiply to m_in form the
 * inner group, where m_in is the largest product of a suffix of dims that divides 64
 * (the tile width); the path applies when m_in >= 8.  Then a 64-column tile holds
 * a = 64 / m_in consecutive indices of the outer modes, every block of the
 * normalised right factor between two tiles is (an a x a block of the outer
 * factors' product) (x) (the inner factor), and a tile's right feedback from
 * tiles two or more to its left costs a multiply-adds per entry per source tile
 * instead of a 64 x 64 x 64 product; the inner factor is applied once per tile.
 * Memory: the factors as given plus O(m n); no n x n matrix.
 *   W, w_dtype, m, ldw     : as gptq2d_quantize, W is m x n with n = prod dims
 *                            (the tensor of shape (m, dims...) in C order).
 *   M_L, ldl               : the mode-1 factor, as gptq2d_quantize's M_L.
 *   nf, M, dims, ldm       : HOST arrays of nf <= GPTQ2D_MAX_KRON_FACTORS entries;
 *                            M[f] a DEVICE fp64 lower factor of dims[f] x dims[f]
 *                            (gptq2d_prepare of H_{f+2}), leading dimension
 *                            ldm[f] >= dims[f]; strict upper triangles not read.
 *                            prod dims <= 2^20.
 *   scales, bits, clamp, Q, ldq, stats : as gptq2d_quantize.
 *   ws, ws_bytes           : DEVICE workspace >= gptq2d_quantize_kron_workspace_size,
 *                            256-byte aligned.
 * The result is gptq2d_quantize's with M_R = gptq2d_kron_factor(M) up to the
 * rounding order (the factor entries are formed as products of normalised entries):
 * Q may differ only at near-ties.  Returns GPTQ2D_ERR_INVALID_ARG when the path does
 * not apply (m_in < 8, e.g. a last mode of 3 or 100); the dense
 * gptq2d_kron_factor + gptq2d_quantize route handles every shape. */
int gptq2d_quantize_kron(const void* W, int w_dtype, int64_t m, int64_t ldw, const double* M_L,
                         int64_t ldl, int nf, const double* const* M, const int64_t* dims,
                         const int64_t* ldm, const float* scales, int bits, int clamp, int8_t* Q,
                         int64_t ldq, gptq2d_stats* stats, void* ws, size_t ws_bytes,
                         void* stream);

/* ------------------------------------------------------------------------- */
/* Rounding                                                                    */
/* ------------------------------------------------------------------------- */

/* Bytes of workspace gptq2d_quantize needs for an m x n problem. */
size_t gptq2d_quantize_workspace_size(int64_t m, int64_t n);

/* GPTQ-2D rounding of W under H_R (x) H_L, given the factors from
 * gptq2d_prepare (arxivlens Abstract: same rounding as the quartic Kronecker
 * feedback, cubic work, anti-diagonals in parallel).
 *
 *   W, w_dtype, ldw : device, m x n, GPTQ2D_F32, GPTQ2D_BF16 or GPTQ2D_F64.
 *   M_L, ldl        : device fp64, m x m lower factor of H_L (upper triangle ignored).
 *   M_R, ldr        : device fp64, n x n lower factor of H_R (upper triangle ignored).
 *   scales          : device fp32 [m], grid step of each row; must be finite and > 0.
 *   bits, clamp     : grid [-2^(bits-1), 2^(bits-1)-1] when clamp = 1 (2 <= bits <= 8);
 *                     clamp = 0 rounds to any integer; an integer outside [-128, 127]
 *                     is stored saturated, counted in stats->n_out_of_range and
 *                     reported as GPTQ2D_ERR_RANGE in stats->status (the rounding
 *                     itself, and every later entry, use the true integer).
 *   Q, ldq          : device int8 output, m x n.
 *   stats           : device pointer to one gptq2d_stats, written at the end.
 *   ws, ws_bytes    : device workspace, >= gptq2d_quantize_workspace_size(m, n).
 *
 * Rounding: q = clamp(rint(y / s_i)) with rint = round half to even; the error
 * fed back is W_ij - s_i q_ij with the clamped q.  Entries whose y is not
 * finite are counted in stats->n_nonfinite and set stats->status.
 * m == 0 or n == 0 writes zero statistics and returns GPTQ2D_OK. */
int gptq2d_quantize(const void* W, int w_dtype, int64_t m, int64_t n, int64_t ldw,
                    const double* M_L, int64_t ldl, const double* M_R, int64_t ldr,
                    const float* scales, int bits, int clamp,
                    int8_t* Q, int64_t ldq, gptq2d_stats* stats,
                    void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------- */
/* The proxy loss of a given rounding, and of round-to-nearest (the baseline   */
/* the pages compare GPTQ-2D with: arxivlens, Abstract; mind-verse.de,         */
/* "GPTQ-2D: Eine Weiterentwicklung der adaptiven Rundung")                    */
/* ------------------------------------------------------------------------- */

/* Bytes of workspace gptq2d_proxy_loss needs for an m x n problem (two tile-padded
 * fp64 m x n buffers and one double per 64 x 64 tile); 0 for sizes out of range. */
size_t gptq2d_proxy_loss_workspace_size(int64_t m, int64_t n);

/* L(Q) = tr(dW^T H_L dW H_R) = || M_L dW M_R^T ||_F^2 with dW = W - diag(s) Q, written
 * to *loss (one DEVICE double) on `stream`.
 *
 *   W, w_dtype, ldw : device, m x n, GPTQ2D_F32, GPTQ2D_BF16 or GPTQ2D_F64.
 *   Q, ldq          : device int8, m x n (row stride ldq >= n): the integers to score, e.g.
 *                     gptq2d_quantize's output; NULL scores round-to-nearest,
 *                     q = clamp(rint(W / s)) on the grid of bits / clamp (as in
 *                     gptq2d_quantize).
 *   scales          : device fp32 [m], the per-row grid steps.
 *   M_L, M_R        : the lower factors (M^T M = H) as for gptq2d_quantize; only their
 *                     lower triangles are read.
 *   loss            : device pointer to one double.
 *   ws, ws_bytes    : device workspace, >= gptq2d_proxy_loss_workspace_size(m, n),
 *                     256-byte aligned.
 *
 * This is a full quadratic form (two triangular matrix products, about mn(m + n)
 * flops on the FP64 tensor cores, as much work as the rounding), so the rounding does
 * not compute it: its own loss comes from the nearest-plane residual identity in
 * gptq2d_stats.  Deterministic (fixed reduction order).  m == 0 or n == 0 writes 0. */
int gptq2d_proxy_loss(const void* W, int w_dtype, int64_t m, int64_t n, int64_t ldw,
                      const int8_t* Q, int64_t ldq, const float* scales, int bits, int clamp,
                      const double* M_L, int64_t ldl, const double* M_R, int64_t ldr,
                      double* loss, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------- */
/* Grid variants (the pages fix only a 4-bit integer grid: mind-verse.de       */
/* "Neue Ansätze ...", section "Quantisierung von Large Language Models";      */
/* these are GPTQ's usual variants of it)                                      */
/* ------------------------------------------------------------------------- */

/* The grid of gptq2d_quantize_grid.  Entry (i, j) lies in column group
 * g = j / group_size (g = 0 when group_size is 0) and rounds to s q with
 * s = scales[i * ld_scales + g] and q an integer:
 *   symmetric (zeros NULL): q in [-2^(bits-1), 2^(bits-1) - 1];
 *   asymmetric: z = zeros[i * ld_scales + g], code c = q + z in [0, 2^bits - 1],
 *     the value s (c - z): q in [-z, 2^bits - 1 - z].  With an integer z the
 *     nearest code to y / s + z is the nearest admissible q to y / s plus z, so
 *     the rounding is the same one-coordinate nearest-plane step;
 *   clamp = 0: any integer q (symmetric grid only: zero points need clamp = 1,
 *     since an unclamped code need not fit its byte).
 * Storage of Q:
 *   packed = 0: one byte per entry, row stride ldq >= n bytes: int8 q on the
 *     symmetric grid, uint8 code c on the asymmetric one;
 *   packed = 1 (bits <= 4, clamp = 1): two entries per byte, row stride
 *     ldq >= ceil(n / 2) bytes; byte k of a row holds the code of column 2k in
 *     its low nibble and that of column 2k + 1 in its high nibble (0 past the
 *     last column); the code is q + 2^(bits-1) (offset binary) on the symmetric
 *     grid and c on the asymmetric one. */
typedef struct {
  int bits;               /* 2..8 */
  int clamp;              /* 0 or 1 */
  int64_t group_size;     /* 0: one scale per row; else a multiple of 8, or >= n (one group) */
  const float* scales;    /* DEVICE fp32, m rows of ceil(n / group_size) groups (1 if
                             group_size is 0), row stride ld_scales; finite and > 0 */
  int64_t ld_scales;      /* >= groups per row */
  const uint8_t* zeros;   /* DEVICE, NULL for the symmetric grid; else integer zero points
                             in the layout of scales (requires clamp = 1) */
  int packed;             /* 0 or 1 (see above) */
} gptq2d_grid;

/* gptq2d_quantize with a grid variant: group-wise scales, integer zero points,
 * packed 4-bit output.  Arguments other than `grid` (a HOST pointer), Q (bytes)
 * and ldq (bytes) are those of gptq2d_quantize, as are the rounding, the
 * statistics (the loss uses each entry's own step) and the determinism; with
 * group_size 0, zeros NULL and packed 0 the result is gptq2d_quantize's.
 * A scale that is not finite and > 0 is counted once per group in
 * stats->n_nonfinite. */
int gptq2d_quantize_grid(const void* W, int w_dtype, int64_t m, int64_t n, int64_t ldw,
                         const double* M_L, int64_t ldl, const double* M_R, int64_t ldr,
                         const gptq2d_grid* grid, void* Q, int64_t ldq, gptq2d_stats* stats,
                         void* ws, size_t ws_bytes, void* stream);

/* gptq2d_quantize_kron on a grid variant: the k-way rounding with the right factor
 * kept per mode (arguments, applicability and workspace as gptq2d_quantize_kron)
 * on group-wise scales, integer zero points or packed 4-bit output (grid, Q and ldq
 * as gptq2d_quantize_grid; scale groups run along the flattened trailing modes). */
int gptq2d_quantize_kron_grid(const void* W, int w_dtype, int64_t m, int64_t ldw,
                              const double* M_L, int64_t ldl, int nf, const double* const* M,
                              const int64_t* dims, const int64_t* ldm, const gptq2d_grid* grid,
                              void* Q, int64_t ldq, gptq2d_stats* stats, void* ws, size_t ws_bytes,
                              void* stream);

/* ------------------------------------------------------------------------- */
/* A block of layers (the pages quantize whole models, block by block:         */
/* arxivlens, Abstract, Llama-3.1-70B-Instruct on one GPU)                     */
/* ------------------------------------------------------------------------- */

/* One linear layer of a block.  All pointers are DEVICE pointers except that the
 * grid is held by value (its scales and zeros are device pointers).
 *   W, w_dtype, m, n, ldw  : as in gptq2d_quantize.
 *   H_L, ldhl, H_R, ldhr, h_dtype : the layer's Grams (m x m and n x n, GPTQ2D_F32
 *                            or GPTQ2D_F64, lower triangles read), e.g. from
 *                            gptq2d_gram_accumulate / gptq2d_gram_finalize.
 *   grid                   : as in gptq2d_quantize_grid.
 *   Q, ldq, stats          : outputs, as in gptq2d_quantize_grid. */
typedef struct {
  const void* W;
  int w_dtype;
  int64_t m, n, ldw;
  const void* H_L;
  int64_t ldhl;
  const void* H_R;
  int64_t ldhr;
  int h_dtype;
  gptq2d_grid grid;
  void* Q;
  int64_t ldq;
  gptq2d_stats* stats;
} gptq2d_layer;

/* Bytes of device workspace gptq2d_quantize_block needs for these layers (two factor
 * slots for the largest layer, 512 bytes per layer, one rounding workspace for the
 * largest layer); 0 for invalid sizes. */
size_t gptq2d_block_workspace_size(const gptq2d_layer* layers, int nl);

/* Factors and rounds nl layers, overlapping the factor preparation of layer i + 1
 * with the rounding of layer i: the factors go to library-internal streams of their
 * own, the roundings run one after another in the given order (largest first keeps
 * the GPU busiest), and each of the two factor slots is reused once the layer that
 * read it is rounded.  Every layer's result is exactly what gptq2d_prepare_pair +
 * gptq2d_quantize_grid give it alone.  Waits for `stream` before it starts; later
 * work on `stream` sees every output.  Synchronizes `stream` at the end to read
 * the factors' pivot words: returns GPTQ2D_ERR_NOT_SPD for the first layer with a
 * factor that is not positive definite (*bad_layer, *bad_pivot and *which_factor,
 * each a HOST pointer or NULL, receive the layer, the pivot and 0 for H_L / 1 for
 * H_R; -1 when all are positive definite); that layer's rounding ran on a failed
 * factor and its statistics are not meaningful.  Arguments of every layer are
 * checked before anything is enqueued. */
int gptq2d_quantize_block(const gptq2d_layer* layers, int nl, void* ws, size_t ws_bytes,
                          void* stream, int64_t* bad_layer, int64_t* bad_pivot,
                          int* which_factor);

/* ------------------------------------------------------------------------- */
/* Rounding without any allocation                                             */
/* (no counterpart in the GPTQ-2D pages: an interface for callers of this     */
/* library that may not allocate device memory)                               */
/* ------------------------------------------------------------------------- */

/* Capacity of the library's static rounding scratch: 48 MiB on every device
 * that loads the library, held until the process exits. */
#define GPTQ2D_NOALLOC_SCRATCH_BYTES (48u << 20)

/* gptq2d_quantize without a workspace argument, for callers that cannot call
 * cudaMalloc (a framework that owns all device memory through its own pool,
 * a service that forbids allocation once it is running, or a caller that
 * cannot afford cudaMalloc's implicit device synchronization).  Arguments,
 * rounding and statistics are exactly those of gptq2d_quantize; the scratch is
 * a static device array inside the library instead.
 *
 *   - Size limit: the problem must satisfy
 *     gptq2d_quantize_workspace_size(m, n) <= GPTQ2D_NOALLOC_SCRATCH_BYTES
 *     (for example 1024 x 1024, which needs 40 MiB); larger problems return
 *     GPTQ2D_ERR_WORKSPACE and enqueue nothing.
 *   - Sharing: every call uses the same array.  Calls whose work overlaps on
 *     the GPU (two streams, two threads) race on it; order them.  Each call
 *     clears what must start at zero, so leftovers of earlier calls are harmless.
 *   - Set-up: the first call on each device looks up the array's device
 *     address (cudaGetSymbolAddress) with that device current; make that first
 *     call before any stream capture.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
int gptq2d_quantize_noalloc(const void* W, int w_dtype, int64_t m, int64_t n, int64_t ldw,
                            const double* M_L, int64_t ldl, const double* M_R, int64_t ldr,
                            const float* scales, int bits, int clamp,
                            int8_t* Q, int64_t ldq, gptq2d_stats* stats, void* stream);

/* ------------------------------------------------------------------------- */
/* End to end from host memory                                                 */
/* ------------------------------------------------------------------------- */

/* Bytes of DEVICE workspace gptq2d_round_host needs. */
size_t gptq2d_round_host_workspace_size(int64_t m, int64_t n, int w_dtype, int h_dtype);

/* The whole path from HOST buffers: copies W (m x n, dense), the lower
 * triangles of H_L (m x m) and H_R (n x n) (each 64-row block up to the end of
 * its diagonal block; the rest is never read) and scales to the device
 * workspace, factors both Kronecker factors, rounds, and copies Q (m x n int8,
 * dense) and the statistics back.  The copies go over an internal stream, the
 * larger Gram first, then the other, then W: each factorization starts when its
 * Gram is in, and the later copies run under it.  Host buffers should be pinned for asynchronous
 * copies.  Synchronizes `stream` before returning.  Returns GPTQ2D_ERR_NOT_SPD if either factor is
 * not positive definite (the left factor is checked first; *bad_pivot, if
 * non-NULL, receives the pivot, and *which_factor, if non-NULL, 0 for H_L and
 * 1 for H_R), else the statistics' status. */
int gptq2d_round_host(const void* W, int w_dtype, int64_t m, int64_t n,
                      const void* H_L, const void* H_R, int h_dtype,
                      const float* scales, int bits, int clamp,
                      int8_t* Q, gptq2d_stats* stats,
                      void* ws, size_t ws_bytes, void* stream,
                      int64_t* bad_pivot, int* which_factor);

#ifdef __cplusplus
}
#endif

#endif /* GPTQ2D_H_ */

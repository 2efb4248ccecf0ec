/*
 * shampoo.h -- C ABI of libshampoo: one blocked-Shampoo optimizer step over
 * 3-D stacks of equal-size preconditioner blocks, on one NVIDIA B200
 * (sm_100a).
 *
 * Sources cited below:
 *   [DASH]  "DASH: Faster Shampoo via Batched Block Preconditioning and
 *           Efficient Inverse-Root Solvers" (Modoranu et al.), section summary.
 *   [3D]    "3D-Shampoo optimizer" README, "Hyperparameters".
 *   [Notes] "Shampoo" notes (speedrun/shampoo).
 *
 * Conventions shared by every call
 *   - Matrices are row-major float32.  A "stack" is `count` matrices stored
 *     contiguously: matrix b, row i, column j is at base[(b*rows + i)*cols + j].
 *   - All device memory is owned by the caller.  The library never allocates
 *     device memory; calls that need scratch space take a caller-provided
 *     `workspace` whose size is given by the matching *_workspace_bytes query.
 *     Device pointers must be 16-byte aligned; workspaces 256-byte aligned.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *     call only enqueues work on it and returns without synchronising, except
 *     where stated.  Calls that share a workspace must be ordered on one
 *     stream.
 *   - Arrays of pointers (`const float* const* grads` ...) are HOST arrays
 *     whose elements are DEVICE pointers.
 *   - Invalid arguments are reported before anything is enqueued; the call
 *     then returns a nonzero shp_status and shampoo_last_error() describes it.
 *     Numerical failure of an iteration is not an error: it is written to the
 *     per-matrix status array of the root calls (shampoo_inv_root and its
 *     _static, _warm and _evd forms).
 */
#ifndef SHAMPOO_H
#define SHAMPOO_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SHP_API __attribute__((visibility("default")))
#else
#define SHP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t shp_status;
#define SHP_OK 0
#define SHP_ERR_INVALID_ARG 1 /* null pointer, bad enum, bad scalar */
#define SHP_ERR_SHAPE 2       /* size out of range or inconsistent */
#define SHP_ERR_WORKSPACE 3   /* workspace smaller than the query says */
#define SHP_ERR_CUDA 4        /* a CUDA runtime call failed */
#define SHP_ERR_UNSUPPORTED 5 /* valid request this build does not implement */

/* Inverse-root methods ([DASH] §3 and appendix A). */
#define SHP_METHOD_NDB 0  /* Newton-DB, two chained inverse-square-root calls */
#define SHP_METHOD_CN 1   /* coupled Newton ([Notes] "Roots on idle CPUs") */
#define SHP_METHOD_CHEB 2 /* Chebyshev polynomial, optimised matrix Clenshaw */

/* Arithmetic of the tensor-core contractions; accumulation is always FP32.
 * FP32 is emulated by three fp16 passes (hi*hi, lo*hi, hi*lo) on a hi/lo
 * split of both operands scaled by a power of two per matrix
 * (x * 2^e = hi + lo * 2^-11, about 22 significant bits). */
#define SHP_DTYPE_FP32 0
#define SHP_DTYPE_TF32 1
#define SHP_DTYPE_FP16 2
#define SHP_DTYPE_BF16 3

/* Scaling before the iterations ([DASH] §3 Matrix scaling). */
#define SHP_SCALE_FROBENIUS 0
#define SHP_SCALE_POWER 1 /* multi-power-iteration, largest Rayleigh quotient */

/* Grafting ([DASH] §2; [3D] graft_type). */
#define SHP_GRAFT_NONE 0
#define SHP_GRAFT_SGD 1
#define SHP_GRAFT_ADAGRAD 2
#define SHP_GRAFT_ADAM 3

/* Bits of the per-matrix status written by shampoo_inv_root. */
#define SHP_ROOT_NONFINITE 1
#define SHP_ROOT_UNCONVERGED 2 /* shampoo_inv_root_evd: sweep limit reached */

/* Dampening heuristics of shampoo_inv_root_evd ([DASH] B.1, B.2). */
#define SHP_EVD_CORRECTED 0
#define SHP_EVD_SHIFTED_RELU 1
#define SHP_EVD_ABS_ADD 2
#define SHP_EVD_SHMP 3

/* Largest side shampoo_inv_root_evd accepts (shared-memory resident). */
#define SHP_EVD_MAX_N 128

/* Columns of the block table (shampoo_plan_tables). */
#define SHP_BLOCK_FIELDS 13
/* layer, block_row, block_col, row0, col0, rows, cols,
 * g_bucket, g_index, l_bucket, l_index, r_bucket, r_index */

/* Largest matrix side accepted by the root and GEMM calls. */
#define SHP_MAX_N 8192

typedef struct shp_plan shp_plan; /* opaque host object owned by the library */

/* Message describing the last failed call of this thread ("" if none). */
SHP_API const char* shampoo_last_error(void);

/* Library version, major*10000 + minor*100 + patch. */
SHP_API int32_t shampoo_version(void);

/* Number of kernels this library has launched in this process (all threads,
 * all devices); a diagnostic for counting launches inside a timed region. */
SHP_API uint64_t shampoo_launch_count(void);

/* Reads and clears the device error word (bit 0: a kernel gave up waiting on
 * an on-chip barrier after ~2 s and skipped its stores).  Synchronises the
 * device.  *out = 0 means no kernel reported an error. */
SHP_API shp_status shampoo_device_error(int32_t* out);

/* ---------------------------------------------------------------------
 * a1  Partition + stack   ([3D] block_size; [DASH] §1, §4 Blocking Strategy)
 *
 * Every layer (rows x cols) is cut into blocks: a dimension larger than
 * block_size becomes floor(d/B) blocks of B plus one remainder block of
 * d mod B; a dimension <= B (or B == 0) stays whole.  Gradient blocks are
 * bucketed by (rows, cols); left factors (rows x rows) and right factors
 * (cols x cols) are bucketed by size n.  Order inside a bucket: layers in
 * input order; inside a layer, all left factors (blocks row-major) and then
 * all right factors; buckets in order of first appearance.  For a 32000 x
 * 2048 layer at B = 1024 this gives gradient stacks (62,1024,1024) and
 * (2,256,1024) and factor stacks (126,1024,1024) and (2,256,256) ([DASH] §4).
 * ------------------------------------------------------------------- */

/* Plans the partition of n_layers layers (host only, no CUDA call).
 * rows/cols: host arrays [n_layers], each in [1, 2^30).  block_size >= 0.
 * Block sides above SHP_MAX_N are rejected (SHP_ERR_SHAPE).
 * On success *plan_out owns host memory; free it with shampoo_plan_destroy. */
SHP_API shp_status shampoo_plan_create(const int32_t* rows, const int32_t* cols, int32_t n_layers, int32_t block_size,
                               shp_plan** plan_out);

/* shampoo_plan_create with one-sided layers and flags.
 * left_only: NULL, or host [n_layers]; nonzero makes that layer one-sided
 *   ([Notes] "Roots on idle CPUs": embedding, softmax and very large
 *   layers are preconditioned on one side only, L^(-1/2) G): its blocks get
 *   left factors only (r_bucket = r_index = -1), and its gradient and factor
 *   buckets are keyed by that side as well, so no stack mixes one- and
 *   two-sided blocks.  shampoo_update_stats then updates only L for them,
 *   shampoo_precondition computes D = X_L G, and the caller takes inverse
 *   square roots (p = 2) of the buckets shampoo_plan_factor_sides marks 1.
 *   A layer whose large side is its rows is passed transposed.
 * flags: SHP_PLAN_LAYERWISE stacks per layer: gradient buckets are keyed by
 *   (layer, rows, cols) and factor buckets by (layer, n), the "layerwise"
 *   stacking the DASH paper compares with its GPU-level stacking (§4
 *   Blocking Strategy); the order inside a bucket is unchanged.  The paper
 *   has no flag: it names the two variants.  Unknown bits return
 *   SHP_ERR_INVALID_ARG.
 * NULL left_only with flags 0 is shampoo_plan_create. */
#define SHP_PLAN_LAYERWISE 1
SHP_API shp_status shampoo_plan_create_ex(const int32_t* rows, const int32_t* cols, const int32_t* left_only,
                                          int32_t n_layers, int32_t block_size, int32_t flags, shp_plan** plan_out);

/* Side of every factor bucket: host [n_fbuckets], 0 for factors of
 * two-sided blocks, 1 for the left factors of one-sided blocks. */
SHP_API shp_status shampoo_plan_factor_sides(const shp_plan* plan, int32_t* sides);
SHP_API void shampoo_plan_destroy(shp_plan* plan);

/* Table sizes: number of blocks, of gradient buckets, of factor buckets, and
 * the bytes of device memory shampoo_plan_bind needs.  Any output may be NULL. */
SHP_API shp_status shampoo_plan_sizes(const shp_plan* plan, int32_t* n_blocks, int32_t* n_gbuckets, int32_t* n_fbuckets,
                              size_t* device_bytes);

/* Copies the plan's tables into host arrays:
 *   blocks   [n_blocks][SHP_BLOCK_FIELDS]  (columns listed above)
 *   gbuckets [n_gbuckets][3]  rows, cols, count
 *   fbuckets [n_fbuckets][2]  n, count
 * Any output may be NULL. */
SHP_API shp_status shampoo_plan_tables(const shp_plan* plan, int32_t* blocks, int32_t* gbuckets, int32_t* fbuckets);

/* Uploads the plan's index tables into caller-owned device memory
 * (>= device_bytes from shampoo_plan_sizes) and remembers that pointer; every
 * later call with this plan reads the tables from there, so the buffer must
 * outlive the plan's use.  Asynchronous on `stream` (from host memory the
 * plan owns). */
SHP_API shp_status shampoo_plan_bind(shp_plan* plan, void* device_tables, size_t bytes, void* stream);

/* Gathers every layer's gradient blocks into the gradient stacks.
 * grads:    [n_layers] device pointers, layer l is rows_l x cols_l row-major.
 * g_stacks: [n_gbuckets] device pointers, bucket k is (count, rows, cols).
 * Requires a bound plan. */
SHP_API shp_status shampoo_stack_blocks(const shp_plan* plan, const float* const* grads, float* const* g_stacks,
                                void* stream);

/* ---------------------------------------------------------------------
 * a2  Statistics update   ([DASH] §2 Preliminaries on Shampoo)
 *   L <- beta2 L + alpha G G^T,   R <- beta2 R + alpha G^T G
 * for every gradient block G (alpha = 1 - beta2 gives the moving average,
 * alpha = 1 with beta2 = 1 the AdaGrad sums).  f_stacks: [n_fbuckets] device
 * pointers to the factor stacks (count, n, n), updated in place.
 * dtype: SHP_DTYPE_* of the G G^T contractions.
 * ------------------------------------------------------------------- */
SHP_API size_t shampoo_update_stats_workspace_bytes(const shp_plan* plan, int32_t dtype);
SHP_API shp_status shampoo_update_stats(const shp_plan* plan, const float* const* g_stacks, float* const* f_stacks,
                                float beta2, float alpha, int32_t dtype, void* workspace, size_t ws_bytes,
                                void* stream);

/* ---------------------------------------------------------------------
 * a3-a6  Damping, scaling and the inverse p-th root   ([DASH] §3, A.1-A.3)
 *
 * For each of the `count` n x n matrices L_b of the stack A, with the root
 * power p in {2, 4, 8} (4: the inverse fourth root of Shampoo; 2: the
 * square-root power the "Shampoo" notes report as often effective):
 *   NDB : s = scale of L + eps I; Y0 = (L + eps I)/s; call 1 (iters
 *         iterations of Y <- Y T, Z <- T Z, T = (3I - Z Y)/2, the first one
 *         closed-form) gives Y ~ (A/s)^(1/2), Z ~ (A/s)^(-1/2); each further
 *         call runs on the previous Y and halves the power: log2(p) calls
 *         give Z ~ (A/s)^(-1/p); X = s^(-1/p) Z.
 *   CN  : s = scale of L + eps I; M0 = (L + eps I)/s, X0 = I;
 *         T = ((p+1)I - M)/p, X <- X T, M <- T^p M (T^p by squarings);
 *         X = s^(-1/p) X.
 *   CHEB: s = scale of L (undamped); S = 2 L/s - I; X = s^(-1/p) sum_k c_k
 *         T_k(S) with c_k interpolating x^(-1/p) at the iters+1 Chebyshev
 *         nodes of [eps, 1 + eps] (iters = degree d, d-1 matmuls).
 * Any other p returns SHP_ERR_UNSUPPORTED.
 * scaling: SHP_SCALE_FROBENIUS (s = ||.||_F) or SHP_SCALE_POWER (s = largest
 *   Rayleigh quotient after pi_iters steps of power iteration from the
 *   pi_vectors start vectors in pi_starts, device [pi_vectors][n] float32,
 *   run with fp16 operands and fp32 accumulation).
 * Outputs: X_out (count, n, n) float32; scale_out [count] the s used;
 *   status_out [count] (0 ok, SHP_ROOT_NONFINITE if X has a NaN/Inf).
 * Sizes: 1 <= n <= SHP_MAX_N, n % 4 == 0; 1 <= count <= 65535 (32767 for
 *   the two-problem launches of NDB/CN); 1 <= iters <= 1000.
 * A and X_out may not overlap the workspace.
 * ------------------------------------------------------------------- */
SHP_API size_t shampoo_inv_root_workspace_bytes(int32_t count, int32_t n, int32_t method, int32_t dtype, int32_t scaling,
                                        int32_t pi_vectors);
SHP_API shp_status shampoo_inv_root(const float* A, int32_t count, int32_t n, float eps, int32_t p, int32_t method,
                            int32_t iters, int32_t dtype, int32_t scaling, int32_t pi_vectors, int32_t pi_iters,
                            const float* pi_starts, float* X_out, float* scale_out, int32_t* status_out,
                            void* workspace, size_t ws_bytes, void* stream);

/* Bytes of device scratch behind shampoo_inv_root_static (32 MiB). */
#define SHP_STATIC_SCRATCH_BYTES (32u << 20)

/* shampoo_inv_root for callers that cannot allocate device memory.  The
 * pages have no counterpart: this is a property of the library, not of the
 * method.  Callers that cannot call cudaMalloc at the moment they need a
 * root -- code running while a CUDA graph is captured, allocator or
 * memory-pool callbacks that must not re-enter the allocator, programs with
 * a fixed preallocated memory budget -- get the same result as
 * shampoo_inv_root (same arguments minus the workspace) with the scratch
 * taken from a device array of SHP_STATIC_SCRATCH_BYTES that the library
 * defines.  Every GPU that loads this part of the library holds that array
 * until the process exits.
 *   - Rejects (SHP_ERR_WORKSPACE, nothing enqueued) any request whose
 *     shampoo_inv_root_workspace_bytes exceeds SHP_STATIC_SCRATCH_BYTES.
 *   - The first call on a device looks up the array's device address with
 *     that device current; make that first call before any stream capture.
 *   - Calls no cudaMalloc / cudaFree and no allocating library routine.
 *   - All calls on a device share the one array and it keeps the last
 *     call's contents (everything a call reads is written by that call
 *     first); calls whose work overlaps on the GPU (different streams
 *     without ordering) race on it. */
SHP_API shp_status shampoo_inv_root_static(const float* A, int32_t count, int32_t n, float eps, int32_t p,
                                           int32_t method, int32_t iters, int32_t dtype, int32_t scaling,
                                           int32_t pi_vectors, int32_t pi_iters, const float* pi_starts,
                                           float* X_out, float* scale_out, int32_t* status_out, void* stream);

/* Coupled Newton warm-started from a previous root   ([Notes] "Roots on
 * idle CPUs": coupled Newton, started from the previous root)
 *   A = L + eps I; X0 = X0_in; M0 = X0^p A (X0^p by squarings);
 *   T = ((p+1)I - M)/p, X <- X T, M <- T^p M for iters iterations; no
 *   scaling and no final multiplier.  When X0 commutes with L (shares its
 *   eigenvectors) the iterates converge to A^(-1/p); a root of an earlier L
 *   does not commute with the new one, and the iteration then settles at
 *   X0 (X0^p A)^(-1/p), a fixed point of its own, within a few iterations.
 *   It converges when the eigenvalues of M0 lie in (0, p + 1).  Chaining
 *   it step after step from its own results compounds that error (it
 *   diverged within 4 to 6 chained refreshes of a growing Gram factor,
 *   in float64 as well), so a cold root has to be taken now and then. 
 * A, X0: device (count, n, n) float32, row-major, 16-byte aligned; X0 is
 *   read once at the start, so X_out may be X0 (in-place refresh).
 * X_out: device (count, n, n) float32; status_out [count] as for
 *   shampoo_inv_root.  p in {2, 4, 8}; dtype as for shampoo_inv_root;
 *   1 <= iters <= 1000; sizes as for shampoo_inv_root.
 * Products: 4 iters for p = 4 (3 iters + 1 for p = 2, 5 iters + 3 for
 *   p = 8), each a (count, n, n) GEMM.
 * Errors (nothing enqueued): SHP_ERR_INVALID_ARG for NULL pointers, bad
 *   dtype, eps < 0 or not finite, misaligned pointers; SHP_ERR_SHAPE for
 *   n or count out of range; SHP_ERR_UNSUPPORTED for other p;
 *   SHP_ERR_WORKSPACE when ws_bytes is below
 *   shampoo_inv_root_warm_workspace_bytes (0 for invalid sizes). */
SHP_API size_t shampoo_inv_root_warm_workspace_bytes(int32_t count, int32_t n, int32_t dtype);
SHP_API shp_status shampoo_inv_root_warm(const float* A, const float* X0, int32_t count, int32_t n, float eps,
                                         int32_t p, int32_t iters, int32_t dtype, float* X_out,
                                         int32_t* status_out, void* workspace, size_t ws_bytes, void* stream);

/* Inverse p-th roots by eigendecomposition   ([DASH] §3 (EVD, the
 * reference method), B.1 regularisation for EVD, B.2 dampening heuristics)
 *   mu, Q = eig(L + eps I) (L symmetrised as (L + L^T)/2), lambda = mu - eps
 *   (the corrected spectrum), X = Q diag(f) Q^T with, by heuristic:
 *     SHP_EVD_CORRECTED     f = (max(lambda, 0) + eps)^(-1/p)
 *     SHP_EVD_SHIFTED_RELU  f = (lambda - eps)^(-1/p) where lambda > eps,
 *                           else 0 (a rank-r_eps inverse)
 *     SHP_EVD_ABS_ADD       f = (|lambda| + eps)^(-1/p)
 *     SHP_EVD_SHMP          f = (mu - min(min_i mu_i, 0) + eps)^(-1/p), the
 *                           Distributed Shampoo adjustment (eps added twice)
 * The eigensolver is cyclic two-sided Jacobi, one CTA per matrix held in
 * shared memory (the matrix rotated in float64, the eigenvectors
 * accumulated in float32), until a sweep leaves every off-diagonal
 * entry below 2^-21 sqrt(|a_pp a_qq|) (at most 40 sweeps; otherwise the
 * matrix's status gets SHP_ROOT_UNCONVERGED).
 * A: device (count, n, n) float32 row-major; X_out: same shape (may be A);
 * eig_out: NULL or device (count, n) float32, lambda ascending per matrix;
 * status_out: device [count] int32, SHP_ROOT_* bits in bits 0-7
 *   (SHP_ROOT_NONFINITE also when A itself holds a NaN / Inf) and the
 *   number of sweeps taken in bits 8-15 (the final sweep, which rotates
 *   nothing, included).
 * Sizes: 1 <= n <= SHP_EVD_MAX_N (any n), count >= 1; p in {2, 4, 8}.
 * No workspace.  Errors (nothing enqueued): SHP_ERR_INVALID_ARG (NULL
 * pointer, bad heuristic, eps < 0 or not finite), SHP_ERR_SHAPE (n, count),
 * SHP_ERR_UNSUPPORTED (other p), SHP_ERR_CUDA (launch failure). */
SHP_API shp_status shampoo_inv_root_evd(const float* A, int32_t count, int32_t n, float eps, int32_t p,
                                        int32_t heuristic, float* X_out, float* eig_out, int32_t* status_out,
                                        void* stream);

/* ---------------------------------------------------------------------
 * a7  Two-sided preconditioning   ([DASH] §2)
 *   D_b = X_L(b) G_b X_R(b)   for every gradient block b
 * roots:  [n_fbuckets] device pointers to the root stacks (count, n, n), in
 *         the same bucket order and index as the factor stacks.
 * d_stacks: [n_gbuckets] outputs, shaped like the gradient stacks.
 * block_dnorm2: device [n_blocks] float, overwritten with ||D_b||_F^2 in
 *         stack order (gradient bucket 0 first, then bucket 1, ...).
 * ------------------------------------------------------------------- */
SHP_API size_t shampoo_precondition_workspace_bytes(const shp_plan* plan, int32_t dtype);
SHP_API shp_status shampoo_precondition(const shp_plan* plan, const float* const* roots, const float* const* g_stacks,
                                float* const* d_stacks, float* block_dnorm2, int32_t dtype, void* workspace,
                                size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------
 * a8  Grafting + parameter update   ([DASH] §2 grafting; [3D] graft_type,
 *     weight_decay; [Notes] "Roots on idle CPUs")
 *   graft direction g: SGD: G;  AdaGrad: G/(sqrt(v)+eps) with v += G^2;
 *   Adam: m <- b1 m + (1-b1) G, v <- b2 v + (1-b2) G^2,
 *         g = (m/(1-b1^step)) / (sqrt(v/(1-b2^step)) + eps)
 *   rho = ||g||_F / ||D||_F per layer (graft_per_block = 0) or per block (1);
 *   rho = 0 where ||D|| = 0; SHP_GRAFT_NONE uses rho = 1.
 *   W <- W - lr rho D - lr weight_decay W
 * W, G, m, v: [n_layers] device pointers in layer layout (m, v may be NULL
 * when the graft does not use them).  d_stacks / block_dnorm2 as produced by
 * shampoo_precondition.  step >= 1.
 * ------------------------------------------------------------------- */
SHP_API size_t shampoo_graft_step_workspace_bytes(const shp_plan* plan);
SHP_API shp_status shampoo_graft_step(const shp_plan* plan, float* const* W, const float* const* G,
                              const float* const* d_stacks, const float* block_dnorm2, float* const* m,
                              float* const* v, int32_t graft, float lr, float beta1, float beta2, float eps,
                              float weight_decay, int32_t step, int32_t graft_per_block, void* workspace,
                              size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SHAMPOO_H */

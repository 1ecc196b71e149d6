/*
 * muon.h -- C ABI of libmuon.so: the Muon optimizer step on one NVIDIA B200
 * (sm_100a), with standard and Gram Newton-Schulz orthogonalisation, NorMuon
 * row normalisation and Dion3 fractional row selection.
 *
 * Source of the mathematics: "Dion3: Full-stack orthogonal updates"
 * (arXiv 2608.11612), web summary. Each entry point below names the section
 * or equation it computes.
 *
 * Conventions for every entry point
 * ---------------------------------
 * - Matrices are row-major with leading dimension = cols (no padding) unless
 *   stated. "rows" are rows as stored.
 * - Every data pointer is CUDA device memory owned by the caller (for example
 *   from PyTorch). The library never allocates device memory: entry points
 *   that need scratch space take a caller-owned workspace `ws` of at least the
 *   size reported by the matching *_workspace_size function. The workspace
 *   must stay untouched by the caller while work queued on `stream` uses it.
 * - All work is queued asynchronously on `stream` (a cudaStream_t; NULL is the
 *   legacy default stream). Host-side argument errors are returned before any
 *   work is queued; nothing is launched in that case.
 * - Pointers to matrices must be 16-byte aligned (MUON_ERR_ALIGN otherwise).
 * - Errors found on the device (a non-finite norm, a non-finite polar output
 *   such as an fp16 overflow, a device wait that ran out)
 *   cannot be returned synchronously: they are written, as a muon_status
 *   value, to a device int32 status word. The status word is `dev_status`
 *   where a call takes one and it is non-NULL, else the first 4 bytes of the
 *   workspace (cleared to MUON_OK at the start of every call that uses it).
 *   The first error written wins. Read it after synchronising the stream.
 * - No exceptions cross this boundary and nothing calls exit() or abort().
 * - Not thread-safe for concurrent calls that share a workspace.
 */
#ifndef MUON_H_
#define MUON_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MUON_OK = 0,
  MUON_ERR_INVALID_ARG = 1,  /* NULL pointer, bad count, bad parameter value */
  MUON_ERR_SHAPE = 2,        /* rows/cols/k out of range                      */
  MUON_ERR_DTYPE = 3,        /* unsupported dtype combination                 */
  MUON_ERR_ALIGN = 4,        /* a matrix pointer is not 16-byte aligned       */
  MUON_ERR_WORKSPACE = 5,    /* workspace NULL or smaller than required       */
  MUON_ERR_CUDA = 6,         /* a CUDA runtime/driver call failed             */
  MUON_ERR_NONFINITE = 7,    /* (device) a norm, ratio or output not finite   */
  MUON_ERR_TIMEOUT = 8,      /* (device) a bounded device wait ran out        */
  MUON_ERR_UNSUPPORTED = 9   /* valid request this build cannot serve         */
} muon_status;

typedef enum { MUON_F32 = 0, MUON_BF16 = 1, MUON_F16 = 2 } muon_dtype;

/* Dion3 row-selection key: the page's rule is the l1 norm of each momentum
 * row ("3. Dion3 Update Rule", Algorithm 4, step 1); l2 is an option. */
typedef enum { MUON_NORM_L1 = 0, MUON_NORM_L2 = 1 } muon_norm;

#define MUON_MAX_T 16

/* Newton-Schulz parameters ("Standard Newton-Schulz"; "1. Gram Newton-Schulz",
 * Theorem 2 and Algorithm 3).
 *   T            iterations, 1..MUON_MAX_T
 *   coeffs[t]    (a_t, b_t, c_t) of p_t(x) = a x + b x^3 + c x^5, t = 0..T-1
 *   norm_eps     X_0 = X / (||X||_F + norm_eps)   (1e-7 in the workloads)
 *   gram         0: standard iteration, 1: Gram iteration
 *   restart_at   Gram only: restart before step restart_at (3 on the page),
 *                0 = never (the page's naive version)
 *   compute      operand type of the GEMM chain: MUON_BF16 or MUON_F16
 *                (tensor cores, fp32 accumulation), or MUON_F32 (fp32 FFMA,
 *                no TF32) */
typedef struct {
  int32_t T;
  float coeffs[MUON_MAX_T][3];
  float norm_eps;
  int32_t gram;
  int32_t restart_at;
  muon_dtype compute;
} muon_ns_params;

/* One weight matrix and its optimizer state, all fp32, rows x cols row-major.
 * v (NorMuon second moments, one per stored row) may be NULL when NorMuon is
 * off. G is read only. */
typedef struct {
  float* W;
  float* M;
  const float* G;
  float* v;
  int64_t rows;
  int64_t cols;
} muon_matrix;

/* Parameters of one optimizer step.
 *   mu, lr       momentum and learning rate (Eq. (1)); lr is used verbatim
 *                (the page's transfer eta' = eta / sqrt(f) is the caller's)
 *   ns           orthogonalisation parameters
 *   normuon      0/1: apply NorMuon (Eq. (2)) with beta2 and normuon_eps
 *   dion3        0: plain Muon, M <- mu M + G.
 *                1: Dion3 (Algorithm 4): M <- M + G, select
 *                k = ceil(frac_num/frac_den * rows) rows by select_norm,
 *                orthogonalise M[S,:], update W[S,:], then M[S,:] <- mu M[S,:]
 *   dev_status   optional device int32 for deferred device errors (see top);
 *                the library does not clear it: the caller sets it to
 *                MUON_OK before the steps it wants to check */
typedef struct {
  float mu;
  float lr;
  muon_ns_params ns;
  int32_t normuon;
  float beta2;
  float normuon_eps;
  int32_t dion3;
  int32_t frac_num;
  int32_t frac_den;
  muon_norm select_norm;
  int32_t* dev_status;
} muon_params;

/* Bound, in nanoseconds, of every device-side wait inside the library's
 * kernels (default 2e9 = 2 s; 0 restores the default). A wait that runs out
 * records MUON_ERR_TIMEOUT in the status word and the kernel returns early
 * (its outputs are then unspecified) instead of hanging the GPU. Process-wide;
 * applies to launches queued after the call. */
void muon_set_wait_timeout_ns(uint64_t ns);

/* Tensor-core GEMM form used by the Newton-Schulz chain: 1 (default) runs
 * each 256x256 tile on a pair of CTAs (tcgen05 cta_group::2, a cluster of two
 * SMs, each loading half of the operands); 0 runs 128x256 tiles on single
 * CTAs. Both give the same results up to fp32 summation order. Process-wide;
 * applies to launches queued after the call. */
void muon_set_gemm_cta_pair(int32_t enable);

/* How the Newton-Schulz chain's products are launched: 0 (default) one
 * persistent launch per product (all shape groups of the call together); 1
 * the whole chain as one fused persistent launch (or a few, when its
 * products need more kernel parameters than one launch holds), in which the
 * tiles of a product wait, matrix by matrix, until the previous product of
 * the same matrix is in memory (completion counters in the workspace, each
 * wait bounded like every other device wait), so that products of different
 * matrices overlap and no launch boundary separates dependent products.
 * Both give the same results up to fp32 summation order. Process-wide;
 * applies to calls made after it. */
void muon_set_gemm_chain(int32_t enable);

/* Human-readable name of a status value (static string, never NULL). */
const char* muon_status_str(muon_status s);

/* k = ceil(f_num / f_den * n) in exact integer arithmetic ("3. Dion3 Update
 * Rule", Algorithm 4: k = ceil(f n)). Returns -1 if f_num <= 0, f_den <= 0,
 * f_num > f_den or n < 0. */
int64_t muon_rows_for_fraction(int64_t n, int32_t f_num, int32_t f_den);

/* Fill *p with the workload defaults: T = 5, every (a,b,c) =
 * (3.4445, -4.7750, 2.0315), norm_eps = 1e-7, gram = 0, restart_at = 3,
 * compute = MUON_BF16. */
void muon_ns_params_default(muon_ns_params* p);

/* Workspace bytes needed by ns_polar / gram_ns_polar for one rows x cols
 * matrix with parameters p (returns 0 for invalid arguments). Includes the
 * fp32 scratch that X X^T products of a short, wide matrix use to split
 * their inner dimension across the GPU; that part depends on the SM count
 * of the current device, so query with the device that will run the call
 * current. */
size_t muon_ns_workspace_size(int64_t rows, int64_t cols, const muon_ns_params* p);

/* O ~= polar(X) by T quintic Newton-Schulz steps ("Standard Newton-Schulz";
 * Definition 1 gives polar). X is rows x cols of x_dtype (F32 or BF16); O is
 * rows x cols of o_dtype (F32 or BF16), caller-owned, may not alias X. A tall
 * matrix (rows > cols) is orthogonalised in its transposed (wide) form, since
 * polar(X^T) = polar(X)^T; no copy is made. If p->gram is 1 this runs the
 * Gram iteration instead (see gram_ns_polar). ws: see muon_ns_workspace_size.
 * Deferred errors go to the first 4 bytes of ws. */
muon_status ns_polar(const void* X, muon_dtype x_dtype, void* O, muon_dtype o_dtype,
                     int64_t rows, int64_t cols, const muon_ns_params* p,
                     void* ws, size_t ws_bytes, void* stream);

/* O ~= polar(X) by the Gram Newton-Schulz iteration ("1. Gram Newton-Schulz",
 * Theorem 2; restart of Algorithm 3 at p->restart_at, 0 = naive version):
 * R_0 = X X^T; Z_t = a I + b R + c R^2; Q_t = Q_{t-1} Z_t; R_t = Z_t R Z_t;
 * restart X <- Q X, R <- X X^T, Q <- I; output Q_T X. Same arguments as
 * ns_polar; p->gram is ignored. p->compute selects the operand type (F16 is
 * the page's choice for the Gram matrices; BF16 also allowed; F32 = FFMA). */
muon_status gram_ns_polar(const void* X, muon_dtype x_dtype, void* O, muon_dtype o_dtype,
                          int64_t rows, int64_t cols, const muon_ns_params* p,
                          void* ws, size_t ws_bytes, void* stream);

/* NorMuon row scales ("NorMuon Variant", Eq. (2)) for the k x m matrix O
 * (o_dtype F32 or BF16). For each row i, with j = rows ? rows[i] : i:
 *   r_i = sum_c O[i,c]^2;  v[j] <- beta2 v[j] + (1 - beta2) r_i / m;
 *   d_i = 1 / (sqrt(v[j]) + eps);
 *   row_scale_out[i] = d_i * sqrt(sum_i r_i) / sqrt(sum_i d_i^2 r_i)
 * (0 for every row when the denominator is 0), so that the NorMuon update is
 * W[j,:] -= lr * row_scale_out[i] * O[i,:]. v is updated in place (fp32);
 * rows (device int32, k entries, distinct) may be NULL. No workspace needed;
 * row_scale_out (k floats) is also used as scratch. Arithmetic in fp32 with
 * fp64 cross-row sums. Deferred errors go to dev_status if non-NULL. */
muon_status normuon_scale(const void* O, muon_dtype o_dtype, int64_t k, int64_t m,
                          float* v, const int32_t* rows, float beta2, float eps,
                          float* row_scale_out, int32_t* dev_status, void* stream);

/* Workspace bytes for select_rows on an n-row matrix. */
size_t muon_select_workspace_size(int64_t n);

/* Dion3 selection ("3. Dion3 Update Rule", Algorithm 4, step 1): the k rows
 * of the n x m fp32 matrix M with the largest key, key_i = sum_j |M_ij|
 * (MUON_NORM_L1) or sum_j M_ij^2 (MUON_NORM_L2), summed in fp64. Ties go to
 * the lower row index. idx_out (device int32, k entries) receives the chosen
 * rows in ascending order. 1 <= k <= n. */
muon_status select_rows(const float* M, int64_t n, int64_t m, int64_t k, muon_norm norm,
                        int32_t* idx_out, void* ws, size_t ws_bytes, void* stream);

/* select_rows without a workspace, for callers that cannot allocate device
 * memory when they need a selection (a pool that is already carved up, a
 * runtime that forbids cudaMalloc after start-up because it can synchronise
 * the device, a C host without an allocator). The page has no counterpart:
 * this is a packaging of select_rows, same arguments and same result,
 * minus the workspace, plus an optional dev_status for deferred errors.
 *
 * Scratch: a fixed 1 MiB + 256 B __device__ array inside libmuon.so, held by
 * every GPU that loads the library until the process exits. n is limited to
 * 65536 rows (MUON_ERR_SHAPE beyond). The first call on each device looks up
 * the array's device address (cudaGetSymbolAddress) with that device
 * current; make that first call before any stream capture. The address is
 * kept for the life of the process, so do not use the library across a
 * cudaDeviceReset; devices with index 64 or above are rejected
 * (MUON_ERR_INVALID_ARG). All calls share the one array: calls whose work
 * overlaps on the GPU (different streams, or different host threads, without
 * ordering between them) race and give wrong indices; calls ordered on one
 * stream are safe. Allocates nothing.
 *
 * dev_status, as for muon_step, is the caller's: the library never clears it,
 * so the caller sets it to MUON_OK before the calls it wants to check (an
 * error left from an earlier call stays, the first error written wins). With
 * dev_status NULL, device-side errors (a non-finite row key) are not
 * reported. */
muon_status select_rows_noalloc(const float* M, int64_t n, int64_t m, int64_t k, muon_norm norm,
                                int32_t* idx_out, int32_t* dev_status, void* stream);

/* Workspace bytes for muon_step (and muon_orthogonalize) over mats[0..count)
 * with parameters p (0 for invalid arguments). Only the shapes and p matter:
 * the data pointers of mats are not read and may be NULL. Like
 * muon_ns_workspace_size, query with the device that will run the step
 * current. */
size_t muon_workspace_size(const muon_matrix* mats, int32_t count, const muon_params* p);

/* One optimizer step over count independent matrices (host array mats):
 * "Muon Update Rule", Eq. (1) -- M <- mu M + G, W <- W - lr polar(M) -- with
 * polar by standard or Gram Newton-Schulz, optional NorMuon (Eq. (2)) and
 * optional Dion3 (Algorithm 4). W, M and v are updated in place. Matrices of
 * the same shape are batched into shared launches. */
muon_status muon_step(const muon_matrix* mats, int32_t count, const muon_params* p,
                      void* ws, size_t ws_bytes, void* stream);

/* The step in three parts, for callers that hold each matrix as row shards
 * on several GPUs and move whole matrices to an owner GPU for the
 * orthogonalisation ("4. Megabatched Communication": pack the local momentum
 * shards into one all-to-all, assemble, orthogonalise as a batch, scatter
 * back). On one GPU, muon_momentum, then muon_orthogonalize, then
 * muon_apply_update give the same W, M and v as muon_step, bit for bit.
 *
 * muon_momentum: the first line of Eq. (1) on every matrix, elementwise:
 * M <- mu M + G (one rounding, as a fused multiply-add), or M <- M + G when
 * p->dion3 (Algorithm 4 keeps the decay for the error feedback). Reads M and
 * G, writes M; W and v are not touched. No workspace, no deferred errors
 * (a non-finite M surfaces in muon_orthogonalize). */
muon_status muon_momentum(const muon_matrix* mats, int32_t count, const muon_params* p, void* stream);

/* muon_orthogonalize: everything between the momentum and the weight update,
 * on the momentum M as given (muon_momentum already applied): the Frobenius
 * scale, the Dion3 selection (p->dion3), the Newton-Schulz chain and NorMuon
 * (p->normuon, Eq. (2); v is updated in place for the orthogonalised rows).
 * W and G are not read (they may be NULL). Outputs, per matrix i, all
 * caller-owned device memory:
 *   O[i]          rows x cols, ld = cols, 16-byte aligned, element type of
 *                 p->ns.compute (bf16, fp16 or fp32): the orthogonalised row
 *                 at its stored row position; zero rows where not selected
 *   row_scale[i]  rows floats: the update's row scale (NorMuon's scale, or 1);
 *                 0 where not selected
 *   selected[i]   rows int32 (needed when p->dion3, else may be NULL): 1 for
 *                 the selected rows, 0 elsewhere
 * so that the update is W[r,:] -= lr * row_scale[i][r] * O[i][r,:].
 * ws / ws_bytes: as for muon_step (muon_workspace_size). Deferred errors (a
 * non-finite norm or NorMuon ratio, a bounded wait that ran out) go to
 * p->dev_status, else to the first 4 workspace bytes, as for muon_step. */
muon_status muon_orthogonalize(const muon_matrix* mats, int32_t count, const muon_params* p,
                               void* const* O, float* const* row_scale, int32_t* const* selected,
                               void* ws, size_t ws_bytes, void* stream);

/* muon_apply_update: the weight update of Eq. (1) from muon_orthogonalize's
 * outputs (or row shards of them: mats[i] may be a row range of a matrix
 * whose O, row_scale and selected rows are passed for the same range):
 * W[r,:] <- W[r,:] - lr * row_scale[i][r] * O[i][r,:] (one rounding), and,
 * when p->dion3, M[r,:] <- mu M[r,:] for the selected rows, whose W alone
 * changes. Reads O, row_scale, selected; G and v are not touched. A
 * non-finite value of O is reported as MUON_ERR_NONFINITE to p->dev_status
 * when it is set (no workspace, so nothing is reported without it). */
muon_status muon_apply_update(const muon_matrix* mats, int32_t count, const muon_params* p,
                              const void* const* O, const float* const* row_scale,
                              const int32_t* const* selected, void* stream);

/* Per-phase timing and work accounting of one step (muon_step_profiled).
 * Times are CUDA-event milliseconds on the call's stream. FLOPs count the
 * Newton-Schulz products: ns_flops counts a product with a symmetric result
 * as one triangle (the page's FLOP analysis for symmetric GEMMs),
 * ns_flops_dense counts every product as 2 m n k, ns_flops_executed is the
 * tensor-core work actually issued (whole tiles of 128 or 256 rows by 128
 * or 256 columns, diagonal tiles in full). Bytes are the compulsory HBM bytes of the memory-bound phases. */
typedef struct {
  float ms_total;
  float ms_prologue;   /* momentum, norms, selection, operand casts */
  float ms_ns;         /* the Newton-Schulz GEMM chain              */
  float ms_normuon;    /* NorMuon row statistics and scales         */
  float ms_update;     /* weight update (and Dion3 momentum decay)  */
  int64_t kernel_launches;
  int64_t gemm_launches;
  double ns_flops;
  double ns_flops_dense;
  double ns_flops_executed;
  double bytes_prologue;
  double bytes_update;
} muon_step_profile;

/* muon_step with per-phase CUDA events: same arguments and effects, plus
 * *prof filled on return. Synchronises `stream` before returning (so it is
 * for measurement, not the training loop). prof must be non-NULL. */
muon_status muon_step_profiled(const muon_matrix* mats, int32_t count, const muon_params* p,
                               void* ws, size_t ws_bytes, void* stream, muon_step_profile* prof);

/* muon_step that also records five caller-owned CUDA events (cudaEvent_t
 * handles, created by the caller with timing enabled) on `stream` at the phase
 * boundaries: events[0] before the first kernel, events[1] before the
 * Newton-Schulz chain, events[2] after it, events[3] after the NorMuon row
 * scales, events[4] after the weight update. Same arguments and effects as
 * muon_step otherwise; it does not synchronise, so a timed loop can measure
 * each phase of the very steps it times (cudaEventElapsedTime after the
 * loop). events must be non-NULL and hold five valid events. */
muon_status muon_step_events(const muon_matrix* mats, int32_t count, const muon_params* p,
                             void* ws, size_t ws_bytes, void* stream, void* const* events);

/* Number of kernels this library has queued from the calling thread since it
 * was loaded (monotonic; for counting launches inside a timed region). */
int64_t muon_kernel_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* MUON_H_ */

// Per-row, memory-bound kernels of the Muon step (declarations shared by
// rowops.cu and the step/NS orchestration).
#pragma once

#include "internal.h"

namespace muon {

// One matrix in a batched row launch. Every field a kernel does not use may
// be NULL/0. "task" rows are the rows a launch walks: all stored rows, or the
// k selected rows of a Dion3 step.
struct RowMat {
  float* W;
  float* M;
  const void* src;        // generic source rows (cast / sum-of-squares kernels)
  const float* G;
  float* v;               // NorMuon second moments, one per stored row
  void* X;                // operand rows (written by casts, read as O by updates)
  const int32_t* idx;     // task row -> stored row (NULL = identity)
  float* rscale;          // per task row: NorMuon r_i, then the row scale
  double* rsum;           // per stored row: sum of squares (fp64)
  double* rkey;           // per stored row: selection key (fp64)
  const float* mult;      // cast multiplier (device scalar) or NULL
  void* out;              // scatter_rows: destination rows (ld = cols), at stored row positions
  float* out_scale;       // scatter_rows: per stored row, the update's row scale
  int32_t* out_flag;      // scatter_rows: per stored row, 1 where the row was orthogonalised
  const int32_t* flag;    // update: per task row, 0 = skip the row (NULL = every row)
  float kappa;            // extra cast multiplier (host constant)
  int64_t rows, cols, ldx;
  int32_t ntask;          // rows walked by this launch for this matrix
  int32_t task_begin;     // prefix of ntask over the launch's matrices
};

// Matrices per row-kernel launch: the whole Llama-7B-shaped set (192) in one
// launch; the table travels in the kernel parameters (at most 32764 bytes).
constexpr int kMaxRowMats = 200;

struct RowLaunch {
  RowMat m[kMaxRowMats];
  int count;
  int total_tasks;
  float mu, lr;
  int mode;               // kernel-specific variant
  int key_l2;             // selection key: 0 = l1, 1 = sum of squares
  int* status;
};

static_assert(sizeof(RowLaunch) <= 32764, "row-kernel parameters are limited to 32764 bytes");

// Kernel variants of momentum_rows.
enum MomentumMode { MOM_MUON = 0, MOM_DION3 = 1 };

// M <- mu*M + G (MOM_MUON, one fmaf rounding) or M <- M + G (MOM_DION3);
// optionally X <- cast(M) (unscaled); rsum <- sum M^2, rkey <- l1 or l2 key.
muon_status launch_momentum_rows(RowLaunch& L, Op xt, cudaStream_t s);
// rsum[row] = sum_c src[row,c]^2 and rkey[row] = l1 or l2 key (if non-NULL)
// for src of type st (F32 or BF16).
muon_status launch_row_stats(RowLaunch& L, Op st, cudaStream_t s);
// X[i,:] = cast(src[idx[i],:] * (*mult) * kappa), src of type st.
muon_status launch_cast_rows(RowLaunch& L, Op st, Op xt, cudaStream_t s);
// rscale[i] = sum_c O[i,c]^2 (fp32), O = X of type ot.
muon_status launch_normuon_rows(RowLaunch& L, Op ot, cudaStream_t s);
// W[idx[i],:] -= lr * (rscale ? rscale[i] : 1) * O[i,:]; mode 1: M[idx[i],:] *= mu.
// Rows whose flag is 0 are skipped.
muon_status launch_update_rows(RowLaunch& L, Op ot, cudaStream_t s);
// out[idx[i],:] = X[i,:] (type ot, ld cols), out_scale[idx[i]] = rscale ? rscale[i] : 1,
// out_flag[idx[i]] = 1 (where non-NULL).
muon_status launch_scatter_rows(RowLaunch& L, Op ot, cudaStream_t s);

// Per-matrix scalars.
struct NormOut {
  const double* rsum;  // per-row sums of squares
  int64_t rows;
  float* s;            // out: 1 / (||X||_F + eps)
  float* xscale;       // out: true X_0 = xscale * stored operand
  float inv_kappa;     // xscale = s when inv_kappa < 0 (unscaled storage), else inv_kappa
};
// One block per matrix: norm^2 = sum of rsum over its rows (fixed order).
muon_status launch_norm_finalize(const NormOut* out, int count, float eps, int* status, cudaStream_t s);

// Dion3 selection for one matrix: top-k of key (fp64, ties to lower index),
// idx ascending; then s = 1/(sqrt(sum_{i in S} rsum_i) + eps) and xscale.
muon_status launch_select(const double* key, const double* rsum, int64_t n, int64_t k, int32_t* idx, float* s_out,
                          float* xscale_out, float eps, float inv_kappa, int* status, cudaStream_t s);

// NorMuon finalize for one matrix (one block): v, d_i, ratio, row scales.
muon_status launch_normuon_finalize(float* rscale, int64_t k, int64_t m, float* v, const int32_t* idx, float beta2,
                                    float eps, int* status, cudaStream_t s);

// The same for many matrices, one block per matrix, kMaxRowMats per launch.
struct NormuonMat {
  float* rscale;
  int64_t k, m;
  float* v;
  const int32_t* idx;
};
muon_status launch_normuon_finalize_batched(const NormuonMat* mats, int count, float beta2, float eps, int* status,
                                            cudaStream_t s);

// Copy an internal (padded) matrix to a caller buffer (ld = cols).
muon_status launch_copy_out(const void* in, Op it, int64_t ldi, void* out, Op ot, int64_t rows, int64_t cols,
                            int* status, cudaStream_t s);

}  // namespace muon

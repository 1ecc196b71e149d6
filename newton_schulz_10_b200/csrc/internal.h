// Host-side interfaces between the libmuon translation units (not exported).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/muon.h"

namespace muon {

constexpr int kMaxGemmGroups = 4;
constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // bound of every device wait

// Operand element types of the GEMM chain.
enum class Op { BF16 = 1, F16 = 2, F32 = 3 };

inline size_t op_size(Op t) { return t == Op::F32 ? 4 : 2; }

// Padded leading dimension (elements) of every internal matrix: a multiple of
// 64 so that rows start on 128-byte boundaries (TMA strides, 16-byte vectors).
inline int64_t pad_ld(int64_t cols) { return (cols + 63) / 64 * 64; }

// One group of same-shape GEMMs, D_b = epilogue(Aop_b * Bop_b^T), b < batch.
//   Aop[i,k] (M x K): a_mn = 0 -> A[i*lda + k]  (K-major, rows of A)
//                     a_mn = 1 -> A[k*lda + i]  (MN-major)
//   Bop[j,k] (N x K): b_mn = 0 -> B[j*ldb + k];  b_mn = 1 -> B[k*ldb + j]
//   D = alpha*s^alpha_pow*acc + beta*s^beta_pow*C + gamma*I, s = scale[b]
//   (s = 1 when scale is NULL); sym = 1: M == N and D is symmetric: only the
//   lower triangle is computed and mirrored (D is then exactly symmetric).
//   part: optional fp32 scratch of part_bytes for split K (symmetric only).
struct GemmDesc {
  const void* A;
  int64_t lda, strideA;
  const void* B;
  int64_t ldb, strideB;
  void* D;
  int64_t ldd, strideD;
  const void* C;
  int64_t ldc, strideC;
  int M, N, K, batch;
  int a_mn, b_mn, sym;
  float alpha, beta, gamma;
  const float* scale;
  int alpha_pow, beta_pow;
  float* part;
  size_t part_bytes;
};

// Tensor-core GEMM (tcgen05 + TMEM + TMA), all groups in one persistent launch.
// Operand type bf16 or f16. Returns MUON_OK or MUON_ERR_CUDA.
// A symmetric launch with fewer tiles than CTAs (pairs) splits K over the
// `part` scratch when it is large enough, then reduces the parts in a second
// launch.
muon_status tc_gemm(Op t, const GemmDesc* g, int ngroups, int* status, uint64_t timeout_ns, cudaStream_t s);

// Fused chain: the products of a whole Newton-Schulz chain in as few
// persistent launches as the kernel parameters allow. descs holds nphase
// phases of ngroups products each (descs[k * ngroups + i]: phase k, shape
// group i; every phase has the same groups and batch counts). The tiles of
// product (k, i) for matrix b wait (bounded) until every tile of product
// (k - 1, i) for matrix b is in memory, so the products of different matrices
// overlap and no launch boundary separates dependent products. counters:
// tc_chain_counter_words(nphase, sum of the groups' batch) words of
// workspace, cleared by the call. K is never split here.
muon_status tc_chain(Op t, const GemmDesc* descs, int nphase, int ngroups, unsigned* counters, int* status,
                     uint64_t timeout_ns, cudaStream_t s);
size_t tc_chain_counter_words(int nphase, int total_batch);

// 1 (default 0): the Newton-Schulz chains run as fused chains (tc_chain).
void set_gemm_chain(int on);
int gemm_chain();

// Bytes of split-K scratch that X X^T (n x n, inner dimension K) of a group
// of `count` matrices can use in any launch; 0 when it never splits.
size_t tc_split_scratch(int64_t n, int64_t K, int count);

// fp32 FFMA GEMM (no TF32), one group per launch.
muon_status simt_gemm(const GemmDesc& g, cudaStream_t s);

int num_sms();

// 2: tensor-core GEMMs use the CTA-pair kernel (default); 1: single-CTA kernel.
void set_gemm_pair_mode(int pair);

// Per-thread accounting of queued work (launch counts, NS FLOPs).
struct Counters {
  int64_t launches = 0;
  int64_t gemm_launches = 0;
  double flops_sym = 0, flops_dense = 0, flops_exec = 0;
};
Counters& counters();

// One shape group of the Newton-Schulz chain: `count` matrices of
// rows x cols in stored (row-major) orientation. A tall group (rows > cols)
// is iterated in its transposed form through operand layouts; no copy.
//   X[0], X[1]   [count][rows][ldx] operand ping-pong, ldx = pad_ld(cols);
//                X[cur] holds the input on entry and the output on return
//   xscale       per matrix: true X_0 = xscale[b] * stored X[cur] (NULL = 1)
//   nb[]         [count][n][ldn] work matrices, n = min(rows, cols),
//                ldn = pad_ld(n): 2 for the standard chain, 4 for Gram
//   rho          Gram only: R is stored as rho * X X^T (keeps fp16 in range)
//   part         split-K scratch of the X X^T products (NULL: no split)
struct NsGroup {
  int64_t rows, cols;
  int count;
  void* X[2];
  int cur;
  const float* xscale;
  void* nb[4];
  float rho;
  float* part;
  size_t part_bytes;
};

inline int ns_work_buffers(const muon_ns_params* p) { return p->gram ? 4 : 2; }

// Run the chain (standard or Gram per p->gram) on up to kMaxGemmGroups
// groups of operand type t; all groups share each launch. With the fused
// chain on (set_gemm_chain) and `counters` non-NULL (ns_counter_words(...)
// words of workspace), the chain's products run as one fused chain.
muon_status ns_run(Op t, NsGroup* gs, int ng, const muon_ns_params* p, int* status, uint64_t timeout_ns,
                   cudaStream_t s, unsigned* counters);

// Products in one chain: at most 3T (standard) or 4T + 4 (Gram with restart).
int ns_max_phases(const muon_ns_params* p);
// Completion-counter words a fused chain over groups holding `matrices`
// matrices in total needs.
inline size_t ns_counter_words(const muon_ns_params* p, int64_t matrices) {
  return (size_t)ns_max_phases(p) * (size_t)matrices;
}

}  // namespace muon

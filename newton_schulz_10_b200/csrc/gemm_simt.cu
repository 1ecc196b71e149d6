// fp32 FFMA GEMM for the fp32 Newton-Schulz path (no TF32: the fp32 path is
// the accuracy reference of the library, 1e-4 relative).
//
// 32x32 output tile per 256-thread block (2x2 outputs per thread), so that
// the small matrices this path serves still spread over many SMs. K advances
// in slices of 32 through two shared-memory buffers stored as [k][i]; the
// next slice is loaded into registers while the current one is multiplied.
// A symmetric output (sym = 1) is computed on the lower-triangle tiles and
// mirrored, so it is exactly symmetric.
#include "common.cuh"
#include "internal.h"

namespace muon {

namespace simt {

constexpr int TM = 32, TN = 32, TK = 32;
constexpr int THREADS = 256;
constexpr int PER_THREAD = TM * TK / THREADS;  // operand elements each thread stages per slice

struct Slice {
  float a[PER_THREAD], b[PER_THREAD];
};

// Element e of a 32x32 operand slice: K-major reads consecutive k, MN-major
// consecutive rows, so consecutive threads read consecutive addresses.
__device__ __forceinline__ void slice_coords(int e, int mn, int* i, int* k) {
  if (mn) { *k = e / TM; *i = e % TM; } else { *i = e / TK; *k = e % TK; }
}

__device__ __forceinline__ void load_slice(const GemmDesc& g, const float* A, const float* B, int m0, int n0, int k0,
                                           Slice& r) {
#pragma unroll
  for (int u = 0; u < PER_THREAD; ++u) {
    const int e = threadIdx.x + u * THREADS;
    int i, k;
    slice_coords(e, g.a_mn, &i, &k);
    {
      const int gi = m0 + i, gk = k0 + k;
      r.a[u] = (gi < g.M && gk < g.K) ? (g.a_mn ? A[(long long)gk * g.lda + gi] : A[(long long)gi * g.lda + gk]) : 0.f;
    }
    slice_coords(e, g.b_mn, &i, &k);
    {
      const int gj = n0 + i, gk = k0 + k;
      r.b[u] = (gj < g.N && gk < g.K) ? (g.b_mn ? B[(long long)gk * g.ldb + gj] : B[(long long)gj * g.ldb + gk]) : 0.f;
    }
  }
}

__global__ void __launch_bounds__(THREADS) gemm_f32_kernel(GemmDesc g) {
  __shared__ __align__(16) float sa[2][TK][TM + 4];
  __shared__ __align__(16) float sb[2][TK][TN + 4];
  const int b = blockIdx.z;
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  if (g.sym && n0 > m0) return;  // symmetric output: lower tiles only, mirrored below
  const float* A = reinterpret_cast<const float*>(g.A) + (long long)b * g.strideA;
  const float* B = reinterpret_cast<const float*>(g.B) + (long long)b * g.strideB;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  auto stage = [&](const Slice& r, int buf) {
#pragma unroll
    for (int u = 0; u < PER_THREAD; ++u) {
      const int e = threadIdx.x + u * THREADS;
      int i, k;
      slice_coords(e, g.a_mn, &i, &k);
      sa[buf][k][i] = r.a[u];
      slice_coords(e, g.b_mn, &i, &k);
      sb[buf][k][i] = r.b[u];
    }
  };
  float acc[2][2] = {};
  Slice r;
  load_slice(g, A, B, m0, n0, 0, r);
  stage(r, 0);
  __syncthreads();
  int buf = 0;
  for (int k0 = 0; k0 < g.K; k0 += TK) {
    const bool more = k0 + TK < g.K;
    if (more) load_slice(g, A, B, m0, n0, k0 + TK, r);  // in flight during the products below
#pragma unroll
    for (int k = 0; k < TK; ++k) {
      const float2 av = *reinterpret_cast<const float2*>(&sa[buf][k][ty * 2]);
      const float2 bv = *reinterpret_cast<const float2*>(&sb[buf][k][tx * 2]);
      acc[0][0] = fmaf(av.x, bv.x, acc[0][0]);
      acc[0][1] = fmaf(av.x, bv.y, acc[0][1]);
      acc[1][0] = fmaf(av.y, bv.x, acc[1][0]);
      acc[1][1] = fmaf(av.y, bv.y, acc[1][1]);
    }
    if (more) stage(r, buf ^ 1);  // the other buffer: everyone left it at the last barrier
    __syncthreads();
    buf ^= 1;
  }
  float s = g.scale ? g.scale[b] : 1.f;
  float alpha = g.alpha, beta = g.beta;
  for (int i = 0; i < g.alpha_pow; ++i) alpha *= s;
  for (int i = 0; i < g.beta_pow; ++i) beta *= s;
  float* D = reinterpret_cast<float*>(g.D) + (long long)b * g.strideD;
  const float* C = reinterpret_cast<const float*>(g.C) + (long long)b * g.strideC;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r0 = m0 + ty * 2 + i;
    if (r0 >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int c = n0 + tx * 2 + j;
      if (c >= g.N) continue;
      if (g.sym && c > r0) continue;
      float v = alpha * acc[i][j];
      if (g.beta != 0.f) v += beta * C[(long long)r0 * g.ldc + c];
      if (r0 == c) v += g.gamma;
      D[(long long)r0 * g.ldd + c] = v;
      if (g.sym && c < r0) D[(long long)c * g.ldd + r0] = v;
    }
  }
}

}  // namespace simt

muon_status simt_gemm(const GemmDesc& g, cudaStream_t s) {
  if (g.batch <= 0 || g.M <= 0 || g.N <= 0 || g.K <= 0) return MUON_OK;
  dim3 grid((g.N + simt::TN - 1) / simt::TN, (g.M + simt::TM - 1) / simt::TM, g.batch);
  Counters& cn = counters();
  cn.launches += 1;
  cn.gemm_launches += 1;
  const double mnk = (double)g.M * g.N * g.K * g.batch;
  cn.flops_dense += 2.0 * mnk;
  cn.flops_sym += g.sym ? mnk : 2.0 * mnk;
  cn.flops_exec += g.sym ? mnk + (double)g.M * g.K * g.batch : 2.0 * mnk;
  simt::gemm_f32_kernel<<<grid, simt::THREADS, 0, s>>>(g);
  return cudaGetLastError() == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}

}  // namespace muon

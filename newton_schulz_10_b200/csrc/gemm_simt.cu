// fp32 FFMA GEMM for the fp32 Newton-Schulz path (no TF32: the fp32 path is
// the accuracy reference of the library, 1e-4 relative).
//
// 64x64 output tile per 256-thread block, 4x4 outputs per thread, K in
// slices of 16 staged through shared memory as [k][i] so the inner loop reads
// broadcast-free float4s. A symmetric output (sym = 1) is computed on the
// lower-triangle tiles and mirrored, so it is exactly symmetric.
#include "common.cuh"
#include "internal.h"

namespace muon {

namespace simt {

constexpr int TM = 64, TN = 64, TK = 16;

__global__ void __launch_bounds__(256) gemm_f32_kernel(GemmDesc g) {
  __shared__ __align__(16) float sa[TK][TM + 4];
  __shared__ __align__(16) float sb[TK][TN + 4];
  const int b = blockIdx.z;
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  if (g.sym && n0 > m0) return;  // symmetric output: lower tiles only, mirrored below
  const float* A = reinterpret_cast<const float*>(g.A) + (long long)b * g.strideA;
  const float* B = reinterpret_cast<const float*>(g.B) + (long long)b * g.strideB;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < g.K; k0 += TK) {
    // 64x16 = 1024 elements per operand, 4 per thread
    for (int e = threadIdx.x; e < TM * TK; e += 256) {
      int i, k;
      if (g.a_mn) { k = e / TM; i = e % TM; } else { i = e / TK; k = e % TK; }
      const int gi = m0 + i, gk = k0 + k;
      float x = 0.f;
      if (gi < g.M && gk < g.K) x = g.a_mn ? A[(long long)gk * g.lda + gi] : A[(long long)gi * g.lda + gk];
      sa[k][i] = x;
    }
    for (int e = threadIdx.x; e < TN * TK; e += 256) {
      int j, k;
      if (g.b_mn) { k = e / TN; j = e % TN; } else { j = e / TK; k = e % TK; }
      const int gj = n0 + j, gk = k0 + k;
      float x = 0.f;
      if (gj < g.N && gk < g.K) x = g.b_mn ? B[(long long)gk * g.ldb + gj] : B[(long long)gj * g.ldb + gk];
      sb[k][j] = x;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < TK; ++k) {
      const float4 av = *reinterpret_cast<const float4*>(&sa[k][ty * 4]);
      const float4 bv = *reinterpret_cast<const float4*>(&sb[k][tx * 4]);
      const float a4[4] = {av.x, av.y, av.z, av.w};
      const float b4[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a4[i], b4[j], acc[i][j]);
    }
    __syncthreads();
  }
  float s = g.scale ? g.scale[b] : 1.f;
  float alpha = g.alpha, beta = g.beta;
  for (int i = 0; i < g.alpha_pow; ++i) alpha *= s;
  for (int i = 0; i < g.beta_pow; ++i) beta *= s;
  float* D = reinterpret_cast<float*>(g.D) + (long long)b * g.strideD;
  const float* C = reinterpret_cast<const float*>(g.C) + (long long)b * g.strideC;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = m0 + ty * 4 + i;
    if (r >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = n0 + tx * 4 + j;
      if (c >= g.N) continue;
      if (g.sym && c > r) continue;
      float v = alpha * acc[i][j];
      if (g.beta != 0.f) v += beta * C[(long long)r * g.ldc + c];
      if (r == c) v += g.gamma;
      D[(long long)r * g.ldd + c] = v;
      if (g.sym && c < r) D[(long long)c * g.ldd + r] = v;
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
  simt::gemm_f32_kernel<<<grid, 256, 0, s>>>(g);
  return cudaGetLastError() == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}

}  // namespace muon

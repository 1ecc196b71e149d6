// Memory-bound per-row kernels of the Muon step: momentum with the fused
// Frobenius / selection-key reduction and operand cast, row gathers, NorMuon
// row statistics, the fused weight update, and the small per-matrix
// finalisers. Rows are walked by a warp (short rows) or a whole block (long
// rows) with 16-byte vector accesses when the row length allows; every
// reduction runs in a fixed order, so results are bit-reproducible.
#include <mutex>

#include "common.cuh"
#include "rowops.cuh"

namespace muon {

namespace {

constexpr int BLOCK = 256;
constexpr int UNROLL = 4;  // 16-byte vectors in flight per lane (momentum, row statistics, copy-out)

__device__ __forceinline__ int find_mat(const RowLaunch& L, int task) {
  int lo = 0, hi = L.count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (L.m[mid].task_begin <= task) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Sum over a worker group of WG threads (a warp or the whole block).
template <int WG>
__device__ __forceinline__ double group_sum(double v, double* scratch) {
  if (WG == 32) return warp_sum(v);
  return block_sum(v, scratch);
}
template <int WG>
__device__ __forceinline__ float group_sum_f(float v, double* scratch) {
  if (WG == 32) return warp_sum(v);
  return (float)block_sum((double)v, scratch);  // fp64 across warps: exact for these magnitudes
}

template <typename S> struct Src;
template <> struct Src<float> {
  static __device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
  static __device__ __forceinline__ float load1(const float* p) { return *p; }
};
template <> struct Src<__nv_bfloat16> {
  static __device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const float2 a = Elem<__nv_bfloat16>::unpack2(u.x), b = Elem<__nv_bfloat16>::unpack2(u.y);
    return make_float4(a.x, a.y, b.x, b.y);
  }
  static __device__ __forceinline__ float load1(const __nv_bfloat16* p) { return __bfloat162float(*p); }
};
template <> struct Src<__half> {
  static __device__ __forceinline__ float4 load4(const __half* p) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const float2 a = Elem<__half>::unpack2(u.x), b = Elem<__half>::unpack2(u.y);
    return make_float4(a.x, a.y, b.x, b.y);
  }
  static __device__ __forceinline__ float load1(const __half* p) { return __half2float(*p); }
};

template <typename T> struct Dst;
template <> struct Dst<float> {
  static __device__ __forceinline__ void store4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
  static __device__ __forceinline__ void store1(float* p, float v) { *p = v; }
};
template <typename T> struct DstH {
  static __device__ __forceinline__ void store4(T* p, float4 v) {
    uint2 u;
    u.x = Elem<T>::pack2(v.x, v.y);
    u.y = Elem<T>::pack2(v.z, v.w);
    *reinterpret_cast<uint2*>(p) = u;
  }
  static __device__ __forceinline__ void store1(T* p, float v) { *p = Elem<T>::from_f(v); }
};
template <> struct Dst<__nv_bfloat16> : DstH<__nv_bfloat16> {};
template <> struct Dst<__half> : DstH<__half> {};

// Non-finite output of the Newton-Schulz chain (an fp16 overflow, a NaN that
// entered through the input): reported once per warp as MUON_ERR_NONFINITE.
__device__ __forceinline__ bool finite4(float4 v) {
  return isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w);
}
__device__ __forceinline__ void report_if_any(bool bad, int* status) {
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) report(status, MUON_ERR_NONFINITE);
}

// ---------------------------------------------------------------------------
// momentum + fused reductions + cast
// ---------------------------------------------------------------------------

template <int WG, typename T, int MODE, bool CAST>
__global__ void __launch_bounds__(BLOCK) momentum_rows(const __grid_constant__ RowLaunch L) {
  __shared__ double scratch[32];
  const int task = blockIdx.x * (BLOCK / WG) + threadIdx.x / WG;
  const int l = threadIdx.x % WG;
  bool active = task < L.total_tasks;
  const RowMat& m = L.m[find_mat(L, active ? task : L.total_tasks - 1)];
  const int64_t r = active ? task - m.task_begin : 0;
  if (active) active = MUON_IN_BOUNDS(r >= 0 && r < m.rows && (!CAST || m.ldx >= m.cols), L.status);
  double ss = 0.0, sa = 0.0;
  if (active) {
    float* M = m.M + r * m.cols;
    const float* G = m.G + r * m.cols;
    T* X = CAST ? reinterpret_cast<T*>(m.X) + r * m.ldx : nullptr;
    const float mu = L.mu;
    if ((m.cols & 3) == 0) {
      const int64_t n4 = m.cols >> 2;
      // UNROLL vectors of M and of G in flight per lane before any is used
      for (int64_t c0 = l; c0 < n4; c0 += UNROLL * WG) {
        float4 x[UNROLL], g[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
          const int64_t c = c0 + u * WG;
          if (c < n4) {
            x[u] = *reinterpret_cast<const float4*>(M + 4 * c);
            g[u] = __ldcs(reinterpret_cast<const float4*>(G + 4 * c));
          }
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
          const int64_t c = c0 + u * WG;
          if (c >= n4) break;
          float4 y = x[u];
          if (MODE == MOM_MUON) {
            y.x = fmaf(mu, y.x, g[u].x); y.y = fmaf(mu, y.y, g[u].y);
            y.z = fmaf(mu, y.z, g[u].z); y.w = fmaf(mu, y.w, g[u].w);
          } else {
            y.x += g[u].x; y.y += g[u].y; y.z += g[u].z; y.w += g[u].w;
          }
          *reinterpret_cast<float4*>(M + 4 * c) = y;
          if (CAST) Dst<T>::store4(X + 4 * c, y);
          const double a = y.x, b = y.y, cc = y.z, d = y.w;
          ss += a * a + b * b + cc * cc + d * d;
          sa += fabs(a) + fabs(b) + fabs(cc) + fabs(d);
        }
      }
    } else {
      for (int64_t c = l; c < m.cols; c += WG) {
        float x = M[c];
        const float g = G[c];
        x = MODE == MOM_MUON ? fmaf(mu, x, g) : x + g;
        M[c] = x;
        if (CAST) Dst<T>::store1(X + c, x);
        ss += (double)x * (double)x;
        sa += fabs((double)x);
      }
    }
  }
  ss = group_sum<WG>(ss, scratch);
  sa = group_sum<WG>(sa, scratch);
  if (active && l == 0) {
    if (m.rsum) m.rsum[r] = ss;
    if (m.rkey) m.rkey[r] = L.key_l2 ? ss : sa;
  }
}

// ---------------------------------------------------------------------------
// row statistics of a read-only source matrix (ns_polar input, select_rows)
// ---------------------------------------------------------------------------

template <int WG, typename S>
__global__ void __launch_bounds__(BLOCK) row_stats(const __grid_constant__ RowLaunch L) {
  __shared__ double scratch[32];
  const int task = blockIdx.x * (BLOCK / WG) + threadIdx.x / WG;
  const int l = threadIdx.x % WG;
  bool active = task < L.total_tasks;
  const RowMat& m = L.m[find_mat(L, active ? task : L.total_tasks - 1)];
  const int64_t r = active ? task - m.task_begin : 0;
  if (active) active = MUON_IN_BOUNDS(r >= 0 && r < m.rows, L.status);
  double ss = 0.0, sa = 0.0;
  if (active) {
    const S* x = reinterpret_cast<const S*>(m.src) + r * m.cols;
    if ((m.cols & 3) == 0) {
      const int64_t n4 = m.cols >> 2;
      auto add = [&](const float4 v) {
        const double a = v.x, b = v.y, cc = v.z, d = v.w;
        ss += a * a + b * b + cc * cc + d * d;
        sa += fabs(a) + fabs(b) + fabs(cc) + fabs(d);
      };
      int64_t c = l;
      // UNROLL vectors in flight per lane; summed in the same order as one at a time
      for (; c + (UNROLL - 1) * WG < n4; c += UNROLL * WG) {
        float4 v[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) v[u] = Src<S>::load4(x + 4 * (c + u * WG));
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) add(v[u]);
      }
      for (; c < n4; c += WG) add(Src<S>::load4(x + 4 * c));
    } else {
      for (int64_t c = l; c < m.cols; c += WG) {
        const double a = Src<S>::load1(x + c);
        ss += a * a;
        sa += fabs(a);
      }
    }
  }
  ss = group_sum<WG>(ss, scratch);
  sa = group_sum<WG>(sa, scratch);
  if (active && l == 0) {
    if (m.rsum) m.rsum[r] = ss;
    if (m.rkey) m.rkey[r] = L.key_l2 ? ss : sa;
  }
}

// ---------------------------------------------------------------------------
// scaled cast / row gather into the operand buffer
// ---------------------------------------------------------------------------

template <int WG, typename S, typename T>
__global__ void __launch_bounds__(BLOCK) cast_rows(const __grid_constant__ RowLaunch L) {
  const int task = blockIdx.x * (BLOCK / WG) + threadIdx.x / WG;
  const int l = threadIdx.x % WG;
  if (task >= L.total_tasks) return;
  const RowMat& m = L.m[find_mat(L, task)];
  const int64_t i = task - m.task_begin;
  if (!MUON_IN_BOUNDS(i >= 0 && i < m.ntask && m.ldx >= m.cols, L.status)) return;
  const int64_t j = m.idx ? (int64_t)m.idx[i] : i;
  if (!MUON_IN_BOUNDS(j >= 0 && j < m.rows, L.status)) return;
  const float mult = (m.mult ? *m.mult : 1.f) * m.kappa;
  const S* x = reinterpret_cast<const S*>(m.src) + j * m.cols;
  T* X = reinterpret_cast<T*>(m.X) + i * m.ldx;
  if ((m.cols & 3) == 0) {
    for (int64_t c = l; c < (m.cols >> 2); c += WG) {
      float4 v = Src<S>::load4(x + 4 * c);
      v.x *= mult; v.y *= mult; v.z *= mult; v.w *= mult;
      Dst<T>::store4(X + 4 * c, v);
    }
  } else {
    for (int64_t c = l; c < m.cols; c += WG) Dst<T>::store1(X + c, Src<S>::load1(x + c) * mult);
  }
}

// ---------------------------------------------------------------------------
// NorMuon row statistics and the fused update
// ---------------------------------------------------------------------------

template <int WG, typename T>
__global__ void __launch_bounds__(BLOCK) normuon_rows(const __grid_constant__ RowLaunch L) {
  __shared__ double scratch[32];
  const int task = blockIdx.x * (BLOCK / WG) + threadIdx.x / WG;
  const int l = threadIdx.x % WG;
  bool active = task < L.total_tasks;
  const RowMat& m = L.m[find_mat(L, active ? task : L.total_tasks - 1)];
  const int64_t i = active ? task - m.task_begin : 0;
  if (active) active = MUON_IN_BOUNDS(i >= 0 && i < m.ntask && m.ldx >= m.cols, L.status);
  float acc = 0.f;
  if (active) {
    const T* o = reinterpret_cast<const T*>(m.X) + i * m.ldx;
    if ((m.cols & 3) == 0) {
      for (int64_t c = l; c < (m.cols >> 2); c += WG) {
        const float4 v = Src<T>::load4(o + 4 * c);
        acc = fmaf(v.x, v.x, acc); acc = fmaf(v.y, v.y, acc); acc = fmaf(v.z, v.z, acc); acc = fmaf(v.w, v.w, acc);
      }
    } else {
      for (int64_t c = l; c < m.cols; c += WG) {
        const float v = Src<T>::load1(o + c);
        acc = fmaf(v, v, acc);
      }
    }
  }
  acc = group_sum_f<WG>(acc, scratch);
  if (active && l == 0) m.rscale[i] = acc;
}

template <int WG, typename T, bool DECAY>
__global__ void __launch_bounds__(BLOCK) update_rows(const __grid_constant__ RowLaunch L) {
  const int l = threadIdx.x % WG;
  // persistent: the block walks row groups with a block-uniform stride
  for (int task0 = blockIdx.x * (BLOCK / WG); task0 < L.total_tasks; task0 += gridDim.x * (BLOCK / WG)) {
  const int task = task0 + threadIdx.x / WG;
  if (task >= L.total_tasks) break;
  const RowMat& m = L.m[find_mat(L, task)];
  const int64_t i = task - m.task_begin;
  if (!MUON_IN_BOUNDS(i >= 0 && i < m.ntask && m.ldx >= m.cols, L.status)) continue;
  if (m.flag && !m.flag[i]) continue;  // a row that was not orthogonalised keeps W and M
  const int64_t j = m.idx ? (int64_t)m.idx[i] : i;
  if (!MUON_IN_BOUNDS(j >= 0 && j < m.rows, L.status)) continue;
  const float step = -L.lr * (m.rscale ? m.rscale[i] : 1.f);
  const T* o = reinterpret_cast<const T*>(m.X) + i * m.ldx;
  float* W = m.W + j * m.cols;
  float* M = DECAY ? m.M + j * m.cols : nullptr;
  const float mu = L.mu;
  bool bad = false;
  if ((m.cols & 3) == 0) {
    for (int64_t c = l; c < (m.cols >> 2); c += WG) {
      const float4 ov = Src<T>::load4(o + 4 * c);
      bad |= !finite4(ov);
      float4 w = *reinterpret_cast<const float4*>(W + 4 * c);
      w.x = fmaf(step, ov.x, w.x); w.y = fmaf(step, ov.y, w.y); w.z = fmaf(step, ov.z, w.z); w.w = fmaf(step, ov.w, w.w);
      *reinterpret_cast<float4*>(W + 4 * c) = w;
      if (DECAY) {
        float4 x = *reinterpret_cast<const float4*>(M + 4 * c);
        x.x *= mu; x.y *= mu; x.z *= mu; x.w *= mu;
        *reinterpret_cast<float4*>(M + 4 * c) = x;
      }
    }
  } else {
    for (int64_t c = l; c < m.cols; c += WG) {
      const float ov = Src<T>::load1(o + c);
      bad |= !isfinite(ov);
      W[c] = fmaf(step, ov, W[c]);
      if (DECAY) M[c] *= mu;
    }
  }
  report_if_any(bad, L.status);
  }
}

// Operand rows to caller rows at their stored positions (the output of
// muon_orthogonalize): values copied exactly (same element type).
template <int WG, typename T>
__global__ void __launch_bounds__(BLOCK) scatter_rows(const __grid_constant__ RowLaunch L) {
  const int task = blockIdx.x * (BLOCK / WG) + threadIdx.x / WG;
  const int l = threadIdx.x % WG;
  if (task >= L.total_tasks) return;
  const RowMat& m = L.m[find_mat(L, task)];
  const int64_t i = task - m.task_begin;
  if (!MUON_IN_BOUNDS(i >= 0 && i < m.ntask && m.ldx >= m.cols, L.status)) return;
  const int64_t j = m.idx ? (int64_t)m.idx[i] : i;
  if (!MUON_IN_BOUNDS(j >= 0 && j < m.rows, L.status)) return;
  const T* x = reinterpret_cast<const T*>(m.X) + i * m.ldx;
  T* o = reinterpret_cast<T*>(m.out) + j * m.cols;
  if ((m.cols & 3) == 0) {
    for (int64_t c = l; c < (m.cols >> 2); c += WG) Dst<T>::store4(o + 4 * c, Src<T>::load4(x + 4 * c));
  } else {
    for (int64_t c = l; c < m.cols; c += WG) Dst<T>::store1(o + c, Src<T>::load1(x + c));
  }
  if (l == 0) {
    if (m.out_scale) m.out_scale[j] = m.rscale ? m.rscale[i] : 1.f;
    if (m.out_flag) m.out_flag[j] = 1;
  }
}

// ---------------------------------------------------------------------------
// per-matrix finalisers
// ---------------------------------------------------------------------------

struct FinalizeArgs {
  NormOut m[kMaxRowMats];
};

__global__ void __launch_bounds__(BLOCK) norm_finalize(const __grid_constant__ FinalizeArgs a, float eps, int* status) {
  __shared__ double scratch[32];
  const NormOut& o = a.m[blockIdx.x];
  double t = 0.0;
  for (int64_t r = threadIdx.x; r < o.rows; r += BLOCK) t += o.rsum[r];
  t = block_sum(t, scratch);
  if (threadIdx.x == 0) {
    if (!isfinite(t)) report(status, MUON_ERR_NONFINITE);
    const float s = (float)(1.0 / (sqrt(t) + (double)eps));
    *o.s = s;
    *o.xscale = o.inv_kappa < 0.f ? s : o.inv_kappa;
  }
}

constexpr int SEL_THREADS = 1024;
// Keys of up to this many rows are staged in shared memory once (8 bytes
// each) and every radix pass reads them there; longer key arrays are read
// from global memory in every pass.
constexpr int64_t SEL_SMEM_ROWS = 20480;

// Top-k by radix selection on the fp64 key bits (keys are >= 0, so their bit
// patterns order like the values), then an index-ordered compaction.
__global__ void __launch_bounds__(SEL_THREADS) select_topk(const double* key, const double* rsum, int64_t n,
                                                           int64_t k, int32_t* idx, float* s_out, float* xscale_out,
                                                           float eps, float inv_kappa, int* status) {
  extern __shared__ unsigned long long skeys[];
  __shared__ unsigned int hist[256];
  __shared__ unsigned long long s_prefix;
  __shared__ long long s_remaining;
  __shared__ long long warp_cnt[SEL_THREADS / 32];
  __shared__ double scratch[32];
  const int tid = threadIdx.x;
  const bool staged = n <= SEL_SMEM_ROWS;
  const unsigned long long* u = reinterpret_cast<const unsigned long long*>(key);
  if (staged) {
    for (int64_t i = tid; i < n; i += SEL_THREADS) skeys[i] = u[i];
    u = skeys;
  }
  if (tid == 0) {
    s_prefix = 0ull;
    s_remaining = k;
  }
  unsigned long long mask = 0ull;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += SEL_THREADS) hist[i] = 0u;
    __syncthreads();
    const unsigned long long prefix = s_prefix;
    for (int64_t i = tid; i < n; i += SEL_THREADS) {
      const unsigned long long x = u[i];
      if ((x & mask) == prefix) atomicAdd(&hist[(x >> shift) & 255ull], 1u);
    }
    __syncthreads();
    if (tid < 32) {
      // the digit of the k-th largest key among those with this prefix: lane
      // l holds bins 255 - 8l down to 248 - 8l, an inclusive scan over lanes
      // counts the keys at or above each lane's bins, and the first lane
      // whose count reaches the remaining rank finds the digit in its bins
      unsigned c[8], tot = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = hist[255 - 8 * tid - j];
        tot += c[j];
      }
      unsigned incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += y;
      }
      const long long rem = s_remaining;
      const unsigned hit = __ballot_sync(0xffffffffu, (long long)incl >= rem);
      if (tid == __ffs(hit) - 1) {
        long long cum = (long long)(incl - tot);  // keys above this lane's bins
        int sel = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (cum + (long long)c[j] >= rem) {
            sel = 255 - 8 * tid - j;
            break;
          }
          cum += c[j];
        }
        s_remaining = rem - cum;
        s_prefix = prefix | ((unsigned long long)sel << shift);
      }
    }
    mask |= 255ull << shift;
    __syncthreads();
  }
  const unsigned long long thr = s_prefix;  // bit pattern of the k-th largest key
  const long long need_eq = s_remaining;    // how many keys equal to thr to take
  // contiguous chunk per thread keeps index order across the block scan
  const int64_t chunk = (n + SEL_THREADS - 1) / SEL_THREADS;
  const int64_t lo = tid * chunk, hi = lo + chunk < n ? lo + chunk : n;
  long long eq = 0;
  for (int64_t i = lo; i < hi; ++i) eq += (u[i] == thr);
  // exclusive scan of eq over threads (index order)
  const int lane = tid & 31, w = tid >> 5;
  long long incl = eq;
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_cnt[w] = incl;
  __syncthreads();
  long long base = 0;
  for (int i = 0; i < w; ++i) base += warp_cnt[i];
  long long eq_before = base + incl - eq;
  __syncthreads();
  // count selected per thread
  long long sel = 0;
  {
    long long e = eq_before;
    for (int64_t i = lo; i < hi; ++i) {
      const unsigned long long x = u[i];
      if (x > thr) ++sel;
      else if (x == thr) {
        if (e < need_eq) ++sel;
        ++e;
      }
    }
  }
  incl = sel;
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_cnt[w] = incl;
  __syncthreads();
  base = 0;
  for (int i = 0; i < w; ++i) base += warp_cnt[i];
  long long pos = base + incl - sel;
  {
    long long e = eq_before;
    for (int64_t i = lo; i < hi; ++i) {
      const unsigned long long x = u[i];
      bool take = false;
      if (x > thr) take = true;
      else if (x == thr) {
        take = e < need_eq;
        ++e;
      }
      if (take && MUON_IN_BOUNDS(pos >= 0 && pos < k, status)) idx[pos++] = (int32_t)i;
    }
  }
  __syncthreads();
  // Frobenius norm of the selected rows, ascending-index order
  double t = 0.0;
  for (int64_t i = tid; i < k; i += SEL_THREADS)
    if (MUON_IN_BOUNDS(idx[i] >= 0 && idx[i] < n, status)) t += rsum[idx[i]];
  t = block_sum(t, scratch);
  if (tid == 0) {
    if (!isfinite(t)) report(status, MUON_ERR_NONFINITE);
    const float s = (float)(1.0 / (sqrt(t) + (double)eps));
    *s_out = s;
    *xscale_out = inv_kappa < 0.f ? s : inv_kappa;
  }
}

__device__ void normuon_finalize_block(float* rscale, int64_t k, int64_t m, float* v, const int32_t* idx,
                                       float beta2, float eps, int* status, double* scratch);

__global__ void __launch_bounds__(BLOCK) normuon_finalize(float* rscale, int64_t k, int64_t m, float* v,
                                                          const int32_t* idx, float beta2, float eps, int* status) {
  __shared__ double scratch[32];
  normuon_finalize_block(rscale, k, m, v, idx, beta2, eps, status, scratch);
}

struct NormuonArgs {
  NormuonMat m[kMaxRowMats];
};

__global__ void __launch_bounds__(BLOCK) normuon_finalize_many(const __grid_constant__ NormuonArgs a, float beta2,
                                                               float eps, int* status) {
  __shared__ double scratch[32];
  const NormuonMat& o = a.m[blockIdx.x];
  normuon_finalize_block(o.rscale, o.k, o.m, o.v, o.idx, beta2, eps, status, scratch);
}

// Eq. (2) for one matrix by one block: v_j <- beta2 v_j + (1 - beta2) r_i / m,
// d_i = 1 / (sqrt(v_j) + eps), ratio = sqrt(sum r) / sqrt(sum d^2 r),
// rscale[i] <- ratio * d_i (rscale holds r_i on entry).
__device__ void normuon_finalize_block(float* rscale, int64_t k, int64_t m, float* v, const int32_t* idx,
                                       float beta2, float eps, int* status, double* scratch) {
  double sum_r = 0.0, sum_dr = 0.0;
  const float inv_m = 1.f / (float)m;
  for (int64_t i = threadIdx.x; i < k; i += BLOCK) {
    const int64_t j = idx ? idx[i] : i;
    const float r = rscale[i];
    const float vn = beta2 * v[j] + (1.f - beta2) * (r * inv_m);
    v[j] = vn;
    const float d = 1.f / (sqrtf(vn) + eps);
    rscale[i] = d;
    sum_r += (double)r;
    sum_dr += (double)d * (double)d * (double)r;
  }
  sum_r = block_sum(sum_r, scratch);
  sum_dr = block_sum(sum_dr, scratch);
  const float ratio = sum_dr > 0.0 ? (float)(sqrt(sum_r) / sqrt(sum_dr)) : 0.f;
  if (threadIdx.x == 0 && !isfinite(ratio)) report(status, MUON_ERR_NONFINITE);
  __syncthreads();
  for (int64_t i = threadIdx.x; i < k; i += BLOCK) rscale[i] = ratio * rscale[i];
}

// cols % 4 == 0: block (row, chunk of BLOCK * UNROLL vectors of 4), UNROLL
// vectors in flight per thread, no index division.
template <typename I, typename O>
__global__ void __launch_bounds__(BLOCK) copy_out4(const I* in, int64_t ldi, O* out, int64_t cols, int* status) {
  const int64_t r = blockIdx.x;
  const int64_t n4 = cols >> 2;
  const int64_t c0 = (int64_t)blockIdx.y * (BLOCK * UNROLL) + threadIdx.x;
  const I* src = in + r * ldi;
  O* dst = out + r * cols;
  float4 v[UNROLL];
#pragma unroll
  for (int u = 0; u < UNROLL; ++u) {
    const int64_t c = c0 + u * BLOCK;
    if (c < n4) v[u] = Src<I>::load4(src + 4 * c);
  }
  bool bad = false;
#pragma unroll
  for (int u = 0; u < UNROLL; ++u) {
    const int64_t c = c0 + u * BLOCK;
    if (c < n4) {
      bad |= !finite4(v[u]);
      Dst<O>::store4(dst + 4 * c, v[u]);
    }
  }
  report_if_any(bad, status);
}

template <typename I, typename O>
__global__ void __launch_bounds__(BLOCK) copy_out(const I* in, int64_t ldi, O* out, int64_t rows, int64_t cols,
                                                  int* status) {
  const int64_t total = rows * cols;
  bool bad = false;
  for (int64_t e = blockIdx.x * (int64_t)BLOCK + threadIdx.x; e < total; e += (int64_t)gridDim.x * BLOCK) {
    const int64_t r = e / cols, c = e - r * cols;
    const float x = Src<I>::load1(in + r * ldi + c);
    bad |= !isfinite(x);
    Dst<O>::store1(out + e, x);
  }
  report_if_any(bad, status);
}

// ---------------------------------------------------------------------------
// launch helpers
// ---------------------------------------------------------------------------

int64_t max_cols(const RowLaunch& L) {
  int64_t c = 0;
  for (int i = 0; i < L.count; ++i) c = L.m[i].cols > c ? L.m[i].cols : c;
  return c;
}

// Long rows get a whole block, short ones a warp.
bool use_block(const RowLaunch& L) { return max_cols(L) > 8192; }

int grid_for(const RowLaunch& L, bool block) {
  return block ? L.total_tasks : (L.total_tasks + (BLOCK / 32) - 1) / (BLOCK / 32);
}

// Persistent grid for the update, which loops over row groups: enough blocks
// to fill every SM several times over, never more than there is work.
int persistent_grid(const RowLaunch& L, bool block) {
  const int g = grid_for(L, block);
  const int cap = num_sms() * (2048 / BLOCK);
  return g < cap ? g : cap;
}

void finish(RowLaunch& L) {
  int t = 0;
  for (int i = 0; i < L.count; ++i) {
    L.m[i].task_begin = t;
    t += L.m[i].ntask;
  }
  L.total_tasks = t;
}

muon_status last(int launched = 1) {
  counters().launches += launched;
  return cudaGetLastError() == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}

template <typename T>
void momentum_dispatch(RowLaunch& L, bool cast, bool block, cudaStream_t s) {
  const int g = grid_for(L, block);
#define MOM(WG, MODE, CAST) momentum_rows<WG, T, MODE, CAST><<<g, BLOCK, 0, s>>>(L)
  if (block) {
    if (L.mode == MOM_MUON) { if (cast) MOM(256, MOM_MUON, true); else MOM(256, MOM_MUON, false); }
    else { if (cast) MOM(256, MOM_DION3, true); else MOM(256, MOM_DION3, false); }
  } else {
    if (L.mode == MOM_MUON) { if (cast) MOM(32, MOM_MUON, true); else MOM(32, MOM_MUON, false); }
    else { if (cast) MOM(32, MOM_DION3, true); else MOM(32, MOM_DION3, false); }
  }
#undef MOM
}

}  // namespace

muon_status launch_momentum_rows(RowLaunch& L, Op xt, cudaStream_t s) {
  finish(L);
  if (L.total_tasks == 0) return MUON_OK;
  bool cast = false;
  for (int i = 0; i < L.count; ++i) cast = cast || L.m[i].X != nullptr;
  const bool block = use_block(L);
  if (xt == Op::F16) momentum_dispatch<__half>(L, cast, block, s);
  else if (xt == Op::F32) momentum_dispatch<float>(L, cast, block, s);
  else momentum_dispatch<__nv_bfloat16>(L, cast, block, s);
  return last();
}

muon_status launch_row_stats(RowLaunch& L, Op st, cudaStream_t s) {
  finish(L);
  if (L.total_tasks == 0) return MUON_OK;
  const bool block = use_block(L);
  const int g = grid_for(L, block);
  if (st == Op::F32) {
    if (block) row_stats<256, float><<<g, BLOCK, 0, s>>>(L); else row_stats<32, float><<<g, BLOCK, 0, s>>>(L);
  } else {
    if (block) row_stats<256, __nv_bfloat16><<<g, BLOCK, 0, s>>>(L);
    else row_stats<32, __nv_bfloat16><<<g, BLOCK, 0, s>>>(L);
  }
  return last();
}

template <typename S>
static void cast_dispatch(RowLaunch& L, Op xt, bool block, int g, cudaStream_t s) {
  if (xt == Op::F32) {
    if (block) cast_rows<256, S, float><<<g, BLOCK, 0, s>>>(L); else cast_rows<32, S, float><<<g, BLOCK, 0, s>>>(L);
  } else if (xt == Op::F16) {
    if (block) cast_rows<256, S, __half><<<g, BLOCK, 0, s>>>(L); else cast_rows<32, S, __half><<<g, BLOCK, 0, s>>>(L);
  } else {
    if (block) cast_rows<256, S, __nv_bfloat16><<<g, BLOCK, 0, s>>>(L);
    else cast_rows<32, S, __nv_bfloat16><<<g, BLOCK, 0, s>>>(L);
  }
}

muon_status launch_cast_rows(RowLaunch& L, Op st, Op xt, cudaStream_t s) {
  finish(L);
  if (L.total_tasks == 0) return MUON_OK;
  const bool block = use_block(L);
  const int g = grid_for(L, block);
  if (st == Op::F32) cast_dispatch<float>(L, xt, block, g, s);
  else cast_dispatch<__nv_bfloat16>(L, xt, block, g, s);
  return last();
}

muon_status launch_normuon_rows(RowLaunch& L, Op ot, cudaStream_t s) {
  finish(L);
  if (L.total_tasks == 0) return MUON_OK;
  const bool block = use_block(L);
  const int g = grid_for(L, block);
#define NR(WG, T) normuon_rows<WG, T><<<g, BLOCK, 0, s>>>(L)
  if (ot == Op::F32) { if (block) NR(256, float); else NR(32, float); }
  else if (ot == Op::F16) { if (block) NR(256, __half); else NR(32, __half); }
  else { if (block) NR(256, __nv_bfloat16); else NR(32, __nv_bfloat16); }
#undef NR
  return last();
}

muon_status launch_update_rows(RowLaunch& L, Op ot, cudaStream_t s) {
  finish(L);
  if (L.total_tasks == 0) return MUON_OK;
  const bool block = use_block(L);
  const int g = persistent_grid(L, block);
  const bool decay = L.mode == 1;
#define UP(WG, T) (decay ? update_rows<WG, T, true><<<g, BLOCK, 0, s>>>(L) : update_rows<WG, T, false><<<g, BLOCK, 0, s>>>(L))
  if (ot == Op::F32) { if (block) UP(256, float); else UP(32, float); }
  else if (ot == Op::F16) { if (block) UP(256, __half); else UP(32, __half); }
  else { if (block) UP(256, __nv_bfloat16); else UP(32, __nv_bfloat16); }
#undef UP
  return last();
}

muon_status launch_scatter_rows(RowLaunch& L, Op ot, cudaStream_t s) {
  finish(L);
  if (L.total_tasks == 0) return MUON_OK;
  const bool block = use_block(L);
  const int g = grid_for(L, block);
#define SR(WG, T) scatter_rows<WG, T><<<g, BLOCK, 0, s>>>(L)
  if (ot == Op::F32) { if (block) SR(256, float); else SR(32, float); }
  else if (ot == Op::F16) { if (block) SR(256, __half); else SR(32, __half); }
  else { if (block) SR(256, __nv_bfloat16); else SR(32, __nv_bfloat16); }
#undef SR
  return last();
}

muon_status launch_norm_finalize(const NormOut* out, int count, float eps, int* status, cudaStream_t s) {
  for (int b0 = 0; b0 < count; b0 += kMaxRowMats) {
    FinalizeArgs a;
    const int n = count - b0 < kMaxRowMats ? count - b0 : kMaxRowMats;
    for (int i = 0; i < n; ++i) a.m[i] = out[b0 + i];
    norm_finalize<<<n, BLOCK, 0, s>>>(a, eps, status);
  }
  return last((count + kMaxRowMats - 1) / kMaxRowMats);
}

muon_status launch_select(const double* key, const double* rsum, int64_t n, int64_t k, int32_t* idx, float* s_out,
                          float* xscale_out, float eps, float inv_kappa, int* status, cudaStream_t s) {
  // the staged keys need more than the default 48 KB of dynamic shared
  // memory: allowed once per device
  static std::mutex mu;
  static bool set_up[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return MUON_ERR_CUDA;
  }
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!set_up[dev]) {
      if (cudaFuncSetAttribute((const void*)select_topk, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)(SEL_SMEM_ROWS * sizeof(unsigned long long))) != cudaSuccess)
        return MUON_ERR_CUDA;
      set_up[dev] = true;
    }
  }
  const size_t smem = n <= SEL_SMEM_ROWS ? (size_t)n * sizeof(unsigned long long) : 0;
  select_topk<<<1, SEL_THREADS, smem, s>>>(key, rsum, n, k, idx, s_out, xscale_out, eps, inv_kappa, status);
  return last();
}

muon_status launch_normuon_finalize(float* rscale, int64_t k, int64_t m, float* v, const int32_t* idx, float beta2,
                                    float eps, int* status, cudaStream_t s) {
  normuon_finalize<<<1, BLOCK, 0, s>>>(rscale, k, m, v, idx, beta2, eps, status);
  return last();
}

muon_status launch_normuon_finalize_batched(const NormuonMat* mats, int count, float beta2, float eps, int* status,
                                            cudaStream_t s) {
  int launched = 0;
  for (int b0 = 0; b0 < count; b0 += kMaxRowMats) {
    NormuonArgs a;
    const int n = count - b0 < kMaxRowMats ? count - b0 : kMaxRowMats;
    for (int i = 0; i < n; ++i) a.m[i] = mats[b0 + i];
    normuon_finalize_many<<<n, BLOCK, 0, s>>>(a, beta2, eps, status);
    ++launched;
  }
  return last(launched);
}

muon_status launch_copy_out(const void* in, Op it, int64_t ldi, void* out, Op ot, int64_t rows, int64_t cols,
                            int* status, cudaStream_t s) {
  const int64_t total = rows * cols;
  if (total == 0) return MUON_OK;
  int64_t g = (total + BLOCK - 1) / BLOCK;
  if (g > 148 * 16) g = 148 * 16;
  // rows of out start on 16-byte (f32) / 8-byte (bf16) boundaries when cols % 4 == 0
  const int64_t chunks = ((cols >> 2) + BLOCK * UNROLL - 1) / (BLOCK * UNROLL);
  const bool v4 = (cols & 3) == 0 && rows <= INT32_MAX && chunks <= 65535;
  const dim3 g4((unsigned)rows, (unsigned)chunks);
#define CP(I, O)                                                                                             \
  do {                                                                                                       \
    if (v4) copy_out4<I, O><<<g4, BLOCK, 0, s>>>(reinterpret_cast<const I*>(in), ldi, reinterpret_cast<O*>(out), cols, status); \
    else copy_out<I, O><<<(int)g, BLOCK, 0, s>>>(reinterpret_cast<const I*>(in), ldi, reinterpret_cast<O*>(out), rows, cols, status); \
  } while (0)
  if (it == Op::F32) { if (ot == Op::F32) CP(float, float); else CP(float, __nv_bfloat16); }
  else if (it == Op::F16) { if (ot == Op::F32) CP(__half, float); else CP(__half, __nv_bfloat16); }
  else { if (ot == Op::F32) CP(__nv_bfloat16, float); else CP(__nv_bfloat16, __nv_bfloat16); }
#undef CP
  return last();
}

}  // namespace muon

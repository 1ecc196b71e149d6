// Tensor-core GEMM for the Newton-Schulz chain on sm_100a.
//
// Persistent, warp-specialised kernel, one CTA per SM, 384 threads, in two
// forms sharing everything but the mainloop's data movement, each with
// BN = 256 or 128 tile columns:
//   PAIR = 1  one CTA computes a 128xBN tile: tcgen05.mma cta_group::1,
//             M = 128, N = BN; ring of 4 (BN 256) or 6 (BN 128) stages.
//   PAIR = 2  a cluster of two CTAs computes a 256xBN tile: the leader issues
//             tcgen05.mma cta_group::2, M = 256, N = BN, reading A's 128 rows
//             and B's BN/2 rows from each CTA's own shared memory; each CTA
//             TMA-loads only its halves into a ring of 6 (BN 256) or 8
//             (BN 128) stages, and the copy completions are counted on the
//             leader's barrier. MMA completions are signalled to both CTAs'
//             barriers.
// Roles:
//   warps 0, 3  TMA producers (one thread each: A boxes, B boxes), 128-byte swizzle
//   warp 1      MMA issuer (one thread of the leader), fp32 accumulators in TMEM
//   warp 2      allocates / frees the 512 TMEM columns (two 128xBN fp32
//               accumulators: the epilogue of tile i overlaps the mainloop of
//               tile i+1)
//   warps 4..11 epilogue, two warps per TMEM lane quarter, each owning BN/2
//               of the tile's columns: C blocks loaded (coalesced) before the
//               accumulator wait, 32x32 sub-tiles read from TMEM in the
//               m16n8 fragment layout, fused alpha*acc + beta*C + gamma*I,
//               one rounding to the stored type, then each 32x32 block is
//               staged with stmatrix in 64B-swizzled shared memory and
//               written by a TMA bulk tensor store (clipped at the matrix
//               edge). For symmetric outputs stmatrix.trans stages the
//               transpose, stored at the mirrored position; a block on the
//               diagonal is symmetrised in shared memory and stored once.
//
// Symmetric outputs ("2. Symmetric GEMM Kernels" of the Dion3 page: a
// triangular scheduler over lower tiles and a transposed-tile epilogue) are
// scheduled over the tiles that touch the lower triangle only.
//
// Small launches: a launch whose 256-column tiles leave CTAs (pairs) idle
// either splits K (symmetric X X^T with a long K: each tile's k-blocks in
// `splits` contiguous parts, one work unit each, raw fp32 accumulators to a
// partial buffer, then split_reduce_kernel sums the parts in a fixed order,
// applies the epilogue and writes both triangles, so the result is
// deterministic and exactly symmetric) or, when not split, runs on
// 128-column tiles if they all fit in one wave.
//
// Every wait is bounded (mbar_wait_bounded): on expiry the kernel records
// MUON_ERR_TIMEOUT, every role stops (in both CTAs of a pair), in-flight
// copies and MMAs are drained with bounded waits (for a pair, by counting
// what each producer issued: settle_pair_copies) and TMEM is freed before the
// CTA exits.
#include <algorithm>
#include <atomic>
#include <cstring>
#include <vector>
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace muon {

namespace tc {

constexpr int BM = 128, BK = 64;  // BM: rows per CTA
constexpr int BN_WIDE = 256;      // tile columns: 256, or 128 for launches too small to fill the GPU
constexpr int BN_NARROW = 128;
constexpr int UMMA_K = 16;
constexpr int EPI_WARP0 = 4;
constexpr int EPI_WARPS = 8;                       // two per TMEM lane quarter
constexpr int THREADS = 32 * (EPI_WARP0 + EPI_WARPS);
constexpr int TMEM_COLS = 512;
constexpr int EPI_BLOCK = 32 * 32 * 2;             // one staged 32x32 block of bf16/fp16, 64-byte rows
constexpr int EPI_BUF = 2 * EPI_BLOCK;             // per epilogue warp: direct block + mirrored block
// Drains (in-flight copies and MMAs before exit) use their own bound, so that
// a tiny configurable wait budget never lets a CTA exit with work in flight.
constexpr uint64_t DRAIN_NS = 1000000000ull;

template <int PAIR, int BN>
struct Cfg {
  static constexpr int STAGES = PAIR == 2 ? (BN == BN_WIDE ? 6 : 8) : (BN == BN_WIDE ? 4 : 6);
  static constexpr int A_STAGE = BM * BK * 2;                  // this CTA's 128 rows of A
  static constexpr int B_STAGE = (BN / PAIR) * BK * 2;         // this CTA's share of B's BN rows
  static constexpr int EPI_CHUNKS = BN / 32 / 2;               // 32-column chunks per epilogue warp
  static constexpr int TX_BYTES = PAIR * (A_STAGE + B_STAGE);  // per stage, both CTAs
  static constexpr int TILE_M = BM * PAIR;                     // rows of a (pair) tile
  static constexpr int SMEM = 1024 /*align slack*/ + STAGES * (A_STAGE + B_STAGE) + EPI_WARPS * EPI_BUF +
                              (2 * STAGES + 5) * 8 + 32;
  static_assert(SMEM <= 232448, "exceeds the opt-in shared memory of one sm_100 CTA");
};

// Distinct tensor maps of one launch, and the jobs of one launch. A job is
// one product of one shape group (all its matrices); a standalone launch
// holds up to kMaxGemmGroups jobs, a fused chain launch the products of a
// whole Newton-Schulz chain, phase after phase.
constexpr int kMaxMaps = 48;
constexpr int kMaxJobs = 72;

struct Job {
  void* D;
  const void* C;
  const float* scale;
  long long ldd, sD, ldc, sC;
  int M, N, K, batch;
  int a_mn, b_mn, sym;
  int n_fast;  // non-symmetric tile order: 1 = N fastest, 0 = M fastest
  int alpha_pow, beta_pow;
  float alpha, beta, gamma;
  int tiles_m, tiles_n, tiles_per_batch, tile_begin;  // tiles_per_batch counts (tile, split) units
  int splits, kbps;                                    // K split in parts of kbps k-blocks (1, all)
  int mA, mB, mD, mP;  // tensor maps: operands, output (32x32 boxes, 64-byte swizzle), split-K partials
  // fused chain: counters[done + b] counts the epilogue warps that finished
  // a tile of matrix b of this job; the job's tiles of matrix b wait until
  // counters[dep + b] reaches dep_target (the previous product of the same
  // matrix is complete). -1: no counter / no wait.
  int done, dep;
  unsigned dep_target;
};

struct Params {
  CUtensorMap maps[kMaxMaps];
  Job g[kMaxJobs];
  int ngroups;  // jobs
  int nmaps;
  int total_tiles;
  unsigned* counters;  // fused chain only
  int* status;
  unsigned long long timeout_ns;
};
static_assert(sizeof(Params) <= 32764, "kernel parameters are limited to 32764 bytes");

struct Tile {
  int g, b, m0, n0;  // m0: first row of the (pair) tile
  int kb0, kb1;      // k-blocks [kb0, kb1) of this work unit
  int split;
};

// Tiles (bn columns wide) of row block i (tile_m rows) that touch the lower triangle.
__host__ __device__ inline int sym_row_tiles(int i, int tiles_n, int tile_m, int bn) {
  int c = (i * tile_m + tile_m - 1) / bn + 1;
  return c < tiles_n ? c : tiles_n;
}

template <int PAIR, int BN>
__device__ inline Tile decode(const Params& p, int tile) {
  int lo = 0, hi = p.ngroups - 1;  // the last job whose first tile is <= tile
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.g[mid].tile_begin <= tile) lo = mid; else hi = mid - 1;
  }
  const int gi = lo;
  const Job& g = p.g[gi];
  int local = tile - g.tile_begin;
  int b = local / g.tiles_per_batch;
  int t = local - b * g.tiles_per_batch;
  const int split = t % g.splits;  // the parts of one tile run side by side
  t /= g.splits;
  int tm, tn;
  if (!g.sym) {
    // The fastest dimension cycles through the smaller operand's panels,
    // which stay in L2, while the slow one walks the larger operand's panels
    // so that each is read from memory once; the other order would re-read
    // the whole larger operand every wave (for a tall X times a square P,
    // far more than L2 holds).
    if (g.n_fast) {
      tn = t % g.tiles_n;
      tm = t / g.tiles_n;
    } else {
      tm = t % g.tiles_m;
      tn = t / g.tiles_m;
    }
  } else {
    int i = 0;
    for (;;) {
      int cnt = sym_row_tiles(i, g.tiles_n, Cfg<PAIR, BN>::TILE_M, BN);
      if (t < cnt) break;
      t -= cnt;
      ++i;
    }
    tm = i;
    tn = t;
  }
  const int nkb = (g.K + BK - 1) / BK;
  const int kb0 = split * g.kbps;
  const int kb1 = kb0 + g.kbps < nkb ? kb0 + g.kbps : nkb;
  return Tile{gi, b, tm * Cfg<PAIR, BN>::TILE_M, tn * BN, kb0, kb1, split};
}

__device__ __forceinline__ float powi(float s, int p) {
  float r = 1.f;
  for (int i = 0; i < p; ++i) r *= s;
  return r;
}

// Byte offset of element (r, c) of a staged 32x32 block with 64-byte rows
// and the TMA 64-byte swizzle (16-byte chunk index XOR (r / 2) % 4).
__device__ __forceinline__ uint32_t sw64(int r, int c) {
  return (uint32_t)(r * 64 + ((((c >> 3) ^ (r >> 1)) & 3) << 4) + ((c & 7) << 1));
}

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];"
               ::"l"(reinterpret_cast<uint64_t>(map)), "r"(src), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Wait until at most n (0..4) of this thread's most recent bulk groups are
// still in flight, i.e. every older group has completed.
__device__ __forceinline__ void bulk_wait_upto(int n) {
  switch (n) {
    case 4: asm volatile("cp.async.bulk.wait_group 4;" ::: "memory"); break;
    case 3: asm volatile("cp.async.bulk.wait_group 3;" ::: "memory"); break;
    case 2: asm volatile("cp.async.bulk.wait_group 2;" ::: "memory"); break;
    case 1: asm volatile("cp.async.bulk.wait_group 1;" ::: "memory"); break;
    default: asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); break;
  }
}
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Spin (bounded) until the phase with this parity completed; for drains.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, int* status) {
  const uint32_t addr = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(addr, parity)) {
    if (globaltimer_ns() - t0 > DRAIN_NS) {
      report(status, MUON_ERR_TIMEOUT);
      break;
    }
  }
}

// Fused chain: completion counters in global memory. A finished tile's
// stores are complete (bulk_wait0) and fenced for the async proxy before the
// release increment; a waiter's acquire load is followed by a proxy fence
// before its tensor copies read the data.
__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* a) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_gpu_add(unsigned* a, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }
__device__ __forceinline__ unsigned ld_relaxed_gpu(const unsigned* a) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
  return v;
}
// Acquire ordering after a relaxed load that observed a released value.
__device__ __forceinline__ void fence_acquire_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// Wait (bounded by budget) until matrix b of the job this one depends on is
// complete. Returns false when another role raised *abort, or on expiry, in
// which case it raises *abort and records MUON_ERR_TIMEOUT.
__device__ __forceinline__ bool wait_dep(const Params& p, const Job& g, int b, volatile int* abort, uint64_t budget) {
  if (g.dep < 0) return true;
  const unsigned* c = p.counters + g.dep + b;
  if (ld_acquire_gpu(c) < g.dep_target) {
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
      __nanosleep(100);
      if (ld_acquire_gpu(c) >= g.dep_target) break;
      if (*abort) return false;
      if (globaltimer_ns() - t0 > budget) {
        *abort = 1;
        report(p.status, MUON_ERR_TIMEOUT);
        return false;
      }
    }
  }
  fence_proxy_async_global();
  return true;
}

// CTA-pair early exit: wait until every operand copy that either CTA issued
// has landed, so that no copy writes into shared memory (or signals a
// barrier) after the pair has left. The copies of both CTAs complete on the
// leader's full[] barriers; `cnt` holds how many k-blocks each producer
// issued (leader A, leader B, follower A, follower B). A producer issues
// k-block j only after the MMAs consumed k-block j - STAGES, which needed
// every producer's copies of it, so all k-blocks before max(cnt) - STAGES
// have landed and each of the last STAGES k-blocks occupies its own stage.
// For those, the barrier is settled for the copies that were never issued
// (the missing transaction bytes, or the leader's arrival with the bytes that
// were issued), then waited on with the drain bound.
template <int PAIR, int BN>
__device__ void settle_pair_copies(uint64_t* full, const volatile int* cnt, int* status) {
  using Cf = Cfg<PAIR, BN>;
  constexpr int STAGES = Cf::STAGES;
  const int c[4] = {cnt[0], cnt[1], cnt[2], cnt[3]};
  const uint32_t bytes[4] = {Cf::A_STAGE, Cf::B_STAGE, Cf::A_STAGE, Cf::B_STAGE};
  int hi = 0;
  for (int x = 0; x < 4; ++x) hi = c[x] > hi ? c[x] : hi;
  for (int j = hi > STAGES ? hi - STAGES : 0; j < hi; ++j) {
    uint32_t issued = 0;
    for (int x = 0; x < 4; ++x)
      if (j < c[x]) issued += bytes[x];
    uint64_t* bar = &full[j % STAGES];
    if (j < c[0]) {
      // the leader's A producer arrived, expecting both CTAs' bytes
      if (issued < (uint32_t)Cf::TX_BYTES) mbar_complete_tx(bar, Cf::TX_BYTES - issued);
    } else {
      mbar_arrive_expect_tx(bar, issued);
    }
    drain_wait(bar, (uint32_t)((j / STAGES) & 1), status);
  }
}

template <typename T, int PAIR, int BN>
__global__ void __launch_bounds__(THREADS, 1) gemm_kernel(const __grid_constant__ Params p) {
  using Cf = Cfg<PAIR, BN>;
  constexpr int EPI_CHUNKS = Cf::EPI_CHUNKS;
  constexpr int STAGES = Cf::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Cf::A_STAGE;
  uint8_t* sEpi = sB + STAGES * Cf::B_STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + EPI_WARPS * EPI_BUF);
  uint64_t* full = bars;             // copies landed (the leader's counts both CTAs)
  uint64_t* empty = bars + STAGES;   // MMAs finished reading the stage
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = tfull + 2;      // the leader's counts both CTAs' epilogues
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* issued_cnt = reinterpret_cast<volatile int*>(tmem_slot + 2);  // pair: k-blocks per producer

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR == 2 ? cluster_rank() : 0;  // 0 = leader
  const int unit = PAIR == 2 ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int units = PAIR == 2 ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  // A role that stops early raises the other CTA's abort flag too, so that
  // the pair stops together.
  auto raise_peer = [&]() {
    if (PAIR == 2) st_cluster_u32(mapa_shared(smem_u32(const_cast<int*>(abort_flag)), rank ^ 1u), 1u);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], EPI_WARPS * PAIR);  // one arrival per epilogue warp of the pair
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    for (int i = 0; i < 4; ++i) issued_cnt[i] = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    if (PAIR == 2) {
      tmem_alloc_pair(tmem_slot, TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, TMEM_COLS);
      tmem_relinquish();
    }
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < p.nmaps; ++i) prefetch_tmap(&p.maps[i]);
  }
  tc_fence_before();
  __syncwarp();
  if (PAIR == 2) cluster_sync(); else __syncthreads();  // barriers initialised in both CTAs
  tc_fence_after();
  // The setup above overlaps the previous launch's tail; its outputs are
  // read (and the buffers it reads overwritten) only after this point.
  grid_dependency_wait();
  grid_dependents_launch();
  const uint32_t tmem_base = *tmem_slot;
  const uint64_t budget = p.timeout_ns;

  if ((warp == 0 || warp == 3) && lane == 0) {
    // ------------------------------------------------------------------
    // TMA producers (each CTA loads its own halves). Issuing a tensor copy
    // costs the issuing thread hundreds of cycles, so two threads in
    // different warps issue in parallel: warp 0 the A boxes (and the
    // leader's byte count), warp 3 the B boxes. Each of them has a box in
    // every k-block, so no stage phase can complete without both, and
    // neither can fall two phases behind the parity it waits on.
    // ------------------------------------------------------------------
    const bool issues_a = warp == 0;
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;
    // Fused chain: the dependency counter of the next tile is read (relaxed)
    // one tile ahead, so its latency hides behind this tile's copies; if it
    // was already complete then, an acquire fence stands in for the acquire
    // load, else the tile waits as usual.
    const unsigned* next_ctr = nullptr;
    unsigned next_val = 0;
    for (int tile = unit; tile < p.total_tiles; tile += units) {
      const Tile t = decode<PAIR, BN>(p, tile);
      const Job& g = p.g[t.g];
      const CUtensorMap* mapA = &p.maps[g.mA];
      const CUtensorMap* mapB = &p.maps[g.mB];
      const int am0 = t.m0 + (int)rank * BM;            // this CTA's rows of A
      const int bn0 = t.n0 + (int)rank * (BN / PAIR);   // this CTA's rows of B
      bool ok = true;
      if (g.dep >= 0) {
        if (next_ctr == p.counters + g.dep + t.b && next_val >= g.dep_target) {
          fence_acquire_gpu();
          fence_proxy_async_global();
        } else if (!wait_dep(p, g, t.b, abort_flag, budget)) {
          raise_peer();
          break;
        }
      }
      next_ctr = nullptr;
      if (tile + units < p.total_tiles) {
        const Tile tn = decode<PAIR, BN>(p, tile + units);
        const Job& gn = p.g[tn.g];
        if (gn.dep >= 0) {
          next_ctr = p.counters + gn.dep + tn.b;
          next_val = ld_relaxed_gpu(next_ctr);
        }
      }
      for (int kb = t.kb0; kb < t.kb1; ++kb) {
        if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, budget, p.status)) {
          raise_peer();
          ok = false;
          break;
        }
        if (issues_a && rank == 0) mbar_arrive_expect_tx(&full[stage], Cf::TX_BYTES);
        uint8_t* a = sA + stage * Cf::A_STAGE;
        uint8_t* b = sB + stage * Cf::B_STAGE;
        const int k0 = kb * BK;
        auto load = [&](void* dst, const CUtensorMap* m, int c0, int c1) {
          if (PAIR == 2) tma_load_3d_pair(dst, m, c0, c1, t.b, &full[stage]);
          else tma_load_3d(dst, m, c0, c1, t.b, &full[stage]);
        };
        if (issues_a) {
          if (!g.a_mn) {
            load(a, mapA, k0, am0);
          } else {
            load(a, mapA, am0, k0);
            load(a + 8192, mapA, am0 + 64, k0);
          }
        } else {
          if (!g.b_mn) {
            load(b, mapB, k0, bn0);
          } else {
#pragma unroll
            for (int j = 0; j < BN / PAIR / 64; ++j) load(b + j * 8192, mapB, bn0 + 64 * j, k0);
          }
        }
        ++issued;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
    }
    if (PAIR == 1) {
      // Drain: wait (bounded) until every copy issued into the ring landed.
      int n = issued < STAGES ? issued : STAGES;
      for (int i = 0; i < n; ++i) {
        if (--stage < 0) {
          stage = STAGES - 1;
          phase ^= 1;
        }
        drain_wait(&full[stage], phase, p.status);  // the most recent use of `stage`
      }
    } else {
      // The pair's copies complete on the leader's barriers: publish this
      // producer's k-block count in the leader's table; on an early exit the
      // leader settles and drains those barriers after the final cluster
      // barrier (settle_pair_copies).
      const uint32_t slot = smem_u32(const_cast<int*>(issued_cnt + 2 * rank + (issues_a ? 0 : 1)));
      st_cluster_u32(mapa_shared(slot, 0), (uint32_t)issued);
    }
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ------------------------------------------------------------------
    // MMA issuer (the leader issues for the pair)
    // ------------------------------------------------------------------
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
    constexpr int fmt = std::is_same<T, __nv_bfloat16>::value ? 1 : 0;
    bool ok = true;
    for (int tile = unit; tile < p.total_tiles && ok; tile += units) {
      const Tile t = decode<PAIR, BN>(p, tile);
      const Job& g = p.g[t.g];
      const uint32_t idesc = idesc_f16(fmt, g.a_mn, g.b_mn, BM * PAIR, BN);
      // K-major: 8-row groups 1024 B apart, one K step = 32 B inside the
      // swizzle atom. MN-major: 64-element MN atoms 8 KB apart (LBO), 8-row
      // K groups 1024 B apart (SBO), one K step of 16 rows = 2048 B.
      const uint32_t a_lbo = g.a_mn ? 8192u : 16u, b_lbo = g.b_mn ? 8192u : 16u;
      const uint32_t a_kstep = g.a_mn ? 2048u : 32u, b_kstep = g.b_mn ? 2048u : 32u;
      // descriptor fields other than the start address, fixed for the tile;
      // start addresses (>> 4) stay below 2^14 inside the 228 KB window
      const uint64_t a_hi = smem_desc_sw128(0, a_lbo, 1024), b_hi = smem_desc_sw128(0, b_lbo, 1024);
      if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1, abort_flag, budget, p.status)) {
        raise_peer();
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * BN;
      for (int kb = t.kb0; kb < t.kb1; ++kb) {
        if (!mbar_wait_bounded(&full[stage], phase, abort_flag, budget, p.status)) {
          raise_peer();
          ok = false;
          break;
        }
        // No tcgen05 fence here: the stage barrier completes only when the
        // copies' bytes have landed, and the MMAs that read them are issued
        // after the wait returns.
        const uint32_t a_lo = (a_base + stage * Cf::A_STAGE) >> 4, b_lo = (b_base + stage * Cf::B_STAGE) >> 4;
#pragma unroll
        for (int k = 0; k < BK / UMMA_K; ++k) {
          const uint64_t ad = a_hi | (uint64_t)(a_lo + k * (a_kstep >> 4));
          const uint64_t bd = b_hi | (uint64_t)(b_lo + k * (b_kstep >> 4));
          const bool accumulate = kb != t.kb0 || k != 0;
          if (PAIR == 2) umma_f16_pair(d_tmem, ad, bd, idesc, accumulate);
          else umma_f16(d_tmem, ad, bd, idesc, accumulate);
        }
        // frees the stage (in both CTAs) once these MMAs have read it
        if (PAIR == 2) umma_commit_pair(&empty[stage], 0x3); else umma_commit(&empty[stage]);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      // accumulator ready for the epilogue (of both CTAs)
      if (PAIR == 2) umma_commit_pair(&tfull[acc], 0x3); else umma_commit(&tfull[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    // Drain: every MMA issued completes (and every earlier completion signal
    // has arrived) before TMEM is freed.
    if (PAIR == 2) umma_commit_pair(drain, 0x3); else umma_commit(drain);
    drain_wait(drain, 0, p.status);
  } else if (PAIR == 2 && warp == 1 && lane == 0) {
    // the follower learns from the leader's drain signal that no MMA still
    // reads its shared memory or writes its TMEM
    drain_wait(drain, 0, p.status);
  } else if (warp >= EPI_WARP0) {
    // ------------------------------------------------------------------
    // Epilogue
    // ------------------------------------------------------------------
    const int e = warp - EPI_WARP0;
    const int q = warp & 3;   // TMEM lane quarter this warp may access
    const int half = e >> 2;  // which 128 of the tile's 256 columns it owns
    uint8_t* const sd = sEpi + e * EPI_BUF;  // staged direct block (1024-byte aligned)
    uint8_t* const sm = sd + EPI_BLOCK;       // staged mirrored block
    int acc = 0;
    uint32_t acc_phase = 0;
    // Fused chain (lane 0): the counter of this warp's last finished tile,
    // signalled once its stores have completed. It is signalled late, after
    // the next tile's stores are issued (their completion then overlaps that
    // work), but always before this warp blocks on anything, so no tile
    // waits on a signal held back by a waiting warp.
    int pending = -1;
    int groups = 0;  // bulk groups committed for the current tile
    auto signal = [&]() {
      fence_proxy_async_global();
      red_release_gpu_add(p.counters + pending, 1u);
      pending = -1;
    };
    auto flush = [&]() {
      if (pending >= 0) {
        bulk_wait0();
        signal();
      }
    };
    for (int tile = unit; tile < p.total_tiles; tile += units) {
      const Tile t = decode<PAIR, BN>(p, tile);
      const Job& g = p.g[t.g];
      const float s = g.scale ? g.scale[t.b] : 1.f;
      const float alpha = g.alpha * powi(s, g.alpha_pow);
      const float beta = g.beta * powi(s, g.beta_pow);
      const int r0 = t.m0 + (int)rank * BM + q * 32;
      const int cbase = t.n0 + half * (BN / 2);
      // The C blocks of all its chunks (and the scale above) are loaded
      // before waiting for the accumulator, so their latency overlaps that
      // wait. Loads are coalesced: load j of a chunk covers block rows
      // 8j..8j+7, four lanes per 64-byte row; the block is staged in shared
      // memory later and read back in the fragment layout with ldmatrix.
      uint4 cv[EPI_CHUNKS][4];
      const bool part = g.splits > 1;  // store the raw fp32 partial accumulator
      const bool want_c = g.beta != 0.f && !part;  // warp-uniform
      if (want_c && g.dep >= 0) {
        // C was written by an earlier product of the chain: wait for it here
        // too (these loads are issued before this tile's MMAs complete)
        bool dok = true;
        if (lane == 0) {
          if (ld_acquire_gpu(p.counters + g.dep + t.b) >= g.dep_target) {
            fence_proxy_async_global();
          } else {
            flush();  // this warp is about to wait: release its held signal first
            dok = wait_dep(p, g, t.b, abort_flag, budget);
          }
        }
        dok = __shfl_sync(0xffffffffu, dok, 0);
        __syncwarp();  // the other lanes' loads below are ordered after lane 0's acquire
        if (!dok) {
          if (lane == 0) raise_peer();
          break;
        }
      }
      if (want_c) {
        const T* cb = reinterpret_cast<const T*>(g.C) + (long long)t.b * g.sC + (lane & 3) * 8;
#pragma unroll
        for (int ch = 0; ch < EPI_CHUNKS; ++ch) {
          const int c0 = cbase + ch * 32;
          if (c0 < g.N && !(g.sym && c0 > r0 + 31)) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int cr = r0 + 8 * j + (lane >> 2);
              if (cr < g.M && MUON_IN_BOUNDS(c0 + (lane & 3) * 8 + 8 <= g.ldc, p.status))
                cv[ch][j] = __ldcg(reinterpret_cast<const uint4*>(cb + (long long)cr * g.ldc + c0));
            }
          }
        }
      }
      // every lane waits; the result is made warp-uniform so the warp-wide
      // tcgen05.ld below never runs with part of the warp gone
      if (lane == 0 && pending >= 0 && !mbar_try_wait(smem_u32(&tfull[acc]), acc_phase)) flush();
      const bool ok = mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, budget, p.status);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) raise_peer();
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int ch = 0; ch < EPI_CHUNKS; ++ch) {
        const int c0 = cbase + ch * 32;
        if (c0 >= g.N) break;                      // warp-uniform
        if (g.sym && c0 > r0 + 31) break;          // whole sub-tile above the diagonal
        const uint32_t tcol = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN + half * (BN / 2) + ch * 32;
        if (part) {
          uint32_t raw[32];
          tmem_ld_32x32(tcol, raw);
          tmem_wait_ld();
          // 32 fp32 of row `lane` fill one 128-byte row of the staged block
          // (128-byte swizzle: 16-byte chunk index XOR row % 8)
          if (lane == 0) bulk_wait_read0();
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 8; ++k)
            *reinterpret_cast<uint4*>(sd + lane * 128 + ((k ^ (lane & 7)) << 4)) =
                make_uint4(raw[4 * k], raw[4 * k + 1], raw[4 * k + 2], raw[4 * k + 3]);
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&p.maps[g.mP], smem_u32(sd), c0, r0, t.split * g.batch + t.b);
            bulk_commit();
            ++groups;
          }
          continue;
        }
        // The 32x32 block in the m16n8 fragment layout, as two 16-lane
        // halves: v[16h + r] is element (16h + 8*((r>>1)&1) + lane/4,
        // 8*(r>>2) + 2*(lane%4) + (r&1)) of the block. 8x8 matrix (h, s, i)
        // (rows 16h + 8s.., columns 8i..) is v[16h + 4i + 2s], v[16h + 4i + 2s + 1].
        float v[32];
        {
          uint32_t f0[16], f1[16];
          tmem_ld_16x256_x4(tcol, f0);
          tmem_ld_16x256_x4(tcol + (16u << 16), f1);
          tmem_wait_ld();
#pragma unroll
          for (int r = 0; r < 16; ++r) {
            v[r] = alpha * __uint_as_float(f0[r]);
            v[16 + r] = alpha * __uint_as_float(f1[r]);
          }
        }
        // the previous chunk's bulk stores must have finished reading the staging blocks
        if (lane == 0) bulk_wait_read0();
        __syncwarp();
        const uint32_t sd_a = smem_u32(sd), sm_a = smem_u32(sm);
        if (want_c) {
          // C block through the mirror staging block (64-byte swizzle):
          // written as loaded, read back in the fragment layout
#pragma unroll
          for (int j = 0; j < 4; ++j) *reinterpret_cast<uint4*>(sm + sw64(8 * j + (lane >> 2), (lane & 3) * 8)) = cv[ch][j];
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // k = 2h + s
            uint32_t cf[4];
            ldsm_x4(sm_a + sw64(16 * (k >> 1) + 8 * (k & 1) + (lane & 7), 8 * (lane >> 3)), cf);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 f = Elem<T>::unpack2(cf[i]);
              const int x = 16 * (k >> 1) + 4 * i + 2 * (k & 1);
              v[x] += beta * f.x;
              v[x + 1] += beta * f.y;
            }
          }
          __syncwarp();  // the C block is read before the staging block is overwritten
        }
        if (g.gamma != 0.f) {
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            const int rr = 16 * (x >> 4) + 8 * ((x >> 1) & 1) + (lane >> 2);
            const int cc = 8 * ((x >> 2) & 3) + 2 * (lane & 3) + (x & 1);
            if (r0 + rr == c0 + cc) v[x] += g.gamma;
          }
        }
        // Round once to the stored type: the direct and mirrored copies of an
        // element are the same bits, so D is exactly symmetric.
        uint32_t pk[16];  // pk[4k + i]: matrix (h, s, i) with k = 2h + s
#pragma unroll
        for (int k = 0; k < 4; ++k)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int x = 16 * (k >> 1) + 4 * i + 2 * (k & 1);
            pk[4 * k + i] = Elem<T>::pack2(v[x], v[x + 1]);
          }
        const bool diag = g.sym && c0 == r0;   // the block straddles the diagonal
        const bool mirror = g.sym && r0 > c0;  // strictly lower: also store its transpose
#pragma unroll
        for (int k = 0; k < 4; ++k)
          stsm_x4(sd_a + sw64(16 * (k >> 1) + 8 * (k & 1) + (lane & 7), 8 * (lane >> 3)), pk[4 * k], pk[4 * k + 1],
                  pk[4 * k + 2], pk[4 * k + 3]);
        if (diag || mirror) {
          // the transposed block: matrix (h, s, i) lands at rows 8i.., columns 16h + 8s..
#pragma unroll
          for (int k = 0; k < 4; ++k)
            stsm_x4_trans(sm_a + sw64(lane, 16 * (k >> 1) + 8 * (k & 1)), pk[4 * k], pk[4 * k + 1], pk[4 * k + 2],
                          pk[4 * k + 3]);
        }
        if (diag) {
          // symmetrise the diagonal block: above the diagonal (row < col)
          // takes the value computed below it, from the transposed block
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j > lane)
              *reinterpret_cast<uint16_t*>(sd + sw64(lane, j)) = *reinterpret_cast<const uint16_t*>(sm + sw64(lane, j));
        }
        fence_async_smem();  // generic-proxy writes become visible to the bulk copy
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&p.maps[g.mD], smem_u32(sd), c0, r0, t.b);
          if (mirror) tma_store_3d(&p.maps[g.mD], smem_u32(sm), r0, c0, t.b);
          bulk_commit();
          ++groups;
        }
      }
      // this warp's TMEM reads are done: release the accumulator (to the
      // leader's barrier; the MMAs that overwrite it wait there)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR == 2 && rank != 0) mbar_arrive_remote(mapa_shared(smem_u32(&tempty[acc]), 0));
        else mbar_arrive(&tempty[acc]);
        if (g.done >= 0) {
          // fused chain: the previous tile's stores are older than this
          // tile's `groups` bulk groups; once they completed, signal it
          if (pending >= 0) {
            bulk_wait_upto(groups);
            signal();
          }
          pending = g.done + t.b;
        }
        groups = 0;
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    if (lane == 0) {
      bulk_wait0();  // every staged block written before the CTA exits
      if (pending >= 0) signal();
    }
  }

  tc_fence_before();
  __syncwarp();
  if (PAIR == 2) cluster_sync(); else __syncthreads();  // no CTA leaves while its pair still signals it
  tc_fence_after();
  if (PAIR == 2) {
    // every producer has published its count and every early stop has
    // reached both abort flags; the follower stays resident (its shared
    // memory receives its own copies) until the leader's drain ends
    if (rank == 0 && threadIdx.x == 0 && *abort_flag) settle_pair_copies<PAIR, BN>(full, issued_cnt, p.status);
    __syncwarp();
    cluster_sync();
  }
  if (warp == 2) {
    if (PAIR == 2) tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Split-K reduction: D = alpha*s^alpha_pow*sum_parts + beta*s^beta_pow*C +
// gamma*I over the lower triangle of symmetric n x n outputs, parts summed in
// increasing order; each 32x32 lower block is written at its place and, off
// the diagonal, transposed at the mirrored place (a diagonal block takes its
// upper half from its lower half), so D is exactly symmetric.
// ---------------------------------------------------------------------------

struct SplitGroup {
  const float* part;  // [splits][batch][n][ldp]
  void* D;
  const void* C;
  const float* scale;
  long long ldp, ldd, sD, ldc, sC;
  int n, batch, splits, nb32, blocks_per_batch, block_begin;
  int alpha_pow, beta_pow;
  float alpha, beta, gamma;
};

struct SplitParams {
  SplitGroup g[kMaxGemmGroups];
  int ngroups;
  int* status;  // index checks of the bounds-checked build report here
};

constexpr int RED_THREADS = 256;  // one 32x32 block: 32 rows x 8 groups of 4 columns
constexpr int RED_MAX_PARTS = 8;

template <typename T>
__global__ void __launch_bounds__(RED_THREADS) split_reduce_kernel(const __grid_constant__ SplitParams p) {
  __shared__ float tile[32][33];
  grid_dependency_wait();
  int gi = 0;
  while (gi + 1 < p.ngroups && (int)blockIdx.x >= p.g[gi + 1].block_begin) ++gi;
  const SplitGroup& g = p.g[gi];
  const int local = (int)blockIdx.x - g.block_begin;
  const int b = local / g.blocks_per_batch;
  const int k = local - b * g.blocks_per_batch;
  // lower-triangle block k, row by row: (bi, bj) with bj <= bi
  int bi = (int)((sqrtf(8.f * (float)k + 1.f) - 1.f) * 0.5f);
  while (bi * (bi + 1) / 2 > k) --bi;
  while ((bi + 1) * (bi + 2) / 2 <= k) ++bi;
  const int bj = k - bi * (bi + 1) / 2;
  const int rr = threadIdx.x >> 3, cg = (threadIdx.x & 7) * 4;  // this thread: row rr, columns cg..cg+3
  const int r = bi * 32 + rr, c = bj * 32 + cg;
  float v[4] = {0.f, 0.f, 0.f, 0.f};
  if (r < g.n && MUON_IN_BOUNDS(c + 3 < g.ldp && g.splits <= RED_MAX_PARTS, p.status)) {
    // every part's 4 values in flight at once (the rows' padding keeps the
    // 16-byte loads inside the buffer); then summed in part order
    const float* pp = g.part + ((long long)b * g.n + r) * g.ldp + c;
    const long long pstride = (long long)g.batch * g.n * g.ldp;
    float4 pv[RED_MAX_PARTS];
#pragma unroll
    for (int sp = 0; sp < RED_MAX_PARTS; ++sp)
      if (sp < g.splits) pv[sp] = *reinterpret_cast<const float4*>(pp + sp * pstride);
    float4 acc = pv[0];
#pragma unroll
    for (int sp = 1; sp < RED_MAX_PARTS; ++sp)
      if (sp < g.splits) {
        acc.x += pv[sp].x;
        acc.y += pv[sp].y;
        acc.z += pv[sp].z;
        acc.w += pv[sp].w;
      }
    const float sc = g.scale ? g.scale[b] : 1.f;
    const float alpha = g.alpha * powi(sc, g.alpha_pow);
    const float beta = g.beta * powi(sc, g.beta_pow);
    v[0] = alpha * acc.x;
    v[1] = alpha * acc.y;
    v[2] = alpha * acc.z;
    v[3] = alpha * acc.w;
    if (g.beta != 0.f) {
      const T* cr = reinterpret_cast<const T*>(g.C) + (long long)b * g.sC + (long long)r * g.ldc + c;
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] += beta * Elem<T>::to_f(cr[j]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (r == c + j) v[j] += g.gamma;
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) tile[rr][cg + j] = Elem<T>::to_f(Elem<T>::from_f(v[j]));  // rounded once
  __syncthreads();
  T* D = reinterpret_cast<T*>(g.D) + (long long)b * g.sD;
  if (r < g.n) {
    // direct block; a diagonal block takes its upper half from its lower half
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int cc = cg + j;
      const float x = (bi == bj && cc > rr) ? tile[cc][rr] : tile[rr][cc];
      if (c + j < g.n) D[(long long)r * g.ldd + c + j] = Elem<T>::from_f(x);
    }
  }
  if (bi != bj) {
    // mirrored block: D[bj*32 + rr][bi*32 + cg + j] = value at (bi*32 + cg + j, bj*32 + rr)
    const int rm = bj * 32 + rr, cm = bi * 32 + cg;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (rm < g.n && cm + j < g.n) D[(long long)rm * g.ldd + cm + j] = Elem<T>::from_f(tile[cg + j][rr]);
  }
}

}  // namespace tc

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D map over [batch][outer][inner] with row stride ld and batch stride
// (elements), box {box_inner, box_outer, 1}, zero fill out of range (loads)
// and clipping (stores).
bool make_map(CUtensorMap* m, Op t, const void* base, int64_t inner, int64_t outer, int64_t batch, int64_t ld,
              int64_t bstride, int box_outer, int box_inner = 64,
              CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const CUtensorMapDataType dt = t == Op::BF16  ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                 : t == Op::F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const cuuint64_t es = op_size(t);
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)outer, (cuuint64_t)batch};
  cuuint64_t strides[2] = {(cuuint64_t)ld * es, (cuuint64_t)(batch > 1 ? bstride : ld * outer) * es};
  cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)box_outer, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

constexpr int kMaxDevices = 64;

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) {
    cudaGetLastError();
    d = 0;
  }
  return d;
}

// Co-resident CTAs (PAIR = 1) or clusters (PAIR = 2) of the persistent
// kernel on the current device; 0 if its attributes cannot be set. The
// shared-memory attribute is set, and the count taken, once per device.
template <typename T, int PAIR, int BN>
int max_units() {
  static std::mutex mu;
  static int per_device[kMaxDevices];  // 0: not set up on that device yet
  const int dev = current_device();
  std::lock_guard<std::mutex> lock(mu);
  int& units = per_device[dev];
  const void* fn = (const void*)tc::gemm_kernel<T, PAIR, BN>;
  if (units == 0) {
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::Cfg<PAIR, BN>::SMEM) != cudaSuccess)
      return 0;
    int u = num_sms() / PAIR;
    if (PAIR == 2) {
      // not every SM may have a free partner in its GPC: launch only as many
      // persistent pairs as can run at once
      cudaLaunchConfig_t q = {};
      q.gridDim = dim3(2 * u);
      q.blockDim = dim3(tc::THREADS);
      q.dynamicSmemBytes = tc::Cfg<PAIR, BN>::SMEM;
      cudaLaunchAttribute a[1];
      a[0].id = cudaLaunchAttributeClusterDimension;
      a[0].val.clusterDim.x = 2;
      a[0].val.clusterDim.y = 1;
      a[0].val.clusterDim.z = 1;
      q.attrs = a;
      q.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, fn, &q) == cudaSuccess && clusters > 0 && clusters < u)
        u = clusters;
      cudaGetLastError();
    }
    units = u;
  }
  return units;
}

template <typename T, int PAIR, int BN>
muon_status launch(const tc::Params& p, int total_tiles, int max_units, cudaStream_t s) {
  const int units = total_tiles < max_units ? total_tiles : max_units;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(units * PAIR);
  cfg.blockDim = dim3(tc::THREADS);
  cfg.dynamicSmemBytes = tc::Cfg<PAIR, BN>::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = PAIR;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, tc::gemm_kernel<T, PAIR, BN>, p) == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}

template <typename T>
muon_status launch_reduce(const tc::SplitParams& p, int blocks, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(tc::RED_THREADS);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tc::split_reduce_kernel<T>, p) == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}

int g_pair_mode = 2;  // 2: CTA-pair kernel, 1: single-CTA kernel

// Split K only while every part keeps at least kMinSplitKb k-blocks (64 K
// each), so the partial traffic stays small against the part's MMAs.
constexpr int kMaxSplits = 8;
static_assert(kMaxSplits <= tc::RED_MAX_PARTS, "the reduction holds every part in registers");
constexpr int kMinSplitKb = 32;

int sym_tiles(int64_t n, int tile_m, int bn) {
  const int tm = (int)((n + tile_m - 1) / tile_m), tn = (int)((n + bn - 1) / bn);
  int c = 0;
  for (int i = 0; i < tm; ++i) c += tc::sym_row_tiles(i, tn, tile_m, bn);
  return c;
}

// Tiles of one matrix of a group at tile width bn.
int desc_tiles(const GemmDesc& d, int tile_m, int bn) {
  return d.sym ? sym_tiles(d.M, tile_m, bn) : ((d.M + tile_m - 1) / tile_m) * ((d.N + bn - 1) / bn);
}

// Parts for a symmetric launch of `tiles` tiles over `units` CTAs (pairs)
// with nkb k-blocks per tile; sets *kbps to the k-blocks per part.
int split_parts(int tiles, int units, int nkb, int* kbps) {
  *kbps = nkb;
  if (tiles <= 0 || tiles >= units) return 1;
  int want = units / tiles;
  if (want > kMaxSplits) want = kMaxSplits;
  if (want < 2) return 1;
  int per = (nkb + want - 1) / want;
  if (per < kMinSplitKb) per = kMinSplitKb;
  const int parts = (nkb + per - 1) / per;  // every part has at least one k-block
  if (parts < 2) return 1;
  *kbps = per;
  return parts;
}

}  // namespace

int num_sms() {
  static std::atomic<int> per_device[kMaxDevices];  // 0: not queried yet
  const int dev = current_device();
  int n = per_device[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = 148;  // no device here (workspace planning on a host without a GPU)
    }
    per_device[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

void set_gemm_pair_mode(int pair) { g_pair_mode = pair == 1 ? 1 : 2; }

namespace {
int g_chain_mode = 0;
}
void set_gemm_chain(int on) { g_chain_mode = on ? 1 : 0; }
int gemm_chain() { return g_chain_mode; }

size_t tc_split_scratch(int64_t n, int64_t K, int count) {
  size_t best = 0;
  const int nkb = (int)((K + tc::BK - 1) / tc::BK);
  for (int pair = 1; pair <= 2; ++pair) {
    // num_sms() / pair bounds the co-resident units from above, so the
    // reservation covers every launch this group takes part in
    int kbps = 0;
    const int parts = split_parts(count * sym_tiles(n, tc::BM * pair, tc::BN_WIDE), num_sms() / pair, nkb, &kbps);
    if (parts > 1) {
      const size_t b = (size_t)parts * count * n * pad_ld(n) * sizeof(float);
      if (b > best) best = b;
    }
  }
  return best;
}

template <int BN>
int units_for(Op t, int pair) {
  if (pair == 2) return t == Op::BF16 ? max_units<__nv_bfloat16, 2, BN>() : max_units<__half, 2, BN>();
  return t == Op::BF16 ? max_units<__nv_bfloat16, 1, BN>() : max_units<__half, 1, BN>();
}

template <int BN>
muon_status launch_for(Op t, int pair, const tc::Params& p, int total, int units, cudaStream_t s) {
  if (pair == 2)
    return t == Op::BF16 ? launch<__nv_bfloat16, 2, BN>(p, total, units, s) : launch<__half, 2, BN>(p, total, units, s);
  return t == Op::BF16 ? launch<__nv_bfloat16, 1, BN>(p, total, units, s) : launch<__half, 1, BN>(p, total, units, s);
}

namespace {

// Tensor maps of one launch, each distinct map once (a fused chain reuses
// the same few buffers in many products).
struct MapTable {
  struct Key {
    const void* base;
    int64_t inner, outer, batch, ld, bstride;
    int box_outer, box_inner, swz, dt;
    bool operator==(const Key& o) const {
      return base == o.base && inner == o.inner && outer == o.outer && batch == o.batch && ld == o.ld &&
             bstride == o.bstride && box_outer == o.box_outer && box_inner == o.box_inner && swz == o.swz &&
             dt == o.dt;
    }
  };
  tc::Params* p;
  Key keys[tc::kMaxMaps];
  // Index of the map (made on first use); -1 if it cannot be made or the
  // table is full.
  int get(Op t, const void* base, int64_t inner, int64_t outer, int64_t batch, int64_t ld, int64_t bstride,
          int box_outer, int box_inner = 64, CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
    const Key k{base, inner, outer, batch, ld, bstride, box_outer, box_inner, (int)swz, (int)t};
    for (int i = 0; i < p->nmaps; ++i)
      if (keys[i] == k) return i;
    if (p->nmaps >= tc::kMaxMaps) return -1;
    if (!make_map(&p->maps[p->nmaps], t, base, inner, outer, batch, ld, bstride, box_outer, box_inner, swz)) return -1;
    keys[p->nmaps] = k;
    return p->nmaps++;
  }
};

// Tensor maps and scalars of one job at tile width bn, K in `parts` parts of
// `kbps` k-blocks. Returns false if a map cannot be made or the table is full.
bool fill_job(tc::Job& g, const GemmDesc& d, Op t, int pair, int bn, int parts, int kbps, MapTable& mt) {
  const int tile_m = tc::BM * pair;
  // A operand source: K-major [M][K], MN-major [K][M]; 128 rows per CTA.
  // B operand source: K-major [N][K], MN-major [K][N]; bn / pair rows per CTA.
  g.mA = d.a_mn ? mt.get(t, d.A, d.M, d.K, d.batch, d.lda, d.strideA, 64)
                : mt.get(t, d.A, d.K, d.M, d.batch, d.lda, d.strideA, tc::BM);
  g.mB = d.b_mn ? mt.get(t, d.B, d.N, d.K, d.batch, d.ldb, d.strideB, 64)
                : mt.get(t, d.B, d.K, d.N, d.batch, d.ldb, d.strideB, bn / pair);
  g.mD = mt.get(t, d.D, d.N, d.M, d.batch, d.ldd, d.strideD, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
  g.mP = -1;
  if (parts > 1) {
    const int64_t ldp = pad_ld(d.N);
    g.mP = mt.get(Op::F32, d.part, d.N, d.M, (int64_t)parts * d.batch, ldp, (int64_t)d.M * ldp, 32, 32);
    if (g.mP < 0) return false;
  }
  if (g.mA < 0 || g.mB < 0 || g.mD < 0) return false;
  g.D = d.D;
  g.C = d.C;
  g.scale = d.scale;
  g.ldd = d.ldd;
  g.sD = d.strideD;
  g.ldc = d.ldc;
  g.sC = d.strideC;
  g.M = d.M;
  g.N = d.N;
  g.K = d.K;
  g.batch = d.batch;
  g.a_mn = d.a_mn;
  g.b_mn = d.b_mn;
  g.sym = d.sym;
  g.n_fast = !d.sym && d.N < d.M ? 1 : 0;  // B (N x K) is the smaller operand
  g.alpha_pow = d.alpha_pow;
  g.beta_pow = d.beta_pow;
  g.alpha = d.alpha;
  g.beta = d.beta;
  g.gamma = d.gamma;
  g.tiles_m = (d.M + tile_m - 1) / tile_m;
  g.tiles_n = (d.N + bn - 1) / bn;
  g.tiles_per_batch = desc_tiles(d, tile_m, bn) * parts;
  g.splits = parts;
  g.kbps = kbps;
  g.done = -1;
  g.dep = -1;
  g.dep_target = 0;
  return true;
}

muon_status check_desc(const GemmDesc& d) {
  if (d.ldd % 64 || (d.beta != 0.f && d.ldc % 64)) return MUON_ERR_INVALID_ARG;
  if (d.sym && d.M != d.N) return MUON_ERR_INVALID_ARG;
  return MUON_OK;
}

bool has_work(const GemmDesc& d) { return d.batch > 0 && d.M > 0 && d.N > 0 && d.K > 0; }

// Work accounting of one job (dense, symmetric-once and executed FLOPs).
void count_job(const tc::Job& g, int tile_m, int bn) {
  Counters& cn = counters();
  const double mnk = (double)g.M * g.N * g.K * g.batch;
  cn.flops_dense += 2.0 * mnk;
  cn.flops_sym += g.sym ? mnk : 2.0 * mnk;
  cn.flops_exec += 2.0 * tile_m * bn * (double)g.K * (g.tiles_per_batch / g.splits) * g.batch;
}

}  // namespace

muon_status tc_gemm(Op t, const GemmDesc* gd, int ngroups, int* status, uint64_t timeout_ns, cudaStream_t s) {
  if (ngroups < 1 || ngroups > kMaxGemmGroups || (t != Op::BF16 && t != Op::F16)) return MUON_ERR_INVALID_ARG;
  const int pair = g_pair_mode;
  const int tile_m = tc::BM * pair;
  int units = units_for<tc::BN_WIDE>(t, pair);
  if (units <= 0) return MUON_ERR_CUDA;

  // the groups that have work, their tile counts at the wide tile width,
  // and the split of K where a symmetric launch leaves CTAs (pairs) idle
  const GemmDesc* src[kMaxGemmGroups];
  int parts[kMaxGemmGroups], kbps[kMaxGemmGroups];
  int ng = 0, total_wide = 0;
  for (int i = 0; i < ngroups; ++i) {
    const GemmDesc& d = gd[i];
    if (!has_work(d)) continue;
    const muon_status c = check_desc(d);
    if (c != MUON_OK) return c;
    src[ng++] = &d;
    total_wide += desc_tiles(d, tile_m, tc::BN_WIDE) * d.batch;
  }
  if (ng == 0) return MUON_OK;
  bool any_split = false;
  for (int i = 0; i < ng; ++i) {
    const GemmDesc& d = *src[i];
    const int nkb = (d.K + tc::BK - 1) / tc::BK;
    parts[i] = 1;
    kbps[i] = nkb;
    if (!d.sym || !d.part) continue;
    int per = 0;
    const int n = split_parts(total_wide, units, nkb, &per);
    if (n < 2 || (size_t)n * d.batch * d.N * pad_ld(d.N) * sizeof(float) > d.part_bytes) continue;
    parts[i] = n;
    kbps[i] = per;
    any_split = true;
  }
  // A launch that still leaves CTAs (pairs) idle and is not split takes
  // 128-column tiles when they all fit in one wave: twice the tiles, each
  // with half the MMAs and half the epilogue.
  int bn = tc::BN_WIDE;
  if (!any_split && total_wide < units) {
    int total_narrow = 0;
    for (int i = 0; i < ng; ++i) total_narrow += desc_tiles(*src[i], tile_m, tc::BN_NARROW) * src[i]->batch;
    const int units_narrow = units_for<tc::BN_NARROW>(t, pair);
    if (units_narrow <= 0) return MUON_ERR_CUDA;
    if (total_narrow > total_wide && total_narrow <= units_narrow) {
      bn = tc::BN_NARROW;
      units = units_narrow;
    }
  }

  static thread_local tc::Params p;  // ~20 KB: kept off the stack
  memset(&p, 0, sizeof(p));
  static thread_local MapTable mt;
  mt.p = &p;
  tc::SplitParams sp;
  memset(&sp, 0, sizeof(sp));
  int red_blocks = 0;
  for (int i = 0; i < ng; ++i) {
    const GemmDesc& d = *src[i];
    tc::Job& g = p.g[i];
    if (!fill_job(g, d, t, pair, bn, parts[i], kbps[i], mt)) return MUON_ERR_CUDA;
    if (parts[i] < 2) continue;
    tc::SplitGroup& r = sp.g[sp.ngroups++];
    r.part = d.part;
    r.D = d.D;
    r.C = d.C;
    r.scale = d.scale;
    r.ldp = pad_ld(d.N);
    r.ldd = d.ldd;
    r.sD = d.strideD;
    r.ldc = d.ldc;
    r.sC = d.strideC;
    r.n = d.N;
    r.batch = d.batch;
    r.splits = parts[i];
    r.nb32 = (d.N + 31) / 32;
    r.blocks_per_batch = r.nb32 * (r.nb32 + 1) / 2;
    r.block_begin = red_blocks;
    r.alpha_pow = d.alpha_pow;
    r.beta_pow = d.beta_pow;
    r.alpha = d.alpha;
    r.beta = d.beta;
    r.gamma = d.gamma;
    red_blocks += r.blocks_per_batch * d.batch;
    // the GEMM stores raw accumulators; the reduction applies the epilogue
    g.alpha = 1.f;
    g.alpha_pow = 0;
    g.beta = 0.f;
    g.gamma = 0.f;
  }
  int total = 0;
  for (int i = 0; i < ng; ++i) {
    p.g[i].tile_begin = total;
    total += p.g[i].tiles_per_batch * p.g[i].batch;
  }
  p.ngroups = ng;
  p.total_tiles = total;
  p.counters = nullptr;
  p.status = status;
  p.timeout_ns = timeout_ns;
  sp.status = status;

  Counters& cn = counters();
  cn.launches += sp.ngroups ? 2 : 1;
  cn.gemm_launches += 1;
  for (int i = 0; i < ng; ++i) count_job(p.g[i], tile_m, bn);
  const muon_status r = bn == tc::BN_WIDE ? launch_for<tc::BN_WIDE>(t, pair, p, total, units, s)
                                          : launch_for<tc::BN_NARROW>(t, pair, p, total, units, s);
  if (r != MUON_OK || sp.ngroups == 0) return r;
  return t == Op::BF16 ? launch_reduce<__nv_bfloat16>(sp, red_blocks, s) : launch_reduce<__half>(sp, red_blocks, s);
}

size_t tc_chain_counter_words(int nphase, int total_batch) { return (size_t)nphase * total_batch; }

muon_status tc_chain(Op t, const GemmDesc* descs, int nphase, int ngroups, unsigned* ctr, int* status,
                     uint64_t timeout_ns, cudaStream_t s) {
  if (nphase < 1 || ngroups < 1 || ngroups > kMaxGemmGroups || (t != Op::BF16 && t != Op::F16) || !ctr)
    return MUON_ERR_INVALID_ARG;
  const int pair = g_pair_mode;
  const int tile_m = tc::BM * pair;
  const int units_w = units_for<tc::BN_WIDE>(t, pair), units_n = units_for<tc::BN_NARROW>(t, pair);
  if (units_w <= 0 || units_n <= 0) return MUON_ERR_CUDA;
  int goff[kMaxGemmGroups + 1];
  goff[0] = 0;
  for (int i = 0; i < ngroups; ++i) {
    for (int k = 0; k < nphase; ++k) {
      const GemmDesc& d = descs[k * ngroups + i];
      if (!has_work(d) || d.batch != descs[i].batch) return MUON_ERR_INVALID_ARG;
      const muon_status c = check_desc(d);
      if (c != MUON_OK) return c;
    }
    goff[i + 1] = goff[i] + descs[i].batch;
  }
  const int total_batch = goff[ngroups];

  // Tile width per product, by the rule of the standalone launches: 128
  // columns when 256-column tiles leave CTAs (pairs) idle and the narrow
  // tiles still fit in one wave. Consecutive products of one width share a
  // launch; a change of width starts the next launch.
  // A product that the standalone launch would split along K (an X X^T
  // with a long K and fewer tiles than CTA pairs) runs as that split launch
  // (bn_of = 0): the chain stops before it and resumes after it.
  std::vector<int> bn_of(nphase);
  for (int k = 0; k < nphase; ++k) {
    int tw = 0, tn = 0;
    for (int i = 0; i < ngroups; ++i) {
      const GemmDesc& d = descs[k * ngroups + i];
      tw += desc_tiles(d, tile_m, tc::BN_WIDE) * d.batch;
      tn += desc_tiles(d, tile_m, tc::BN_NARROW) * d.batch;
    }
    bool split = false;
    for (int i = 0; i < ngroups; ++i) {
      const GemmDesc& d = descs[k * ngroups + i];
      int per = 0;
      const int parts = d.sym && d.part ? split_parts(tw, units_w, (d.K + tc::BK - 1) / tc::BK, &per) : 1;
      split = split || (parts > 1 && (size_t)parts * d.batch * d.N * pad_ld(d.N) * sizeof(float) <= d.part_bytes);
    }
    bn_of[k] = split ? 0 : (tw < units_w && tn > tw && tn <= units_n) ? tc::BN_NARROW : tc::BN_WIDE;
  }

  if (cudaMemsetAsync(ctr, 0, tc_chain_counter_words(nphase, total_batch) * sizeof(unsigned), s) != cudaSuccess)
    return MUON_ERR_CUDA;
  static thread_local tc::Params p;
  static thread_local MapTable mt;
  mt.p = &p;
  Counters& cn = counters();
  int k = 0;
  while (k < nphase) {
    if (bn_of[k] == 0) {
      const muon_status r = tc_gemm(t, descs + k * ngroups, ngroups, status, timeout_ns, s);
      if (r != MUON_OK) return r;
      ++k;
      continue;
    }
    // one launch: as many whole phases of one tile width as its jobs and
    // tensor maps allow
    memset(&p, 0, sizeof(p));
    const int k0 = k;
    const int bn = bn_of[k0];
    const int units = bn == tc::BN_NARROW ? units_n : units_w;
    for (; k < nphase; ++k) {
      if (bn_of[k] != bn || p.ngroups + ngroups > tc::kMaxJobs) break;
      const int nmaps0 = p.nmaps;
      bool ok = true;
      for (int i = 0; i < ngroups && ok; ++i) {
        tc::Job& g = p.g[p.ngroups + i];
        ok = fill_job(g, descs[k * ngroups + i], t, pair, bn, 1, (descs[k * ngroups + i].K + tc::BK - 1) / tc::BK,
                      mt);
        g.done = k * total_batch + goff[i];
        if (k > k0) {
          // the previous product of the same matrices, in this launch
          const tc::Job& prev = p.g[p.ngroups - ngroups + i];
          g.dep = prev.done;
          g.dep_target = (unsigned)prev.tiles_per_batch * tc::EPI_WARPS * pair;
        }
      }
      if (!ok) {
        p.nmaps = nmaps0;  // the table is full: this phase starts the next launch
        if (k == k0) return MUON_ERR_CUDA;
        break;
      }
      p.ngroups += ngroups;
    }
    int total = 0;
    for (int j = 0; j < p.ngroups; ++j) {
      p.g[j].tile_begin = total;
      total += p.g[j].tiles_per_batch * p.g[j].batch;
      count_job(p.g[j], tile_m, bn);
    }
    p.total_tiles = total;
    p.counters = ctr;
    p.status = status;
    p.timeout_ns = timeout_ns;
    cn.launches += 1;
    cn.gemm_launches += 1;
    const muon_status r = bn == tc::BN_WIDE ? launch_for<tc::BN_WIDE>(t, pair, p, total, units, s)
                                            : launch_for<tc::BN_NARROW>(t, pair, p, total, units, s);
    if (r != MUON_OK) return r;
  }
  return MUON_OK;
}

}  // namespace muon

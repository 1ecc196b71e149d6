// select_rows_noalloc: the Dion3 row selection without a caller workspace.
//
// Some callers cannot allocate device memory at the point where they need a
// selection: code running inside a memory pool that is already carved up, a
// runtime that forbids cudaMalloc after start-up (allocation can synchronise
// the device and fragment a pool), or a C host with no allocator of its own.
// This entry point takes only its inputs and outputs. Its scratch (the
// per-row fp64 keys and sums of squares) lives in a file-scope __device__
// array of fixed size, which every GPU that loads this library holds until
// the process exits.
#include <mutex>

#include "internal.h"
#include "rowops.cuh"

namespace muon {
namespace {

constexpr int64_t kNoAllocMaxRows = 65536;
constexpr size_t kHeaderBytes = 256;  // s and xscale outputs of the selection kernel
constexpr size_t kScratchBytes = kHeaderBytes + 2 * kNoAllocMaxRows * sizeof(double);

// 1 MiB + 256 B of device memory per GPU: [s, xscale | sums[max] | keys[max]].
static __device__ __align__(256) unsigned char g_select_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;

// Device address of g_select_scratch on the current device, looked up once
// per device (the symbol's host-side name is not a device address). The
// cached address belongs to the device's current context: after
// cudaDeviceReset it would be stale, so the library is not to be used across
// a device reset.
void* scratch_for_current_device(muon_status* err) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    *err = MUON_ERR_CUDA;
    return nullptr;
  }
  if (dev < 0 || dev >= kMaxDevices) {  // beyond the per-device address table
    *err = MUON_ERR_INVALID_ARG;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_select_scratch) != cudaSuccess || !p) {
      *err = MUON_ERR_CUDA;
      return nullptr;
    }
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace
}  // namespace muon

using namespace muon;

extern "C" muon_status select_rows_noalloc(const float* M, int64_t n, int64_t m, int64_t k, muon_norm norm,
                                           int32_t* idx_out, int32_t* dev_status, void* stream) {
  if (n < 0 || m < 0 || m > INT32_MAX) return MUON_ERR_SHAPE;
  if (n > kNoAllocMaxRows) return MUON_ERR_SHAPE;  // the fixed scratch holds kNoAllocMaxRows rows
  if (k < 1 || k > n) return MUON_ERR_SHAPE;
  if (norm != MUON_NORM_L1 && norm != MUON_NORM_L2) return MUON_ERR_INVALID_ARG;
  if (!M || !idx_out) return MUON_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(M) & 15u) != 0) return MUON_ERR_ALIGN;
  if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return MUON_ERR_ALIGN;
  muon_status err = MUON_OK;
  char* base = static_cast<char*>(scratch_for_current_device(&err));
  if (!base) return err;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Nothing here must start at zero: the row kernel writes every sum and key
  // of rows [0, n) before the selection kernel reads them, and the selection
  // kernel writes s and xscale. Stale contents of earlier calls are never read.
  float* s_out = reinterpret_cast<float*>(base);
  float* xscale_out = s_out + 1;
  double* sums = reinterpret_cast<double*>(base + kHeaderBytes);
  double* keys = sums + kNoAllocMaxRows;
  RowLaunch L{};
  L.count = 1;
  L.status = dev_status;
  L.key_l2 = norm == MUON_NORM_L2;
  RowMat& r = L.m[0];
  r.src = M;
  r.rows = n;
  r.cols = m;
  r.ntask = (int32_t)n;
  r.rsum = sums;
  r.rkey = keys;
  muon_status st = launch_row_stats(L, Op::F32, s);
  if (st != MUON_OK) return st;
  return launch_select(keys, sums, n, k, idx_out, s_out, xscale_out, 0.f, -1.f, dev_status, s);
}

// kcommon.cuh -- pieces shared by the SVDQuant kernels: bounded mbarrier
// waits, error bits, and the layout constants of the tensor-core scale tiles.
#pragma once

#include <cstdint>
#include <cstdlib>
#include <cuda_runtime.h>

#include <map>
#include <mutex>
#include <utility>

#include "ptx.cuh"

namespace svdq {

// Device error word bits (read back by svdq_device_status).
constexpr unsigned kErrQuantTimeout = 1u;
constexpr unsigned kErrGemmTimeout = 2u;

// A wait that has not completed after this long is treated as a fault: the
// kernel records it, skips its remaining work, releases its tensor memory and
// returns.  Legitimate waits in these kernels last microseconds.
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;

// Scale-factor tiles consumed by the block-scaled MMA: for every 128 rows and
// every 64 K elements (4 scale bytes per row), one 512-byte atom in which the
// scale of (row r, 16-element block j) sits at byte (r % 32) * 16 + (r / 32) * 4 + j.
// Lane l of a warp thus reads its 16 bytes with one vector load and holds
// exactly the four TMEM columns (rows l, l+32, l+64, l+96) the MMA expects in
// TMEM lane l of every 32-lane sub-partition.  Atoms are stored K-fastest:
// (row tile t, K atom a) at (t * ka_pad + a) * 512.
constexpr int kSfAtomBytes = 512;
__host__ __device__ __forceinline__ int sf_atom_offset(int r_in_tile, int j) {
  return (r_in_tile & 31) * 16 + (r_in_tile >> 5) * 4 + j;
}

// Slot of channel pair j in the smoothing-factor table: within each group of
// 64 pairs (one 128-channel quantizer chunk) pair pp sits at (pp % 8) * 8 +
// pp / 8, so the eight threads that read pairs 8t + i (t = 0..7) at once hit
// eight consecutive 16-byte slots (no shared-memory bank conflict).
__host__ __device__ __forceinline__ int lam_slot(int j) {
  return (j & ~63) | ((j & 7) << 3) | ((j & 63) >> 3);
}

// Spin on an mbarrier phase.  Returns false, after setting *abort and the
// error bit, when the wait exceeds kWaitTimeoutNs; returns false at once when
// another thread of the CTA has already set *abort.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort,
                                             unsigned* err, unsigned code) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
        *abort = 1;
        atomicOr(err, code);
        return false;
      }
    }
  }
}

// Bounded wait used during cleanup after an abort (ignores the abort flag).
__device__ __forceinline__ bool wait_for(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > timeout_ns) return false;
  }
  return true;
}

// Programmatic dependent launch of the hot-path kernels (on unless the
// environment sets SVDQ_PDL=0): a kernel's launch and prologue overlap the
// previous kernel's tail; each kernel waits (griddep_wait) before touching
// global memory.
inline bool pdl_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("SVDQ_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}

// Raise a kernel's dynamic shared-memory limit once per (kernel, device) and
// size: keeps the per-call path free of attribute calls (and graph-capture safe).
inline cudaError_t ensure_smem_limit_ptr(const void* kern, size_t bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, size_t> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  size_t& cur = done[std::make_pair(kern, dev)];
  if (bytes <= cur) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) cur = bytes;
  return e;
}
template <typename Kernel>
inline cudaError_t ensure_smem_limit(Kernel kern, size_t bytes) {
  return ensure_smem_limit_ptr(reinterpret_cast<const void*>(kern), bytes);
}

}  // namespace svdq

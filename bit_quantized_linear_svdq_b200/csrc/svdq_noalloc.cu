// svdq_noalloc.cu -- svdq_linear_forward_noalloc: the forward pass with its
// intermediates (FP4 codes, scale tiles, rank-R activations) kept in a fixed
// array that the library owns, for callers that cannot hand it a workspace.
//
// Who needs it: a host that gives a kernel its inputs and outputs but no
// scratch buffer (a C plugin interface, or a runtime that owns every byte of
// device memory and offers no workspace hook at call time), and a
// latency-bound loop that may not call cudaMalloc because that call can block
// on, and synchronize with, work already queued on the device.
//
// The array is a file-scope __device__ variable: one copy per device, placed
// by the driver when it loads this file's module on that device and kept until
// the process exits.  Host code never takes its address directly (on the host
// the symbol is only a stand-in); the device address comes from
// cudaGetSymbolAddress, looked up once per device by the first call made with
// that device current, and cached together with the identity of the device's
// context.  A cudaDeviceReset replaces that context (and reloads the module,
// so the array may move): the next call sees a new context id and looks the
// address up again instead of writing through a stale pointer.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "svdq.h"

namespace {

constexpr size_t kScratchBytes = SVDQ_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices];
unsigned long long g_scratch_ctx[kMaxDevices];   // context id the cached address belongs to

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Id of the context current on this thread (0 when none is, or the driver
// calls are unavailable).  Driver entry points come through the runtime.
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of this device's copy of the array; NULL (and the CUDA error
// cleared) if the lookup fails.  Looked up on the first call for the device
// and again whenever the device's current context is not the one the cached
// address came from.
void* scratch_on(int dev) {
  std::lock_guard<std::mutex> lock(g_mu);
  const unsigned long long ctx = current_ctx_id();
  if (!g_scratch_addr[dev] || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_scratch) != cudaSuccess || !ptr) {
      cudaGetLastError();
      g_scratch_addr[dev] = nullptr;
      return nullptr;
    }
    g_scratch_addr[dev] = ptr;
    g_scratch_ctx[dev] = current_ctx_id();   // the lookup made the primary context current
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" {

svdq_status svdq_linear_forward_noalloc(const svdq_linear* h, const void* x, int M, void* y, void* stream) {
  if (!h || M < 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  // Size check first: nothing is looked up or launched for an M that does not fit.
  if (svdq_workspace_bytes(h, M) > kScratchBytes) return SVDQ_ERR_WORKSPACE;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return SVDQ_ERR_UNSUPPORTED;
  void* scratch = scratch_on(dev);
  if (!scratch) return SVDQ_ERR_CUDA;
  return svdq_linear_forward(h, x, M, y, scratch, stream);
}

}  // extern "C"

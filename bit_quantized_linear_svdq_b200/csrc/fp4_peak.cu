// fp4_peak.cu -- the dense block-scaled FP4 tensor-core rate of this device,
// measured: the denominator of the GEMM's roofline fraction.  One CTA per SM
// keeps its tensor core busy with back-to-back tcgen05.mma
// kind::mxf4nvf4.block_scale.block16 (M = 128, N = 256, K = 64, fp32
// accumulate in TMEM) from operands resident in shared memory, the shape and
// operand path of the GEMM kernels, with no loads in the loop.  The caller
// times the launch (CUDA events) and counts 2 * 128 * 256 * 64 flops per MMA.
//
// Operand values do not affect the rate; the tiles hold a fixed byte pattern
// and every scale factor is e4m3 1.0.  The only wait (for the MMAs to finish
// before the tensor memory is released) is bounded.
#include <cuda_runtime.h>

#include "kcommon.cuh"
#include "svdq.h"

namespace svdq {
namespace {

constexpr int kPeakThreads = 128;
constexpr int kARows = 128, kBRows = 256, kRowBytes = 128;      // one 256-element K tile, 128B swizzle
constexpr int kABytes = kARows * kRowBytes, kBBytes = kBRows * kRowBytes;
constexpr uint32_t kTmemCols = 512, kColSf = 256;

__device__ __forceinline__ uint64_t sdesc_sw128_rows(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(16u >> 4) << 16) | ((uint64_t)((8u * kRowBytes) >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}

__global__ void __launch_bounds__(kPeakThreads, 1) fp4_mma_loop_kernel(int iters, unsigned* err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_slot;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Fixed operand bytes: a mix of all E2M1 codes.
  for (int i = tid; i < (kABytes + kBBytes) / 4; i += kPeakThreads)
    reinterpret_cast<uint32_t*>(base)[i] = 0x9E2B7C41u * (uint32_t)(i + 1);
  if (tid == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = tmem_slot;
  // Scale factors e4m3 1.0 (0x38) in columns kColSf .. +47 of every lane (the
  // layout of the 128 x 256 GEMM: A atom a -> 4a..4a+3, B -> 16 + 8a ..).
  {
    uint32_t v[32], w[16];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = 0x38383838u;
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = 0x38383838u;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16) + kColSf;
    tmem_st32(lane_base, v);
    tmem_st16(lane_base + 32, w);
    tmem_st_wait();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (tid == 0) {
    const uint32_t idesc = idesc_nvfp4(kARows, kBRows);
    const uint32_t a = smem_u32(base), b = a + kABytes;
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int kb = 0; kb < 4; ++kb)
        mma_nvfp4(tmem, sdesc_sw128_rows(a + kb * 32), sdesc_sw128_rows(b + kb * 32), idesc, tmem + kColSf + 4 * kb,
                  tmem + kColSf + 16 + 8 * kb, (it | kb) != 0);
    }
    tc_commit(smem_u32(&bar));
    if (!wait_for(smem_u32(&bar), 0, kWaitTimeoutNs)) atomicOr(err, kErrGemmTimeout);
  }
  __syncwarp();
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
  (void)lane;
}

}  // namespace

cudaError_t launch_fp4_mma_loop(int iters, int ctas, unsigned* err, cudaStream_t stream) {
  // More than half of an SM's shared memory, so no two CTAs share an SM (and
  // its tensor core); the tiles use the first 49 KB.
  const size_t smem = 120 * 1024;
  cudaError_t e = ensure_smem_limit(fp4_mma_loop_kernel, smem);
  if (e != cudaSuccess) return e;
  fp4_mma_loop_kernel<<<ctas, kPeakThreads, smem, stream>>>(iters, err);
  return cudaGetLastError();
}

}  // namespace svdq

namespace svdq {
namespace {
__device__ unsigned g_fp4_loop_err;
}  // namespace
}  // namespace svdq

extern "C" {

svdq_status svdq_fp4_mma_loop(int iters, int* ctas, void* stream) {
  // At most about a quarter of a second of MMAs, well inside the bounded wait.
  if (iters < 1 || iters > (1 << 20)) return SVDQ_ERR_INVALID_ARG;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  unsigned* err = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&err), svdq::g_fp4_loop_err) != cudaSuccess) {
    cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  if (svdq::launch_fp4_mma_loop(iters, sms, err, static_cast<cudaStream_t>(stream)) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (ctas) *ctas = sms;
  return SVDQ_OK;
}

svdq_status svdq_fp4_mma_loop_status(int* flags) {
  unsigned v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess || cudaMemcpyFromSymbol(&v, svdq::g_fp4_loop_err, sizeof(v)) != cudaSuccess) {
    cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  if (v) {
    const unsigned z = 0;
    cudaMemcpyToSymbol(svdq::g_fp4_loop_err, &z, sizeof(z));
  }
  if (flags) *flags = (int)v;
  return v ? SVDQ_ERR_DEVICE : SVDQ_OK;
}

}  // extern "C"

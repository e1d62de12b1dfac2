// quantize_weight.cu -- offline NVFP4 quantization of a dense bf16 weight on
// the GPU: W (N, K) -> qweight (N, K/2) packed E2M1 + wscales (K/16, N) e4m3,
// with the optional 128-block rotation of every row.
//
// The checkpoint of "SVDQuant W4A4" (vLLM-Omni svdquant.md, "Checkpoint
// contract") stores W as (N, K) rows of packed FP4 codes and one e4m3 scale per
// 16 K elements in a (K/16, N) tensor.  Rotating the weight offline ("Rotate in
// quantization and its vLLM implementation", section 2.1: W' = R W in the
// page's (K, N) orientation) rotates each (N, K) row exactly like an
// activation row.  Quantization follows the activation rules:
//   w_hat = fp32(w)                    (exact from bf16), optionally
//   w_hat = fp32(butterfly_128(w_hat) * fp32(1/sqrt(128)))
//   scale = e4m3_rne_satfinite(fp32(amax16 / 6)),  code = e2m1_rne_satfinite(fp32(w_hat / scale))
// with correctly rounded fp32 divisions (nvfp4_block.cuh: a block whose scale
// rounds to zero gets codes 0; a block holding a NaN or an infinity takes the
// IEEE-division path).
//
// One CTA of 128 threads covers 32 rows x 128 K elements: four threads per
// row, 32 consecutive elements (two scale blocks) each, so a warp reads and
// writes 8 contiguous row segments.  The CTA's 8 x 32 scale bytes go through
// shared memory so that the (K/16, N) stores are 32-byte row segments.
#include <cuda_runtime.h>

#include "hadamard.cuh"
#include "kcommon.cuh"
#include "nvfp4_block.cuh"
#include "svdq_kernels.h"

namespace svdq {
namespace {

constexpr int kRowsW = 32, kChunkW = 128, kThreadsW = 128;

template <bool ROT>
__global__ void __launch_bounds__(kThreadsW)
    quantize_weight_kernel(const __nv_bfloat16* __restrict__ w, int N, int K, uint8_t* __restrict__ qweight,
                           uint8_t* __restrict__ wscales) {
  __shared__ uint8_t sc[kChunkW / 16][kRowsW];      // [block in chunk][row]
  __shared__ float2 srec[128];                       // e4m3 code -> {-s, RN(1/s)}
  const int tid = threadIdx.x, rl = tid >> 2, qq = tid & 3;
  {
    const float s = e4m3_to_f32((uint32_t)tid);
    srec[tid] = make_float2(-s, tid ? __frcp_rn(s) : 0.0f);
  }
  const float y6 = __frcp_rn(6.0f);
  __syncthreads();
  const int n0 = blockIdx.y * kRowsW, n = n0 + rl;
  const int k0 = blockIdx.x * kChunkW + 32 * qq;     // first element of this thread's quarter
  uint64_t v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = 0ull;
  if (n < N) {
    const uint4* src = reinterpret_cast<const uint4*>(w + (size_t)n * K + k0);   // rows 16-byte aligned (K % 8 == 0)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (k0 + 8 * c < K) {                            // K % 16 == 0: 8-element groups are whole
        const uint4 pw = src[c];
        const uint32_t x4[4] = {pw.x, pw.y, pw.z, pw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) v[4 * c + i] = pk2(__uint_as_float(x4[i] << 16), __uint_as_float(x4[i] & 0xFFFF0000u));
      }
    }
  }
  if (ROT) hadamard128_quarter(v, qq);               // every lane: full-warp shuffles (K % 128 == 0)
  uint32_t cw[4], sbytes = 0;
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    uint64_t blk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) blk[i] = v[8 * b + i];
    sbytes |= quantize_any(blk, srec, y6, cw[2 * b], cw[2 * b + 1]) << (8 * b);
  }
  if (n < N) {
    uint2* dst = reinterpret_cast<uint2*>(qweight + (size_t)n * (K / 2) + k0 / 2);   // 8-byte aligned
#pragma unroll
    for (int b = 0; b < 2; ++b)
      if (k0 + 16 * b < K) dst[b] = make_uint2(cw[2 * b], cw[2 * b + 1]);
  }
  sc[2 * qq][rl] = (uint8_t)sbytes;
  sc[2 * qq + 1][rl] = (uint8_t)(sbytes >> 8);
  __syncthreads();
  // Scale bytes: block kb of the chunk for rows n0 .. n0+31 -> wscales[kb, n0 ..].
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int kbl = (tid >> 5) + 4 * i, r = tid & 31;
    const int kb = blockIdx.x * (kChunkW / 16) + kbl;
    if (n0 + r < N && kb < K / 16) wscales[(size_t)kb * N + n0 + r] = sc[kbl][r];
  }
}

}  // namespace

cudaError_t launch_quantize_weight(const void* w, int N, int K, int rotate_block, void* qweight, void* wscales,
                                   cudaStream_t stream) {
  const dim3 grid((unsigned)((K + kChunkW - 1) / kChunkW), (unsigned)((N + kRowsW - 1) / kRowsW));
  if (rotate_block == 128)
    quantize_weight_kernel<true><<<grid, kThreadsW, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(w), N, K, static_cast<uint8_t*>(qweight), static_cast<uint8_t*>(wscales));
  else
    quantize_weight_kernel<false><<<grid, kThreadsW, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(w), N, K, static_cast<uint8_t*>(qweight), static_cast<uint8_t*>(wscales));
  return cudaGetLastError();
}

}  // namespace svdq

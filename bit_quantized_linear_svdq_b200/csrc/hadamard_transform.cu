// hadamard_transform.cu -- the standalone in-place Walsh-Hadamard transform
// x <- x H_n / sqrt(n) of every length-n row (n = 2^k <= 32768), bf16 or fp16.
//
// "Rotate in quantization and its vLLM implementation", section 3.1 (the
// Hadacore kernel): the Sylvester recursion gives an O(n log n) transform with
// no stored matrix, and since H is symmetric the same operation is its own
// inverse.  Arithmetic, in fp32 as the quantizers' online rotation: butterfly
// stages h = 1, 2, ..., n/2 in that order, each replacing (x[i], x[i+h]) with
// i & h == 0 by (x[i] + x[i+h], x[i] - x[i+h]); then one multiply by
// fp32(1/sqrt(n)); then round to the storage type (to nearest, ties to even).
//
// A CTA holds whole rows; the stages run in passes of up to five: in pass p
// every thread takes groups of 2^b elements 32^p apart and does their b stages
// in registers (the stages of the row in increasing h), with a CTA barrier
// between passes.  The first pass reads its 32-element runs straight from
// global memory and the last pass writes straight back; the passes between
// them keep the rows in shared memory as fp32 (element i at word i + i/32, so
// both the contiguous runs and the strided groups hit 32 different banks).
// The row is read once and written once.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "kcommon.cuh"
#include "svdq_kernels.h"

namespace svdq {
namespace {

constexpr int kThreadsH = 256;

__device__ __forceinline__ int padw(int i) { return i + (i >> 5); }

template <typename T>
__device__ __forceinline__ float load_f32(const T* p);
template <>
__device__ __forceinline__ float load_f32<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }
template <>
__device__ __forceinline__ float load_f32<__half>(const __half* p) { return __half2float(*p); }

template <typename T>
__device__ __forceinline__ float to_f32(uint32_t bits);
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(uint32_t bits) { return __uint_as_float(bits << 16); }
template <>
__device__ __forceinline__ float to_f32<__half>(uint32_t bits) {
  return __half2float(__ushort_as_half((unsigned short)bits));
}
__device__ __forceinline__ uint32_t bits16(__nv_bfloat16 v) { return __bfloat16_as_ushort(v); }
__device__ __forceinline__ uint32_t bits16(__half v) { return __half_as_ushort(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }
template <>
__device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }

// One pass: groups of 2^B elements `stride` apart; their B butterfly stages;
// the final multiply when this is the last pass.  With `out` set (the last
// pass of the register path) the results go straight to the rows in global
// memory: for each t the lanes of a warp hold consecutive columns.
template <int B, typename T>
__device__ __forceinline__ void pass(float* buf, int pad_n, int nrows, int log2n, int shift, bool last, float c,
                                     T* out = nullptr) {
  constexpr int kR = 1 << B;
  const int stride = 1 << shift;
  const int per_row = 1 << (log2n - B);
  for (int g = threadIdx.x; g < nrows * per_row; g += blockDim.x) {
    const int row = g >> (log2n - B), gi = g & (per_row - 1);
    const int lo = gi & (stride - 1), hi = gi >> shift;
    float* rb = buf + row * pad_n;
    const int base = hi * (stride << B) + lo;
    float v[kR];
#pragma unroll
    for (int t = 0; t < kR; ++t) v[t] = rb[padw(base + t * stride)];
#pragma unroll
    for (int h = 1; h < kR; h <<= 1) {
#pragma unroll
      for (int t = 0; t < kR; ++t) {
        if ((t & h) == 0) {
          const float a = v[t], b = v[t + h];
          v[t] = __fadd_rn(a, b);
          v[t + h] = __fsub_rn(a, b);
        }
      }
    }
    if (last) {
#pragma unroll
      for (int t = 0; t < kR; ++t) v[t] = __fmul_rn(v[t], c);
    }
    if (out) {
      T* orow = out + ((size_t)row << log2n);
#pragma unroll
      for (int t = 0; t < kR; ++t) orow[base + t * stride] = from_f32<T>(v[t]);
    } else {
#pragma unroll
      for (int t = 0; t < kR; ++t) rb[padw(base + t * stride)] = v[t];
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreadsH) hadamard_transform_kernel(T* __restrict__ x, int rows, int log2n,
                                                                       int rows_per_cta, float c) {
  extern __shared__ float buf[];
  const int n = 1 << log2n, pad_n = n + (n >> 5);
  const int row0 = blockIdx.x * rows_per_cta;
  const int nrows = min(rows_per_cta, rows - row0);
  T* xr = x + (size_t)row0 * n;
  const int passes = (log2n + 4) / 5;          // n = 1: none (the multiply by 1 changes nothing)
  if (log2n >= 5 && (reinterpret_cast<uintptr_t>(x) & 15u) == 0) {
    // Register path: the first pass takes each 32-element run straight from
    // global memory (four 16-byte loads per thread; consecutive threads,
    // consecutive runs), the last pass writes straight back, and only the
    // passes between them go through shared memory (lane L's 32 words at
    // 33L .. 33L+31: 32 different banks for each t).
    for (int g = threadIdx.x; g < nrows << (log2n - 5); g += blockDim.x) {
      const uint4* src = reinterpret_cast<const uint4*>(xr + ((size_t)g << 5));
      uint4 w[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) w[q] = src[q];
      float v[32];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t u[4] = {w[q].x, w[q].y, w[q].z, w[q].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          v[8 * q + 2 * j] = to_f32<T>(u[j] & 0xFFFFu);
          v[8 * q + 2 * j + 1] = to_f32<T>(u[j] >> 16);
        }
      }
#pragma unroll
      for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          if ((t & h) == 0) {
            const float a = v[t], b = v[t + h];
            v[t] = __fadd_rn(a, b);
            v[t + h] = __fsub_rn(a, b);
          }
        }
      }
      if (passes == 1) {
        uint4* dst = reinterpret_cast<uint4*>(xr + ((size_t)g << 5));
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t o[4];
#pragma unroll
          for (int j = 0; j < 4; ++j)
            o[j] = bits16(from_f32<T>(__fmul_rn(v[8 * q + 2 * j], c))) |
                   (bits16(from_f32<T>(__fmul_rn(v[8 * q + 2 * j + 1], c))) << 16);
          dst[q] = make_uint4(o[0], o[1], o[2], o[3]);
        }
      } else {
        float* d = buf + (g >> (log2n - 5)) * pad_n + padw((g << 5) & (n - 1));
#pragma unroll
        for (int t = 0; t < 32; ++t) d[t] = v[t];
      }
    }
    for (int p = 1; p < passes; ++p) {
      __syncthreads();
      const int b = min(5, log2n - 5 * p);
      const bool last = p == passes - 1;
      T* out = last ? xr : nullptr;
      switch (b) {
        case 1: pass<1>(buf, pad_n, nrows, log2n, 5 * p, last, c, out); break;
        case 2: pass<2>(buf, pad_n, nrows, log2n, 5 * p, last, c, out); break;
        case 3: pass<3>(buf, pad_n, nrows, log2n, 5 * p, last, c, out); break;
        case 4: pass<4>(buf, pad_n, nrows, log2n, 5 * p, last, c, out); break;
        default: pass<5>(buf, pad_n, nrows, log2n, 5 * p, last, c, out); break;
      }
    }
    return;
  }
  // Shared-memory path (n < 32 or a base address without 16-byte alignment).
  // 16-byte accesses (8 elements, inside one row since 8 | n) when the rows
  // allow it; lane L's eight words then sit in banks distinct from the other
  // lanes' (8L + L/4 covers 0..31 once).
  const bool vec = log2n >= 3 && (reinterpret_cast<uintptr_t>(x) & 15u) == 0;
  if (vec) {
    const uint4* src = reinterpret_cast<const uint4*>(xr);
#pragma unroll 4
    for (int v = threadIdx.x; v < (nrows << log2n) >> 3; v += blockDim.x) {
      const uint4 w = src[v];
      const uint32_t u[4] = {w.x, w.y, w.z, w.w};
      const int e0 = v << 3;
      float* d = buf + (e0 >> log2n) * pad_n + padw(e0 & (n - 1));   // 8 consecutive words
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        d[2 * j] = to_f32<T>(u[j] & 0xFFFFu);
        d[2 * j + 1] = to_f32<T>(u[j] >> 16);
      }
    }
  } else {
    for (int e = threadIdx.x; e < nrows * n; e += blockDim.x)
      buf[(e >> log2n) * pad_n + padw(e & (n - 1))] = load_f32(xr + e);
  }
  __syncthreads();
  for (int p = 0; p < passes; ++p) {
    const int b = min(5, log2n - 5 * p);
    const bool last = p == passes - 1;
    switch (b) {
      case 1: pass<1, T>(buf, pad_n, nrows, log2n, 5 * p, last, c); break;
      case 2: pass<2, T>(buf, pad_n, nrows, log2n, 5 * p, last, c); break;
      case 3: pass<3, T>(buf, pad_n, nrows, log2n, 5 * p, last, c); break;
      case 4: pass<4, T>(buf, pad_n, nrows, log2n, 5 * p, last, c); break;
      default: pass<5, T>(buf, pad_n, nrows, log2n, 5 * p, last, c); break;
    }
    __syncthreads();
  }
  if (vec) {
    uint4* dst = reinterpret_cast<uint4*>(xr);
#pragma unroll 4
    for (int v = threadIdx.x; v < (nrows << log2n) >> 3; v += blockDim.x) {
      const int e0 = v << 3;
      const float* sv = buf + (e0 >> log2n) * pad_n + padw(e0 & (n - 1));
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) o[j] = bits16(from_f32<T>(sv[2 * j])) | (bits16(from_f32<T>(sv[2 * j + 1])) << 16);
      dst[v] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  } else {
    for (int e = threadIdx.x; e < nrows * n; e += blockDim.x)
      xr[e] = from_f32<T>(buf[(e >> log2n) * pad_n + padw(e & (n - 1))]);
  }
}

template <typename T>
cudaError_t launch_t(void* x, int rows, int log2n, cudaStream_t stream) {
  const int n = 1 << log2n;
  const int rows_per_cta = n >= 8192 ? 1 : 8192 / n;
  const size_t smem = (size_t)rows_per_cta * (n + (n >> 5)) * sizeof(float);
  cudaError_t e = ensure_smem_limit(hadamard_transform_kernel<T>, smem);
  if (e != cudaSuccess) return e;
  // fp32(1/sqrt(n)), rounded from the double-precision quotient (exact for
  // even log2n; 0x3DB504F3 for n = 128, the quantizers' constant).
  const float c = (float)(1.0 / sqrt((double)n));
  const int grid = (rows + rows_per_cta - 1) / rows_per_cta;
  hadamard_transform_kernel<T><<<grid, kThreadsH, smem, stream>>>(static_cast<T*>(x), rows, log2n, rows_per_cta, c);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_hadamard_transform(void* x, int rows, int log2n, int dtype, cudaStream_t stream) {
  return dtype == 0 ? launch_t<__nv_bfloat16>(x, rows, log2n, stream) : launch_t<__half>(x, rows, log2n, stream);
}

}  // namespace svdq

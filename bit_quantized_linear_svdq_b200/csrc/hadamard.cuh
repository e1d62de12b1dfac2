// hadamard.cuh -- two-lane packed fp32 helpers and the in-register 128-point
// Walsh-Hadamard rotation shared by the activation and weight quantizers.
//
// The rotation of "Rotate in quantization and its vLLM implementation"
// (sections 2.1-2.2, 3.3): x <- fp32(butterfly_128(x) * fp32(1/sqrt(128))),
// stages h = 1, 2, 4, ..., 64 in that order, each replacing the pair
// (x[i], x[i+h]) with i & h == 0 by (x[i] + x[i+h], x[i] - x[i+h]), every
// operation rounded to fp32 -- the order the quantized codes depend on.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace svdq {

__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float lo2(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float hi2(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}


// Four lanes 4r .. 4r+3 (lane & 3 = qq) hold the quarters of one 128-element
// rotation block, 32 consecutive elements each: element e of the quarter is
// lane (e & 1) of v[e >> 1].  Stages h = 1 .. 16 stay in registers; h = 32 and
// 64 pair the quarter with the one in lane ^ 1 and lane ^ 2, the lower of the
// two taking a + b and the upper a - b, each as one fused op (+-mine + other)
// with a single rounding.  Then the multiply by fp32(1/sqrt(128)).  Every lane
// of the warp must call it (full-warp shuffles).
__device__ __forceinline__ void hadamard128_quarter(uint64_t (&v)[16], int qq) {
  // h = 1: the pair (2i, 2i+1) is the two lanes of v[i]; regroup two words so
  // each packed op yields two results.
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint64_t a = pk2(lo2(v[2 * j]), lo2(v[2 * j + 1]));
    const uint64_t b = pk2(hi2(v[2 * j]), hi2(v[2 * j + 1]));
    const uint64_t sm = add2(a, b), df = sub2(a, b);
    v[2 * j] = pk2(lo2(sm), lo2(df));
    v[2 * j + 1] = pk2(hi2(sm), hi2(df));
  }
  // h = 2, 4, 8, 16: words (i, i + h/2).
#pragma unroll
  for (int st = 0; st < 4; ++st) {
    const int hp = 1 << st;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if ((i & hp) == 0) {
        const uint64_t a = v[i], b = v[i + hp];
        v[i] = add2(a, b);
        v[i + hp] = sub2(a, b);
      }
    }
  }
  // h = 32 (lane ^ 1) and h = 64 (lane ^ 2).
#pragma unroll
  for (int st = 0; st < 2; ++st) {
    const float sg = (qq >> st) & 1 ? -1.0f : 1.0f;
    const uint64_t sg2 = pk2(sg, sg);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float olo = __shfl_xor_sync(0xFFFFFFFFu, lo2(v[i]), 1 << st);
      const float ohi = __shfl_xor_sync(0xFFFFFFFFu, hi2(v[i]), 1 << st);
      v[i] = fma2(sg2, v[i], pk2(olo, ohi));
    }
  }
  const float cn = 0.0883883461356163f;        // fp32(1/sqrt(128)) = 0x3DB504F3
  const uint64_t cn2 = pk2(cn, cn);
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = mul2(v[i], cn2);
}

}  // namespace svdq

// nvfp4_block.cuh -- quantization of one 16-element block to NVFP4 (one
// e4m3 scale, sixteen E2M1 codes), shared by the activation and weight
// quantizers.
//
//   scale = e4m3_rne_satfinite(fp32(amax / 6)),  code = e2m1_rne_satfinite(fp32(v / scale))
//
// Exact fp32 division without the divide unit: with y = RN(1/b),
//   q0 = RN(a*y), r = RN(a - b*q0) (fused), q1 = RN(q0 + r*y) (fused)
// is the correctly rounded a/b (Markstein's iteration; checked exhaustively
// for every significand pair that occurs here: fp32/e4m3 and fp32/6 for the
// scale and codes, bf16/bf16 for the activation smoothing).  Two lanes run per
// instruction (fma.rn.f32x2).  Blocks whose values overflow or hold NaN take
// an IEEE-division path, so results equal the divide unit's in every case.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "hadamard.cuh"
#include "ptx.cuh"

namespace svdq {

// Correctly rounded a / B for two lanes, given nb = -B and y = RN(1 / B).
// Zero results may carry the wrong sign (q0 + r*y with r = +0).
__device__ __forceinline__ uint64_t div_mk2(uint64_t a, uint64_t nb, uint64_t y) {
  const uint64_t q0 = mul2(a, y);
  const uint64_t r = fma2(q0, nb, a);
  return fma2(r, y, q0);
}

// As div_mk2, but the result keeps the sign of a*y, so a signed zero divides
// to a correctly signed zero for any divisor.
__device__ __forceinline__ uint64_t div_rn2(uint64_t a, uint64_t nb, uint64_t y) {
  const uint64_t q0 = mul2(a, y);
  const uint64_t r = fma2(q0, nb, a);
  const uint64_t q1 = fma2(r, y, q0);
  return (q1 & 0x7FFFFFFF7FFFFFFFull) | (q0 & 0x8000000080000000ull);
}

// With a negative divisor B = -b (b > 0), div_mk2 returns correctly signed
// zeros as well: a = +-0 gives q0 = -+0, r = +0 and q1 = -+0 = a / B.  The
// "negated" layout divides x by -smooth (giving -x_hat exactly) and -x_hat by
// -scale (giving x_hat / scale), so no sign fix-up is needed when every smooth
// factor is positive.

// max(acc, |v|) that propagates NaN (the scale of a block holding a NaN is NaN).
__device__ __forceinline__ float amax_nan(float acc, float v) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(acc), "f"(fabsf(v)));
  return r;
}

// NaN-propagating max of three magnitudes (sm_100 three-input form).
__device__ __forceinline__ float amax3_nan(float a, float b, float c) {
  float r;
  asm("max.NaN.abs.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// max |v| over a 16-element block (NaN if any element is NaN): eight
// three-input maxes in a tree of depth three.
__device__ __forceinline__ float amax8(const uint64_t (&v)[8]) {
  const float m0 = amax3_nan(lo2(v[0]), hi2(v[0]), lo2(v[1]));
  const float m1 = amax3_nan(hi2(v[1]), lo2(v[2]), hi2(v[2]));
  const float m2 = amax3_nan(lo2(v[3]), hi2(v[3]), lo2(v[4]));
  const float m3 = amax3_nan(hi2(v[4]), lo2(v[5]), hi2(v[5]));
  const float m4 = amax3_nan(lo2(v[6]), hi2(v[6]), lo2(v[7]));
  return amax3_nan(amax3_nan(m0, m1, m2), amax3_nan(m3, m4, hi2(v[7])), 0.0f);
}

// bf16 word (two channels) -> packed fp32 pair
__device__ __forceinline__ uint64_t bf16x2_to_f2(uint32_t w) {
  return pk2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

struct Tables {
  // e4m3 code -> {-B, RN(1/B)} for the scale division: B = s (sign-fixed
  // layout) or B = -s (negated layout).  Entry 0 is unused.
  float2 srec[128];
};

// Quantize one 16-element block held as 8 packed pairs of finite values:
// returns the scale byte and the 16 codes (w0: elements 0-7, w1: 8-15).
template <bool NEG>
__device__ __forceinline__ uint32_t quant_block(const uint64_t (&v)[8], float amax, const float2* srec, float y6,
                                                uint32_t& w0, uint32_t& w1) {
  // amax / 6, correctly rounded (Markstein with y6 = RN(1/6)).
  const float q0 = amax * y6;
  const float q1 = fmaf(fmaf(q0, -6.0f, amax), y6, q0);
  const uint32_t sb = cvt_e4m3(q1);
  // Branch-free: a zero scale (table entry {+-0, 0}) divides every value to a
  // finite +-0, and the mask then clears those codes to 0.
  const float2 sr = srec[sb];
  const uint64_t ns = pk2(sr.x, sr.x), ys = pk2(sr.y, sr.y);
  uint64_t q[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) q[i] = NEG ? div_mk2(v[i], ns, ys) : div_rn2(v[i], ns, ys);
  const uint32_t keep = sb != 0u ? 0xFFFFFFFFu : 0u;
  w0 = keep & cvt_e2m1x8(lo2(q[0]), hi2(q[0]), lo2(q[1]), hi2(q[1]), lo2(q[2]), hi2(q[2]), lo2(q[3]), hi2(q[3]));
  w1 = keep & cvt_e2m1x8(lo2(q[4]), hi2(q[4]), lo2(q[5]), hi2(q[5]), lo2(q[6]), hi2(q[6]), lo2(q[7]), hi2(q[7]));
  return sb;
}

// IEEE-division path for blocks holding +-inf or NaN.
__device__ __forceinline__ uint32_t quant_block_slow(const uint64_t (&v)[8], uint32_t& w0, uint32_t& w1) {
  float f[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    f[2 * i] = lo2(v[i]);
    f[2 * i + 1] = hi2(v[i]);
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = amax_nan(amax, f[i]);
  const uint32_t sb = cvt_e4m3(__fdiv_rn(amax, 6.0f));
  const float s = e4m3_to_f32(sb);
  w0 = w1 = 0u;
  if (s > 0.0f) {
#pragma unroll
    for (int i = 0; i < 16; ++i) f[i] = __fdiv_rn(f[i], s);
    w0 = cvt_e2m1x8(f[0], f[1], f[2], f[3], f[4], f[5], f[6], f[7]);
    w1 = cvt_e2m1x8(f[8], f[9], f[10], f[11], f[12], f[13], f[14], f[15]);
  }
  return sb;
}

// Two-op division for activations: a / b for two lanes from b's reciprocal
// pair (yh, yl) = (RZ(1/b), RN(1/b - RZ(1/b)) carrying the sign of yh):
// RN(a*yh + RN(a*yl)), the correctly rounded quotient for every operand pair
// the activation quantizers meet (bf16 / bf16 smoothing, fp32 / e4m3 codes,
// fp32 / 6 scales; exhaustive checks in the tests), with zeros carrying the
// sign of a/b.
__device__ __forceinline__ uint64_t div_rr2(uint64_t a, uint64_t yh, uint64_t yl) {
  return fma2(a, yh, mul2(a, yl));
}

// {RZ(1/b), RN(1/b - RZ(1/b)) with the sign of RZ(1/b)} for a finite nonzero b.
__device__ __forceinline__ float2 recip_pair(float b) {
  const double inv = 1.0 / static_cast<double>(b);
  const float yh = __double2float_rz(inv);
  const float yl = __double2float_rn(inv - static_cast<double>(yh));
  return make_float2(yh, copysignf(fabsf(yl), yh));
}

// One 16-element block of finite values with two-op divisions, the scale's
// reciprocal pair formed per block (the few-row quantizers): returns the
// scale byte and the codes (w0: elements 0-7, w1: 8-15).  (yh6, yl6) is
// recip_pair(6).
__device__ __forceinline__ uint32_t quant_block_rp(const uint64_t (&v)[8], float amax, float yh6, float yl6,
                                                   uint32_t& w0, uint32_t& w1) {
  const float q6 = fmaf(amax, yh6, amax * yl6);       // amax / 6, correctly rounded
  const uint32_t sb = cvt_e4m3(q6);
  const float2 sr = sb ? recip_pair(e4m3_to_f32(sb)) : make_float2(0.0f, 0.0f);
  const uint64_t yh = pk2(sr.x, sr.x), yl = pk2(sr.y, sr.y);
  uint64_t q[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) q[i] = div_rr2(v[i], yh, yl);
  const uint32_t keep = sb != 0u ? 0xFFFFFFFFu : 0u;
  w0 = keep & cvt_e2m1x8(lo2(q[0]), hi2(q[0]), lo2(q[1]), hi2(q[1]), lo2(q[2]), hi2(q[2]), lo2(q[3]), hi2(q[3]));
  w1 = keep & cvt_e2m1x8(lo2(q[4]), hi2(q[4]), lo2(q[5]), hi2(q[5]), lo2(q[6]), hi2(q[6]), lo2(q[7]), hi2(q[7]));
  return sb;
}

// x / smooth for 2N channels (bf16 words xin) with the IEEE divide: the path
// for blocks whose fast quotients overflowed or hold NaN.
template <int N>
__device__ __forceinline__ void smooth_ieee(const uint32_t (&xin)[N], const float* lamf, int k, uint64_t (&v)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i)
    v[i] = pk2(__fdiv_rn(__uint_as_float(xin[i] << 16), lamf[k + 2 * i]),
               __fdiv_rn(__uint_as_float(xin[i] & 0xFFFF0000u), lamf[k + 2 * i + 1]));
}

__device__ __forceinline__ uint32_t quantize_any(const uint64_t (&v)[8], const float2* srec, float y6, uint32_t& w0,
                                                 uint32_t& w1) {
  const float amax = amax8(v);
  return (amax < 3.0e38f) ? quant_block<false>(v, amax, srec, y6, w0, w1) : quant_block_slow(v, w0, w1);
}

}  // namespace svdq

// quantize_few.cu -- the activation quantizer for 1..4 token rows, on CUDA
// cores, for the few-row forward (the CUDA-core matrix-vector product that
// follows reads its outputs).  Same arithmetic as quantize_act.cu, per block:
//
//   x_hat = fp32(x / smooth_factor)       two-op division, y = RZ(1/s), y' = RN(1/s - y)
//   x_hat = fp32(butterfly_128(x_hat) * fp32(1/sqrt(128)))   (optional rotation)
//   scale = e4m3_rne_satfinite(fp32(amax16 / 6)),  code = e2m1_rne_satfinite(fp32(x_hat / scale))
//
// ("SVDQuant W4A4", "Checkpoint contract"; the rotation of "Rotate in
// quantization and its vLLM implementation", sections 2.1-2.2, 3.3), with the
// blocks whose quotients overflow or hold NaN on the divide unit, so codes
// and scales are bit-identical to the tiled quantizer's.
//
// The 128-row machinery of the tiled quantizer (clusters, TMA tiles, tensor
// memory) is all fixed cost for a handful of rows.  Here one CTA of 128
// threads takes one 128-channel slice of K for every row: warp 0 quantizes
// (lane = (row, 16-channel block), or with rotation four lanes per row and
// quarter), and every thread takes ranks of the rank-R down-projection,
// L_slice[m, r] = sum over the slice of x[m, k] P[k, r] (P = diag(1/smooth)
// R^T proj_down, formed at create; products exact in fp32, summed in channel
// order).  The slices' fp32 partial sums go to the workspace; the
// matrix-vector kernel adds them in slice order (deterministic) as it stages
// the token rows.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "hadamard.cuh"
#include "kcommon.cuh"
#include "nvfp4_block.cuh"
#include "svdq_kernels.h"

namespace svdq {
namespace {

constexpr int kFewThreads = 128;
constexpr int kSlice = 128;                       // channels per CTA

struct FewParams {
  const uint32_t* x;        // bf16 pairs, (M, K) row-major
  const float4* lamq;       // smoothing reciprocal pairs, lam_slot order
  const float* lamf;        // smoothing factors (IEEE path)
  const __nv_bfloat16* pdT; // P^T (R, Kp)
  uint8_t* codes;           // (M, Kp/2)
  uint8_t* sfa;             // scale atoms of row tile 0 (ka_pad atoms)
  float* part;              // [slices][M][R] fp32 partial L
  int M, K, Kp, R, ka_pad;
};

template <bool ROT>
__global__ void __launch_bounds__(kFewThreads) quantize_few_kernel(const FewParams p) {
  __shared__ float xs[kGemvMaxRows][kSlice];          // x of the slice, every row
  __shared__ float lsum[kFewThreads / 32][kGemvMaxRows][32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int k0 = blockIdx.x * kSlice;
  // The smoothing operands of warp 0's blocks and this thread's first rank
  // row of P^T are library-owned weights, written at create: requested
  // before the dependency wait, so only x is read after it.
  constexpr int kLamPre = ROT ? 16 : 8;
  float4 lam_pre[kLamPre];
  if (warp == 0) {
    const int kl = ROT ? (k0 + 32 * (lane & 3)) / 2 : (k0 + 16 * (lane & 7)) / 2;
#pragma unroll
    for (int i = 0; i < kLamPre; ++i) lam_pre[i] = __ldg(p.lamq + lam_slot(kl + i));
  }
  uint4 pd_pre[4];
  if (lane < p.R) {
    const uint4* prow = reinterpret_cast<const uint4*>(p.pdT + (size_t)lane * p.Kp + k0 + 32 * warp);
#pragma unroll
    for (int c = 0; c < 4; ++c) pd_pre[c] = __ldg(prow + c);
  }
  griddep_wait();                                     // x may be the previous kernel's output
  // x of the slice as fp32 (zeros beyond K and for rows beyond M).
  for (int i = tid; i < kGemvMaxRows * kSlice / 2; i += kFewThreads) {
    const int m = i / (kSlice / 2), c = 2 * (i % (kSlice / 2));
    uint32_t w = 0u;
    if (m < p.M && k0 + c < p.K) w = p.x[((size_t)m * p.K + k0 + c) / 2];
    xs[m][c] = __uint_as_float(w << 16);
    xs[m][c + 1] = __uint_as_float(w & 0xFFFF0000u);
  }
  __syncthreads();
  if (tid == 0) griddep_launch_dependents();

  // ---- codes and scales (warp 0)
  if (warp == 0) {
    const float2 r6 = recip_pair(6.0f);
    if (!ROT) {
      const int m = lane >> 3, j = lane & 7;               // row, 16-channel block
      const int k = k0 + 16 * j;
      uint32_t xin[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t lo = __float_as_uint(xs[m][16 * j + 2 * i]) >> 16;
        const uint32_t hi = __float_as_uint(xs[m][16 * j + 2 * i + 1]) & 0xFFFF0000u;
        xin[i] = lo | hi;
      }
      uint64_t v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 l = lam_pre[i];
        v[i] = div_rr2(bf16x2_to_f2(xin[i]), pk2(l.x, l.y), pk2(l.z, l.w));
      }
      const float amax = amax8(v);
      uint32_t w0, w1, sb;
      if (amax < 3.0e38f) {
        sb = quant_block_rp(v, amax, r6.x, r6.y, w0, w1);
      } else {
        smooth_ieee(xin, p.lamf, k, v);
        sb = quant_block_slow(v, w0, w1);
      }
      if (m < p.M) {
        *reinterpret_cast<uint2*>(p.codes + (size_t)m * (p.Kp / 2) + k / 2) = make_uint2(w0, w1);
        p.sfa[(size_t)(k >> 6) * kSfAtomBytes + sf_atom_offset(m, (k >> 4) & 3)] = (uint8_t)sb;
      }
    } else {
      // Lanes 4m .. 4m+3: the four 32-channel quarters of row m's 128-block
      // (lanes 16-31 carry rows beyond 4 as zeros; every lane must take part
      // in the butterfly's shuffles).
      const int m = lane >> 2, qq = lane & 3;
      const int kq = k0 + 32 * qq;
      uint32_t xin[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int mm = m < kGemvMaxRows ? m : 0;
        const uint32_t lo = __float_as_uint(xs[mm][32 * qq + 2 * i]) >> 16;
        const uint32_t hi = __float_as_uint(xs[mm][32 * qq + 2 * i + 1]) & 0xFFFF0000u;
        xin[i] = m < kGemvMaxRows ? (lo | hi) : 0u;
      }
      uint64_t v[16];
      float big = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float4 l = lam_pre[i];
        v[i] = div_rr2(bf16x2_to_f2(xin[i]), pk2(l.x, l.y), pk2(l.z, l.w));
        big = amax_nan(amax_nan(big, lo2(v[i])), hi2(v[i]));
      }
      if (!(big < 3.0e38f)) smooth_ieee(xin, p.lamf, kq, v);
      hadamard128_quarter(v, qq);
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        uint64_t blk[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) blk[i] = v[8 * b + i];
        const float amax = amax8(blk);
        uint32_t w0, w1, sb;
        if (amax < 3.0e38f)
          sb = quant_block_rp(blk, amax, r6.x, r6.y, w0, w1);
        else
          sb = quant_block_slow(blk, w0, w1);
        const int k = kq + 16 * b;
        if (m < p.M) {
          *reinterpret_cast<uint2*>(p.codes + (size_t)m * (p.Kp / 2) + k / 2) = make_uint2(w0, w1);
          p.sfa[(size_t)(k >> 6) * kSfAtomBytes + sf_atom_offset(m, (k >> 4) & 3)] = (uint8_t)sb;
        }
      }
    }
  }
  // The slice that holds the last channels zero-fills the scale atoms past
  // Kp (the matrix-vector kernel reads whole 256-element K tiles' atoms).
  if (blockIdx.x == gridDim.x - 1 && tid < p.M) {
    for (int ka = p.Kp / 64; ka < p.ka_pad; ++ka)
      *reinterpret_cast<uint32_t*>(p.sfa + (size_t)ka * kSfAtomBytes + sf_atom_offset(tid, 0)) = 0u;
  }

  // ---- partial rank-R down-projection of the slice: thread t takes rank
  // t % 32 + 32 g over channel quarter t / 32 (32 channels), then the four
  // quarters are added in order.
  const int q = tid >> 5;
  for (int r0 = 0; r0 < p.R; r0 += 32) {
    const int r = r0 + lane;
    float a[kGemvMaxRows] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (r < p.R) {
      const uint4* prow = reinterpret_cast<const uint4*>(p.pdT + (size_t)r * p.Kp + k0 + 32 * q);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 pw = r0 == 0 ? pd_pre[c] : __ldg(prow + c);
        const uint32_t pv[4] = {pw.x, pw.y, pw.z, pw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int kk = 32 * q + 8 * c + 2 * i;
          const float p0 = __uint_as_float(pv[i] << 16), p1 = __uint_as_float(pv[i] & 0xFFFF0000u);
#pragma unroll
          for (int m = 0; m < kGemvMaxRows; ++m) a[m] = fmaf(xs[m][kk + 1], p1, fmaf(xs[m][kk], p0, a[m]));
        }
      }
    }
#pragma unroll
    for (int m = 0; m < kGemvMaxRows; ++m) lsum[q][m][lane] = a[m];
    __syncthreads();
    if (tid < kGemvMaxRows * 32) {
      const int m = tid >> 5;
      const float s = ((lsum[0][m][lane] + lsum[1][m][lane]) + lsum[2][m][lane]) + lsum[3][m][lane];
      if (m < p.M && r < p.R) p.part[((size_t)blockIdx.x * p.M + m) * p.R + r] = s;
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_quantize_few(const FewQuantLaunch& L, cudaStream_t stream) {
  if (L.M <= 0) return cudaSuccess;
  if (L.M > kGemvMaxRows) return cudaErrorInvalidValue;
  FewParams p;
  p.x = static_cast<const uint32_t*>(L.x);
  p.lamq = reinterpret_cast<const float4*>(L.lamq);
  p.lamf = L.lamf;
  p.pdT = static_cast<const __nv_bfloat16*>(L.pdT);
  p.codes = L.codes;
  p.sfa = L.sfa;
  p.part = L.part;
  p.M = L.M;
  p.K = L.K;
  p.Kp = L.Kp;
  p.R = L.R;
  p.ka_pad = L.ka_pad;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(L.Kp / kSlice), 1, 1);
  cfg.blockDim = dim3(kFewThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  if (L.rotate_block == 128) return cudaLaunchKernelEx(&cfg, quantize_few_kernel<true>, p);
  return cudaLaunchKernelEx(&cfg, quantize_few_kernel<false>, p);
}

int quantize_few_slices(int Kp) { return Kp / kSlice; }

}  // namespace svdq

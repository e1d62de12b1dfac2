// gemv_nvfp4.cu -- the SVDQuant W4A4 product for 1..4 token rows on CUDA cores.
//
//   y[m, n] = bf16( alpha[n] * sum_k Q(x_hat)[m, k] Q(W)[n, k]  +  sum_r L[m, r] proj_up[n, r] )
//
// ("SVDQuant W4A4", vLLM-Omni svdquant.md: the NVFP4 GEMM followed by the
// bf16 rank correction of "Runtime support".)  With at most four token rows
// the product is a matrix-vector product: every weight byte is used for at
// most eight multiply-adds, so the time is the weight read from HBM and the
// kernel is a coalesced stream, not a tensor-core tile loop.
//
// Decomposition.  One CTA of 16 warps per SM, on all but 8 SMs (left to the
// quantizer that runs before it); warp w of the grid owns weight
// rows w, w + W, w + 2W, ... (W = warps in the grid), two at a time.  Lane l
// reads 16-byte pieces l, l + 32, ... of a row (32 FP4 codes = two scale
// blocks each), so every load instruction of a warp covers 512 contiguous
// bytes.  The token rows are decoded once per CTA into shared memory as fp16
// (exact: every E2M1 value is an fp16 value), in an order that makes each
// lane's four 16-byte reads per piece conflict-free; their block scales go to
// shared memory as fp32.
//
// Arithmetic.  cvt.rn.f16x2.e2m1x2 turns a weight byte into two exact fp16
// values; the 16 products of a scale block go into two fp16 lanes of eight
// products each.  E2M1 products are multiples of 1/4 of magnitude <= 36, so a
// lane's partial sum (<= 288 in steps of 1/4) is exact in fp16, and so is the
// block sum in fp32.  The block scale product s_a * s_w of two e4m3 values is
// exact in fp32; each block adds fma(block_sum, s_a * s_w, acc) into an fp32
// accumulator, the rounding the tensor-core path also makes per block.  The
// warp reduces acc and the rank-R term with a fixed shuffle tree (results do
// not depend on timing) and stores y = bf16(fma(alpha, acc, lr)).
//
// The weights are library-owned and written once at create time (which
// synchronizes), so each warp's first two rows are requested before the
// programmatic-dependent-launch wait and stream in while the previous kernel
// (the activation quantizer) is still running.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "kcommon.cuh"
#include "svdq_kernels.h"

namespace svdq {
namespace {

constexpr int kWarps = 16, kThreads = 32 * kWarps;
// SMs left to the kernel before this one (the activation quantizer, whose K
// split for at most four rows is one cluster of up to 8 CTAs), so that every
// CTA of this kernel can start, and request its weights, while it runs.
constexpr int kReserveSms = 8;
constexpr int kPieces = 4;                 // 16-byte pieces per lane per row per pass (4096 K elements)
constexpr int kPass = 32 * kPieces;        // pieces per row per pass

struct GvParams {
  const uint8_t* qw;       // (N, Kp/2) weight codes
  const uint8_t* sfr;      // (N, Kp/16) weight block scales, row-major e4m3
  const uint8_t* codes;    // (M, Kp/2) activation codes
  const uint8_t* sfa;      // activation scale atoms (row tile 0)
  const __nv_bfloat16* lowrank;   // (M, R), when lr_part is null
  const float* lr_part;           // [n_parts][M][R] fp32 partial L, or null
  int n_parts;
  const __nv_bfloat16* pu;        // (N, R)
  const float* alpha;             // (N)
  __nv_bfloat16* y;               // (M, N)
  int M, N, K, Kp, R;
};

// Shared-memory fp16 slot of element k of a token row: within each group of
// 1024 elements, 16-byte piece q (0..3) of lane l sits at q * 256 + l * 8.
__device__ __forceinline__ int act_slot(int k) {
  return (k & ~1023) + ((k >> 3) & 3) * 256 + ((k >> 5) & 31) * 8 + (k & 7);
}

// Four bytes of packed E2M1 codes (eight values) -> four fp16 pairs, exact.
__device__ __forceinline__ void e2m1x8_to_f16x8(uint32_t w, uint32_t (&d)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(w));
}

// One e4m3 byte -> fp32, exact (the byte fills both halves of the pair, so
// the result does not depend on which half the conversion puts first).
__device__ __forceinline__ float e4m3_to_f(uint32_t byte) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"((unsigned short)(byte * 0x101u)));
  return __low2float(*reinterpret_cast<const __half2*>(&h));
}

__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ float f16x2_sum(uint32_t v) {
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&v));
  return f.x + f.y;
}

// One pass of 16-byte weight pieces of row n (and their two block-scale
// bytes each); zeros past N or the row's end.
__device__ __forceinline__ void load_pass(const GvParams& p, int n, int pass, int lane, uint4 (&v)[kPieces],
                                          uint32_t (&s)[kPieces]) {
  const int pieces = p.Kp / 32, rb = p.Kp / 2, sb = p.Kp / 16;
#pragma unroll
  for (int j = 0; j < kPieces; ++j) {
    const int u = pass * kPass + j * 32 + lane;
    if (n < p.N && u < pieces) {
      v[j] = __ldg(reinterpret_cast<const uint4*>(p.qw + (size_t)n * rb) + u);
      s[j] = __ldg(reinterpret_cast<const unsigned short*>(p.sfr + (size_t)n * sb) + u);
    } else {
      v[j] = make_uint4(0u, 0u, 0u, 0u);
      s[j] = 0u;
    }
  }
}

// A warp's first two weight rows (first pass), their proj_up entries (rank
// r = lane) and alpha.  All are library-owned weights written at create
// (which synchronizes), so they are requested before the dependency wait and
// stream in while the previous kernel is still running.
struct RowPrefetch {
  uint4 wv[2][kPieces];
  uint32_t ws2[2][kPieces];
  float pu[2], al[2];
};

__device__ __forceinline__ void prefetch_rows(const GvParams& p, int w0, int W, int lane, RowPrefetch& f) {
  load_pass(p, w0, 0, lane, f.wv[0], f.ws2[0]);
  load_pass(p, w0 + W, 0, lane, f.wv[1], f.ws2[1]);
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int n = w0 + r * W;
    f.pu[r] = 0.0f;
    f.al[r] = 0.0f;
    if (n < p.N) {
      if (lane < p.R) f.pu[r] = __bfloat162float(p.pu[(size_t)n * p.R + lane]);
      f.al[r] = __ldg(p.alpha + n);
    }
  }
}

// The product for the warp's weight rows w0, w0 + W, ... (two at a time),
// from the token rows in shared memory: act (fp16, act_slot order, kgrp
// slots per row), sa (fp32 block scales, Kp/16 per row) and lr (L, R per row).
template <int MT>
__device__ __forceinline__ void dot_rows(const GvParams& p, const uint16_t* act, const float* sa, const float* lr,
                                         int kgrp, int w0, int W, int lane, RowPrefetch& f) {
  const int pieces = p.Kp / 32, sb = p.Kp / 16;
  const int passes = (pieces + kPass - 1) / kPass;
  for (int n0 = w0; n0 < p.N; n0 += 2 * W) {
    float acc[2][MT];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[r][m] = 0.0f;
    for (int pass = 0; pass < passes; ++pass) {
      if (n0 != w0 || pass != 0) {
        load_pass(p, n0, pass, lane, f.wv[0], f.ws2[0]);
        load_pass(p, n0 + W, pass, lane, f.wv[1], f.ws2[1]);
      }
#pragma unroll
      for (int j = 0; j < kPieces; ++j) {
        const int u = pass * kPass + j * 32 + lane;
        if (u >= pieces) break;
        const int k0 = 32 * u;
        const uint4* ap = reinterpret_cast<const uint4*>(act + act_slot(k0));
        float2 sav[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) sav[m] = *reinterpret_cast<const float2*>(sa + m * sb + 2 * u);
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const uint32_t wb[4] = {f.wv[r][j].x, f.wv[r][j].y, f.wv[r][j].z, f.wv[r][j].w};
          uint32_t wf[4][4];
#pragma unroll
          for (int q = 0; q < 4; ++q) e2m1x8_to_f16x8(wb[q], wf[q]);
          const float2 sw = make_float2(e4m3_to_f(f.ws2[r][j] & 0xFF), e4m3_to_f(f.ws2[r][j] >> 8));
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            uint32_t h0 = 0u, h1 = 0u;                       // +0.0 in both halves
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 a = ap[m * (kgrp / 8) + q * 32];
              const uint32_t av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
              for (int b = 0; b < 4; ++b) {
                if (q < 2) h0 = hfma2(wf[q][b], av[b], h0);
                else h1 = hfma2(wf[q][b], av[b], h1);
              }
            }
            acc[r][m] = fmaf(f16x2_sum(h0), sav[m].x * sw.x, acc[r][m]);
            acc[r][m] = fmaf(f16x2_sum(h1), sav[m].y * sw.y, acc[r][m]);
          }
        }
      }
    }
    // Rank-R term, then the warp reductions (fixed tree) and the store.
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int n = n0 + r * W;
      if (n >= p.N) break;                                 // warp-uniform
      const float al = n0 == w0 ? f.al[r] : p.alpha[n];
      float l[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) l[m] = 0.0f;
      for (int rr = lane; rr < p.R; rr += 32) {
        const float pv = (n0 == w0 && rr == lane) ? f.pu[r] : __bfloat162float(p.pu[(size_t)n * p.R + rr]);
#pragma unroll
        for (int m = 0; m < MT; ++m) l[m] = fmaf(lr[m * p.R + rr], pv, l[m]);
      }
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        float a = acc[r][m], b = l[m];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
          a += __shfl_xor_sync(0xffffffffu, a, o);
          b += __shfl_xor_sync(0xffffffffu, b, o);
        }
        if (lane == m && m < p.M) p.y[(size_t)m * p.N + n] = __float2bfloat16_rn(fmaf(al, a, b));
      }
    }
  }
}

template <int MT>
__global__ void __launch_bounds__(kThreads, 1) gemv_nvfp4_kernel(const GvParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int kgrp = (p.Kp + 1023) & ~1023;                  // fp16 slots per token row
  uint16_t* act = reinterpret_cast<uint16_t*>(smem);        // [MT][kgrp] fp16
  float* sa = reinterpret_cast<float*>(act + MT * kgrp);    // [MT][Kp/16] block scales (0 beyond K)
  float* lr = sa + MT * (p.Kp / 16);                        // [MT][R]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int W = gridDim.x * kWarps, w0 = blockIdx.x * kWarps + warp;
  const int rb = p.Kp / 2, sb = p.Kp / 16;                  // row bytes: codes, scales
  const int K16 = p.K / 16;

  RowPrefetch f;
  prefetch_rows(p, w0, W, lane, f);

  griddep_wait();
  if (tid == 0) griddep_launch_dependents();

  // Token rows -> shared memory: codes as fp16 (8 per 4-byte word), block
  // scales as fp32 (zero for blocks at or beyond K), L as fp32.  Every
  // thread issues its loads of all three first, so their latencies overlap.
  constexpr int kCodeIters = 2, kScaleIters = 1;           // loads issued up front; any remainder uses plain loops
  uint32_t cw[kCodeIters];
  uint32_t sbv[kScaleIters];
#pragma unroll
  for (int c = 0; c < kCodeIters; ++c) {
    const int i = tid + c * kThreads;
    const int m = i / (kgrp / 8), k = (i % (kgrp / 8)) * 8;
    cw[c] = (i < MT * (kgrp / 8) && m < p.M && k < p.K) ? __ldg(reinterpret_cast<const uint32_t*>(p.codes + (size_t)m * rb + k / 2)) : 0u;
  }
#pragma unroll
  for (int c = 0; c < kScaleIters; ++c) {
    const int i = tid + c * kThreads;
    const int m = i / sb, kb = i % sb;
    sbv[c] = (i < MT * sb && m < p.M && kb < K16) ? p.sfa[(size_t)(kb >> 2) * kSfAtomBytes + sf_atom_offset(m, kb & 3)] : 0xFFFFFFFFu;
  }
  for (int i = tid + kCodeIters * kThreads; i < MT * (kgrp / 8); i += kThreads) {   // larger K: the plain loop
    const int m = i / (kgrp / 8), k = (i % (kgrp / 8)) * 8;
    uint4 o = make_uint4(0u, 0u, 0u, 0u);
    if (m < p.M && k < p.K) {
      uint32_t d[4];
      e2m1x8_to_f16x8(*reinterpret_cast<const uint32_t*>(p.codes + (size_t)m * rb + k / 2), d);
      o = make_uint4(d[0], d[1], d[2], d[3]);
    }
    *reinterpret_cast<uint4*>(act + m * kgrp + act_slot(k)) = o;
  }
  for (int i = tid + kScaleIters * kThreads; i < MT * sb; i += kThreads) {
    const int m = i / sb, kb = i % sb;
    float v = 0.0f;
    if (m < p.M && kb < K16) v = e4m3_to_f(p.sfa[(size_t)(kb >> 2) * kSfAtomBytes + sf_atom_offset(m, kb & 3)]);
    sa[i] = v;
  }
  if (p.lr_part) {
    // The few-row quantizer's per-slice partial sums of L: sixteen threads
    // per (row, rank) each add the slices s = sub, sub + 16, ... in order,
    // then a fixed shuffle tree adds the sixteen (deterministic), so every
    // load is in flight at once.
    for (int i0 = 0; i0 < MT * p.R; i0 += kThreads / 16) {
      const int i = i0 + (tid >> 4), sub = tid & 15;
      const int m = i / p.R, r = i % p.R;
      float v = 0.0f;
      if (i < MT * p.R && m < p.M)
        for (int s = sub; s < p.n_parts; s += 16) v += __ldg(p.lr_part + ((size_t)s * p.M + m) * p.R + r);
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (sub == 0 && i < MT * p.R) lr[i] = v;
    }
  } else {
    for (int i = tid; i < MT * p.R; i += kThreads) {
      const int m = i / p.R;
      lr[i] = m < p.M ? __bfloat162float(p.lowrank[i]) : 0.0f;
    }
  }
  // The first iterations' values, loaded above.
#pragma unroll
  for (int c = 0; c < kCodeIters; ++c) {
    const int i = tid + c * kThreads;
    if (i < MT * (kgrp / 8)) {
      const int m = i / (kgrp / 8), k = (i % (kgrp / 8)) * 8;
      uint32_t d[4];
      e2m1x8_to_f16x8(cw[c], d);
      *reinterpret_cast<uint4*>(act + m * kgrp + act_slot(k)) = make_uint4(d[0], d[1], d[2], d[3]);
    }
  }
#pragma unroll
  for (int c = 0; c < kScaleIters; ++c) {
    const int i = tid + c * kThreads;
    if (i < MT * sb) sa[i] = sbv[c] == 0xFFFFFFFFu ? 0.0f : e4m3_to_f(sbv[c]);
  }
  __syncthreads();
  dot_rows<MT>(p, act, sa, lr, kgrp, w0, W, lane, f);
}

template <int MT>
cudaError_t launch_mt(const GvParams& p, int grid, size_t smem, cudaStream_t stream) {
  cudaError_t e = ensure_smem_limit(gemv_nvfp4_kernel<MT>, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gemv_nvfp4_kernel<MT>, p);
}

}  // namespace

size_t gemv_smem_bytes(int M, int Kp, int R) {
  const int mt = M <= 1 ? 1 : (M <= 2 ? 2 : 4);
  const size_t kgrp = (size_t)(Kp + 1023) / 1024 * 1024;
  return (size_t)mt * (kgrp * 2 + (size_t)(Kp / 16) * 4 + (size_t)R * 4);
}

bool gemv_applies(int M, int Kp, int R) {
  return M >= 1 && M <= kGemvMaxRows && gemv_smem_bytes(M, Kp, R) <= 200 * 1024;
}

cudaError_t launch_gemv_nvfp4(const GemvLaunch& L, cudaStream_t stream) {
  if (L.M <= 0) return cudaSuccess;
  if (!gemv_applies(L.M, L.Kp, L.R)) return cudaErrorInvalidValue;
  GvParams p;
  p.qw = L.qw;
  p.sfr = L.sfr;
  p.codes = L.codes;
  p.sfa = L.sfa;
  p.lowrank = static_cast<const __nv_bfloat16*>(L.lowrank);
  p.lr_part = L.lr_part;
  p.n_parts = L.n_parts;
  p.pu = static_cast<const __nv_bfloat16*>(L.pu);
  p.alpha = L.alpha;
  p.y = static_cast<__nv_bfloat16*>(L.y);
  p.M = L.M;
  p.N = L.N;
  p.K = L.K;
  p.Kp = L.Kp;
  p.R = L.R;
  const int grid = std::max(1, std::min(L.num_sms - kReserveSms, (L.N + kWarps - 1) / kWarps));
  const size_t smem = gemv_smem_bytes(L.M, L.Kp, L.R);
  if (L.M == 1) return launch_mt<1>(p, grid, smem, stream);
  if (L.M == 2) return launch_mt<2>(p, grid, smem, stream);
  return launch_mt<4>(p, grid, smem, stream);
}

}  // namespace svdq


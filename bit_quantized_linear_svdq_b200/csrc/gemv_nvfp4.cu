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
// Decomposition.  One CTA of 16 warps owns a contiguous block of rpc weight
// rows (a multiple of 4), on at most all but 8 SMs (left to the quantizer
// that runs before it).  Its codes, block scales, proj_up rows and alpha come
// into shared memory by four bulk copies; warp w takes local rows w, w + 16,
// ... two at a time, and lane l reads 16-byte pieces l, l + 32, ... of a row
// (32 FP4 codes = two scale blocks each).  The token rows are decoded once per
// CTA into shared memory as fp16 (exact: every E2M1 value is an fp16 value),
// in an order that makes each lane's four 16-byte reads per piece
// conflict-free; their block scales go to shared memory as fp32.
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
// synchronizes), so the bulk copies are issued before the
// programmatic-dependent-launch wait: the copy engine streams them while the
// previous kernel (the activation quantizer) is still running, the threads
// reach the wait at once, and after it only the token rows are loaded.
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
  unsigned* err;
  int rpc;                        // weight rows per CTA (a multiple of 4)
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

// Shared-memory layout of a CTA (byte offsets): the weight rows' barrier and
// abort flag, codes [rpc][Kp/2], block scales [rpc][Kp/16], proj_up [rpc][R]
// bf16, alpha [rpc] f32, token rows [MT][kgrp] fp16, token block scales
// [MT][Kp/16] f32, L [MT][R] f32.
struct GvLayout {
  size_t wq, wsf, wpu, wal, act, sa, lr, total;
};
__host__ __device__ inline GvLayout gv_layout(int MT, int Kp, int R, int rpc) {
  GvLayout l;
  const size_t kgrp = (size_t)(Kp + 1023) / 1024 * 1024;
  l.wq = 16;
  l.wsf = l.wq + (size_t)rpc * (Kp / 2);
  l.wpu = l.wsf + (size_t)rpc * (Kp / 16);
  l.wal = l.wpu + (size_t)rpc * R * 2;
  l.act = l.wal + (size_t)rpc * 4;
  l.sa = l.act + (size_t)MT * kgrp * 2;
  l.lr = l.sa + (size_t)MT * (Kp / 16) * 4;
  l.total = l.lr + (size_t)MT * R * 4;
  return l;
}

template <int MT>
__global__ void __launch_bounds__(kThreads, 1) gemv_nvfp4_kernel(const GvParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  const GvLayout Ls = gv_layout(MT, p.Kp, p.R, p.rpc);
  const int kgrp = (p.Kp + 1023) & ~1023;                  // fp16 slots per token row
  const int rb = p.Kp / 2, sb = p.Kp / 16;                  // row bytes: codes, scales
  const int K16 = p.K / 16;
  uint64_t* wbar = reinterpret_cast<uint64_t*>(smem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 8);
  const uint8_t* wq = smem + Ls.wq;
  const uint8_t* wsf = smem + Ls.wsf;
  const __nv_bfloat16* wpu = reinterpret_cast<const __nv_bfloat16*>(smem + Ls.wpu);
  const float* wal = reinterpret_cast<const float*>(smem + Ls.wal);
  uint16_t* act = reinterpret_cast<uint16_t*>(smem + Ls.act);   // [MT][kgrp] fp16
  float* sa = reinterpret_cast<float*>(smem + Ls.sa);            // [MT][Kp/16] block scales (0 beyond K)
  float* lr = reinterpret_cast<float*>(smem + Ls.lr);            // [MT][R]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_begin = blockIdx.x * p.rpc;
  const int rows = max(0, min(p.rpc, p.N - n_begin));

  // This CTA's weight rows -> shared memory by bulk copies: library-owned
  // weights written at create, so requested before the dependency wait; the
  // copy engine streams them while the previous kernel runs and leaves the
  // load path free for the token rows after the wait.  Scale rows are copied
  // in pairs and alpha in fours (their buffers are padded so).
  if (tid == 0) {
    mbar_init(smem_u32(wbar), 1);
    *abort_flag = 0;
    fence_mbar_init();
    if (rows > 0) {
      const int rows2 = (rows + 1) & ~1, rows4 = (rows + 3) & ~3;
      const uint32_t wb = smem_u32(wbar);
      mbar_arrive_expect_tx(wb, (uint32_t)((size_t)rows * rb + (size_t)rows2 * sb + (size_t)rows * p.R * 2 +
                                           (size_t)rows4 * 4));
      bulk_load(smem_u32(wq), p.qw + (size_t)n_begin * rb, (uint32_t)((size_t)rows * rb), wb);
      bulk_load(smem_u32(wsf), p.sfr + (size_t)n_begin * sb, (uint32_t)((size_t)rows2 * sb), wb);
      bulk_load(smem_u32(wpu), p.pu + (size_t)n_begin * p.R, (uint32_t)((size_t)rows * p.R * 2), wb);
      bulk_load(smem_u32(wal), p.alpha + n_begin, (uint32_t)(rows4 * 4), wb);
    }
  }

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
  __syncthreads();                                          // token rows staged; barrier initialized
  // The weight rows have landed (bounded wait; on expiry the CTA records an
  // error and stores nothing).
  const bool have = rows == 0 || wait_bounded(smem_u32(wbar), 0, abort_flag, p.err, kErrGemmTimeout);
  if (!__syncthreads_and(have)) return;

  // The product: warp w takes local rows w, w + 16, ... two at a time; lane
  // l reads 16-byte pieces l, l + 32, ... of a row.
  const int pieces = p.Kp / 32;
  for (int i0 = warp; i0 < rows; i0 += 2 * kWarps) {
    const bool two = i0 + kWarps < rows;
    float acc[2][MT];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[r][m] = 0.0f;
    for (int u = lane; u < pieces; u += 32) {
      const int k0 = 32 * u;
      const uint4* ap = reinterpret_cast<const uint4*>(act + act_slot(k0));
      float2 sav[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) sav[m] = *reinterpret_cast<const float2*>(sa + m * sb + 2 * u);
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        if (r == 1 && !two) break;
        const int i = i0 + r * kWarps;
        const uint4 wv = *reinterpret_cast<const uint4*>(wq + (size_t)i * rb + 16 * u);
        const uint32_t ws2 = *reinterpret_cast<const unsigned short*>(wsf + (size_t)i * sb + 2 * u);
        const uint32_t wb[4] = {wv.x, wv.y, wv.z, wv.w};
        uint32_t wf[4][4];
#pragma unroll
        for (int q = 0; q < 4; ++q) e2m1x8_to_f16x8(wb[q], wf[q]);
        const float2 sw = make_float2(e4m3_to_f(ws2 & 0xFF), e4m3_to_f(ws2 >> 8));
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          uint32_t h0 = 0u, h1 = 0u;                       // +0.0 in both halves
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 a = ap[m * (kgrp / 8) + q * 32];
            const uint32_t av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int b2 = 0; b2 < 4; ++b2) {
              if (q < 2) h0 = hfma2(wf[q][b2], av[b2], h0);
              else h1 = hfma2(wf[q][b2], av[b2], h1);
            }
          }
          acc[r][m] = fmaf(f16x2_sum(h0), sav[m].x * sw.x, acc[r][m]);
          acc[r][m] = fmaf(f16x2_sum(h1), sav[m].y * sw.y, acc[r][m]);
        }
      }
    }
    // Rank-R term, then the warp reductions (fixed tree) and the store.
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      if (r == 1 && !two) break;                            // warp-uniform
      const int i = i0 + r * kWarps;
      float l[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) l[m] = 0.0f;
      for (int rr = lane; rr < p.R; rr += 32) {
        const float pv = __bfloat162float(wpu[(size_t)i * p.R + rr]);
#pragma unroll
        for (int m = 0; m < MT; ++m) l[m] = fmaf(lr[m * p.R + rr], pv, l[m]);
      }
      const float al = wal[i];
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        float a = acc[r][m], b = l[m];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
          a += __shfl_xor_sync(0xffffffffu, a, o);
          b += __shfl_xor_sync(0xffffffffu, b, o);
        }
        if (lane == m && m < p.M) p.y[(size_t)m * p.N + n_begin + i] = __float2bfloat16_rn(fmaf(al, a, b));
      }
    }
  }
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

namespace {

// Weight rows per CTA: enough that the grid (all but kReserveSms SMs) covers
// N, a multiple of 4, and no more than shared memory allows.
int gemv_rpc(int M, int N, int Kp, int R, int num_sms) {
  const int mt = M <= 1 ? 1 : (M <= 2 ? 2 : 4);
  const int ctas = std::max(1, num_sms - kReserveSms);
  int rpc = ((N + ctas - 1) / ctas + 3) & ~3;
  while (rpc > 4 && gv_layout(mt, Kp, R, rpc).total > 200 * 1024) rpc -= 4;
  return rpc;
}

}  // namespace

// Shared memory with the fewest weight rows per CTA (4): the product applies
// when that fits.
size_t gemv_smem_bytes(int M, int Kp, int R) {
  const int mt = M <= 1 ? 1 : (M <= 2 ? 2 : 4);
  return gv_layout(mt, Kp, R, 4).total;
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
  p.err = L.err;
  p.rpc = gemv_rpc(L.M, L.N, L.Kp, L.R, L.num_sms);
  const int grid = (L.N + p.rpc - 1) / p.rpc;
  const int mt = L.M <= 1 ? 1 : (L.M <= 2 ? 2 : 4);
  const size_t smem = gv_layout(mt, L.Kp, L.R, p.rpc).total;
  if (L.M == 1) return launch_mt<1>(p, grid, smem, stream);
  if (L.M == 2) return launch_mt<2>(p, grid, smem, stream);
  return launch_mt<4>(p, grid, smem, stream);
}

}  // namespace svdq


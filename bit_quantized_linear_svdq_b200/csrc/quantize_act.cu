// quantize_act.cu -- fused SVDQuant activation quantizer for sm_100a.
//
// One read of x produces everything the layer needs from the activations
// ("SVDQuant W4A4", vLLM-Omni svdquant.md, "Checkpoint contract"; rotation:
// "Rotate in quantization and its vLLM implementation", sections 2.1-2.2 and
// 3.3, where fusing the rotation into the quantize kernel avoids a launch and
// a round trip through memory):
//
//   x_hat = fp32(x / smooth_factor)                 per input channel
//   x_hat = fp32(butterfly_128(x_hat) * fp32(1/sqrt(128)))   (optional)
//   scale = e4m3_rne_satfinite(fp32(amax16 / 6)),  code = e2m1_rne_satfinite(fp32(x_hat / scale))
//   L     = bf16(x_hat) @ proj_down                 (fp32 accumulate, tensor cores)
//
// Work decomposition.  A CTA owns 128 token rows and a contiguous slice of
// K; the K slices of one row tile form a thread-block cluster that reduces
// its partial L in distributed shared memory (fixed order, deterministic).
// Inside a CTA:
//   warp 4 lane 0   TMA producer: x chunk (128 rows x 128 K, two 128B-swizzled
//                   boxes), proj_down^T chunk (R x 128) and {smooth, 1/smooth}
//                   into a STAGES-deep ring; also owns the TMEM allocation.
//   warps 0-3       one thread per row: smooth (+ rotate), quantize, write
//                   codes/scales to global, and write bf16(x_hat) back in place
//                   over x in shared memory -- which is exactly the 128B-swizzled
//                   K-major layout the tensor core reads as the A operand.
//   warp 5 lane 0   issues tcgen05.mma (M=128, N=R, K=16, bf16 -> fp32 TMEM)
//                   for L on each finished chunk, releasing the stage when done.
// Every wait is bounded (kWaitTimeoutNs); on expiry the CTA records an error,
// drains what it started, frees TMEM and exits.
#include <cuda_runtime.h>

#include "kcommon.cuh"
#include "svdq_kernels.h"

namespace svdq {
namespace {

constexpr int kChunk = 128;           // K elements per pipeline stage
constexpr int kRows = 128;            // token rows per CTA (TMEM lanes)
constexpr int kXStageBytes = kRows * kChunk * 2;   // 32 KB: two 64-wide swizzled boxes
constexpr int kXBoxBytes = kXStageBytes / 2;       // 16 KB
constexpr int kLamStageBytes = kChunk * 8;         // float2 per channel
constexpr int kThreads = 192;

struct QParams {
  const float2* lam2;
  uint8_t* codes;
  uint8_t* scales;
  __nv_bfloat16* lowrank;
  unsigned* err;
  int M, K, Kp, R;
  int codes_pitch, scales_pitch, k_limit, ka_pad;
  int chunks_per_cta, n_chunks, ksplit;
};

// Quantize one 16-element block: returns the scale byte, writes 16 codes as two words.
__device__ __forceinline__ uint32_t quant_block16(const float* v, uint32_t& w0, uint32_t& w1) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t sb = cvt_e4m3(__fdiv_rn(amax, 6.0f));
  const float s = e4m3_to_f32(sb);
  if (s > 0.0f) {
    float q[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) q[i] = __fdiv_rn(v[i], s);
    w0 = cvt_e2m1x8(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]);
    w1 = cvt_e2m1x8(q[8], q[9], q[10], q[11], q[12], q[13], q[14], q[15]);
  } else {
    w0 = 0u;
    w1 = 0u;
  }
  return sb;
}

__device__ __forceinline__ void unpack8(const uint4& p, float* v) {
  v[0] = bf16lo_to_f32(p.x); v[1] = bf16hi_to_f32(p.x);
  v[2] = bf16lo_to_f32(p.y); v[3] = bf16hi_to_f32(p.y);
  v[4] = bf16lo_to_f32(p.z); v[5] = bf16hi_to_f32(p.z);
  v[6] = bf16lo_to_f32(p.w); v[7] = bf16hi_to_f32(p.w);
}

__device__ __forceinline__ uint4 pack8(const float* v) {
  return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                    pack_bf16x2(v[6], v[7]));
}

// Byte offset, inside one stage's x tile, of the 16-byte group `c` (8 bf16,
// K elements 8c..8c+7 of the chunk) of row `row`: two 64-column boxes, each
// 128 rows x 128 bytes with the 128-byte swizzle (16B group index XOR row%8).
__device__ __forceinline__ uint32_t xoff(int row, int c) {
  return (uint32_t)((c >> 3) * kXBoxBytes + row * 128 + (((c & 7) ^ (row & 7)) << 4));
}

// Global writes of one quantized 16-element block.
template <bool TILED>
__device__ __forceinline__ void store_block(const QParams& p, int m, int row_in_tile, int k,
                                            uint32_t w0, uint32_t w1, uint32_t sb) {
  if (k >= p.k_limit) return;
  *reinterpret_cast<uint2*>(p.codes + (size_t)m * p.codes_pitch + (k >> 1)) = make_uint2(w0, w1);
  if (TILED) {
    const int ka = k >> 6, j = (k >> 4) & 3;
    p.scales[((size_t)(m >> 7) * p.ka_pad + ka) * kSfAtomBytes + sf_atom_offset(row_in_tile, j)] =
        (uint8_t)sb;
  } else {
    p.scales[(size_t)m * p.scales_pitch + (k >> 4)] = (uint8_t)sb;
  }
}

template <bool ROT, bool TILED>
__device__ __forceinline__ void process_chunk(const QParams& p, uint8_t* xs, const float2* lam,
                                              int row, int m, int kc) {
  const bool valid = m < p.M;
  if (ROT) {
    // The whole 128-element rotation block of this row lives in registers.
    float v[128];
#pragma unroll
    for (int c = 0; c < 16; ++c) unpack8(*reinterpret_cast<const uint4*>(xs + xoff(row, c)), v + 8 * c);
#pragma unroll
    for (int i = 0; i < 128; ++i) v[i] = __fdiv_rn(v[i], lam[i].x);
    // Walsh-Hadamard butterfly, stages h = 1, 2, ..., 64, fp32 adds.
#pragma unroll
    for (int h = 1; h < 128; h <<= 1) {
#pragma unroll
      for (int i = 0; i < 128; ++i) {
        if ((i & h) == 0) {
          const float a = v[i], b = v[i + h];
          v[i] = __fadd_rn(a, b);
          v[i + h] = __fsub_rn(a, b);
        }
      }
    }
    const float cnorm = 0.0883883461356163f;   // fp32(1/sqrt(128)) = 0x3DB504F3
#pragma unroll
    for (int i = 0; i < 128; ++i) v[i] = __fmul_rn(v[i], cnorm);
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      uint32_t w0, w1;
      const uint32_t sb = quant_block16(v + 16 * b, w0, w1);
      if (valid) store_block<TILED>(p, m, row, kc + 16 * b, w0, w1, sb);
      *reinterpret_cast<uint4*>(xs + xoff(row, 2 * b)) = pack8(v + 16 * b);
      *reinterpret_cast<uint4*>(xs + xoff(row, 2 * b + 1)) = pack8(v + 16 * b + 8);
    }
  } else {
#pragma unroll 2
    for (int b = 0; b < 8; ++b) {
      float v[16];
      unpack8(*reinterpret_cast<const uint4*>(xs + xoff(row, 2 * b)), v);
      unpack8(*reinterpret_cast<const uint4*>(xs + xoff(row, 2 * b + 1)), v + 8);
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = __fdiv_rn(v[i], lam[16 * b + i].x);
      uint32_t w0, w1;
      const uint32_t sb = quant_block16(v, w0, w1);
      if (valid) store_block<TILED>(p, m, row, kc + 16 * b, w0, w1, sb);
      *reinterpret_cast<uint4*>(xs + xoff(row, 2 * b)) = pack8(v);
      *reinterpret_cast<uint4*>(xs + xoff(row, 2 * b + 1)) = pack8(v + 8);
    }
  }
}

template <bool ROT, bool TILED, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    quantize_act_kernel(const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_pdT, const QParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int R = p.R;
  const int pd_stage_bytes = R * kChunk * 2;     // two 64-wide boxes of R rows x 128 B
  uint8_t* X = base;
  uint8_t* PD = X + STAGES * kXStageBytes;
  uint8_t* LAM = PD + STAGES * pd_stage_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(LAM + STAGES * kLamStageBytes);
  uint64_t* full = bars;                    // TMA landed
  uint64_t* xready = bars + STAGES;         // x_hat written back (128 arrivals)
  uint64_t* empty = bars + 2 * STAGES;      // MMA finished reading the stage
  uint64_t* done = bars + 3 * STAGES;       // all MMAs of this CTA finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * STAGES + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * kRows;
  const int c_begin = blockIdx.y * p.chunks_per_cta;
  const int nch = min(p.chunks_per_cta, p.n_chunks - c_begin);
  const uint32_t tmem_cols = R <= 32 ? 32u : (R <= 64 ? 64u : 128u);

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&xready[s]), kRows);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(done), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(smem_u32(tmem_slot), tmem_cols);
    tmem_relinquish();
    if (lane == 0) {
      prefetch_tmap(&tm_x);
      prefetch_tmap(&tm_pdT);
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  int issued = 0;   // producer: loads issued
  if (warp == 4) {
    if (lane == 0) {
      for (int i = 0; i < nch; ++i) {
        const int s = i % STAGES;
        if (i >= STAGES &&
            !wait_bounded(smem_u32(&empty[s]), ((i / STAGES) - 1) & 1, abort_flag, p.err, kErrQuantTimeout))
          break;
        const int kc = (c_begin + i) * kChunk;
        const uint32_t fb = smem_u32(&full[s]);
        mbar_arrive_expect_tx(fb, kXStageBytes + pd_stage_bytes + kLamStageBytes);
        uint8_t* xs = X + s * kXStageBytes;
        uint8_t* pds = PD + s * pd_stage_bytes;
        tma_load_2d(smem_u32(xs), &tm_x, fb, kc, m0);
        tma_load_2d(smem_u32(xs + kXBoxBytes), &tm_x, fb, kc + 64, m0);
        tma_load_2d(smem_u32(pds), &tm_pdT, fb, kc, 0);
        tma_load_2d(smem_u32(pds + R * 128), &tm_pdT, fb, kc + 64, 0);
        bulk_load(smem_u32(LAM + s * kLamStageBytes), p.lam2 + kc, kLamStageBytes, fb);
        issued = i + 1;
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, (uint32_t)R);
      for (int i = 0; i < nch; ++i) {
        const int s = i % STAGES;
        const uint32_t par = (i / STAGES) & 1;
        if (!wait_bounded(smem_u32(&full[s]), par, abort_flag, p.err, kErrQuantTimeout)) break;
        if (!wait_bounded(smem_u32(&xready[s]), par, abort_flag, p.err, kErrQuantTimeout)) break;
        tc_fence_after_sync();
        const uint32_t xa = smem_u32(X + s * kXStageBytes);
        const uint32_t pa = smem_u32(PD + s * pd_stage_bytes);
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk) {
          const uint64_t ad = sdesc_kmajor_sw128(xa + (kk >> 2) * kXBoxBytes + (kk & 3) * 32);
          const uint64_t bd = sdesc_kmajor_sw128(pa + (kk >> 2) * (R * 128) + (kk & 3) * 32);
          mma_bf16(tmem, ad, bd, idesc, (i | kk) != 0);
        }
        tc_commit(smem_u32(&empty[s]));
      }
      // Arrives when every MMA issued above has finished; waited on below
      // before the tensor memory is released.
      tc_commit(smem_u32(done));
    }
    __syncwarp();
  } else {
    // warps 0-3: one thread per token row
    const int row = tid;
    const int m = m0 + row;
    for (int i = 0; i < nch; ++i) {
      const int s = i % STAGES;
      if (!wait_bounded(smem_u32(&full[s]), (i / STAGES) & 1, abort_flag, p.err, kErrQuantTimeout)) break;
      const int kc = (c_begin + i) * kChunk;
      process_chunk<ROT, TILED>(p, X + s * kXStageBytes,
                                reinterpret_cast<const float2*>(LAM + s * kLamStageBytes), row, m, kc);
      fence_proxy_async_smem();
      mbar_arrive(smem_u32(&xready[s]));
    }
    // The CTA that owns the last chunk zero-fills the scale atoms beyond Kp
    // (the GEMM's last K tile reads them and they must be finite).
    if (TILED && m < p.M && c_begin + nch == p.n_chunks) {
      for (int ka = p.Kp / 64; ka < p.ka_pad; ++ka)
        *reinterpret_cast<uint32_t*>(p.scales + ((size_t)(m >> 7) * p.ka_pad + ka) * kSfAtomBytes +
                                     sf_atom_offset(row, 0)) = 0u;
    }
  }

  // ---- rank-R down-projection: TMEM -> L (cluster reduction when K is split)
  const bool want_lr = p.lowrank != nullptr;
  float* partial = reinterpret_cast<float*>(base);   // reuses the x ring once all MMAs are done
  if (want_lr && tid < kRows) {
    const bool ok = wait_bounded(smem_u32(done), 0, abort_flag, p.err, kErrQuantTimeout);
    tc_fence_after_sync();
    const int row = tid, m = m0 + row;
    if (ok) {
      for (int j = 0; j < R; j += 16) {
        uint32_t r[16];
        tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)j, r);
        tmem_ld_wait();
        if (p.ksplit == 1) {
          if (m < p.M) {
            uint4* dst = reinterpret_cast<uint4*>(p.lowrank + (size_t)m * R + j);
            float f[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) f[t] = __uint_as_float(r[t]);
            dst[0] = pack8(f);
            dst[1] = pack8(f + 8);
          }
        } else {
#pragma unroll
          for (int t = 0; t < 16; ++t) partial[row * R + j + t] = __uint_as_float(r[t]);
        }
      }
    }
  }
  if (want_lr && p.ksplit > 1) {
    cluster_sync();
    if (tid < kRows && !*abort_flag) {
      const uint32_t rank = cluster_ctarank();
      const int rows_per = kRows / p.ksplit;
      const uint32_t pbase = smem_u32(partial);
      for (int idx = tid; idx < rows_per * R; idx += kRows) {
        const int row = (int)rank * rows_per + idx / R, col = idx % R;
        const int m = m0 + row;
        if (m >= p.M) continue;
        float acc = 0.0f;
        for (int q = 0; q < p.ksplit; ++q)
          acc += ld_shared_cluster_f32(mapa_shared(pbase + (uint32_t)((row * R + col) * 4), (uint32_t)q));
        p.lowrank[(size_t)m * R + col] = __float2bfloat16_rn(acc);
      }
    }
    cluster_sync();
  }

  // ---- cleanup: after an abort, wait (bounded) for the copies this CTA started.
  if (warp == 4 && lane == 0 && *abort_flag) {
    for (int s = 0; s < STAGES && s < issued; ++s) {
      const int last = s + ((issued - 1 - s) / STAGES) * STAGES;
      wait_for(smem_u32(&full[s]), (last / STAGES) & 1, 100000000ull);
    }
  }
  if (warp == 5 && lane == 0) wait_for(smem_u32(done), 0, kWaitTimeoutNs);
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, tmem_cols);
  }
}

template <bool ROT, bool TILED, int STAGES>
cudaError_t launch_impl(const QuantLaunch& L, const QParams& p, int ksplit, cudaStream_t stream) {
  auto kern = quantize_act_kernel<ROT, TILED, STAGES>;
  const size_t smem = 1024 + (size_t)STAGES * (kXStageBytes + L.R * kChunk * 2 + kLamStageBytes) + 256;
  cudaError_t e = ensure_smem_limit(kern, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((L.M + kRows - 1) / kRows), (unsigned)ksplit, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = (unsigned)ksplit;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, L.tm_x, L.tm_pdT, p);
}

}  // namespace

cudaError_t launch_quantize_act(const QuantLaunch& L, cudaStream_t stream) {
  if (L.M <= 0) return cudaSuccess;
  const int n_chunks = L.Kp / kChunk;
  // Split K across a cluster so that small-M batches still spread over many SMs.
  const int row_tiles = (L.M + kRows - 1) / kRows;
  int ksplit = 1;
  for (int cand : {8, 4, 2}) {
    const int cpc = (n_chunks + cand - 1) / cand;
    if (cand <= n_chunks && (cand - 1) * cpc < n_chunks && row_tiles * cand <= 4 * 148) {
      ksplit = cand;
      break;
    }
  }
  if (L.lowrank == nullptr) ksplit = 1;   // no reduction needed: whole rows per CTA are fine too
  const int cpc = (n_chunks + ksplit - 1) / ksplit;

  QParams p;
  p.lam2 = reinterpret_cast<const float2*>(L.lam2);
  p.codes = L.codes;
  p.scales = L.scales;
  p.lowrank = reinterpret_cast<__nv_bfloat16*>(L.lowrank);
  p.err = L.err;
  p.M = L.M; p.K = L.K; p.Kp = L.Kp; p.R = L.R;
  p.codes_pitch = L.codes_pitch;
  p.scales_pitch = L.scales_pitch;
  p.k_limit = L.k_limit;
  p.ka_pad = L.ka_pad;
  p.chunks_per_cta = cpc;
  p.n_chunks = n_chunks;
  p.ksplit = ksplit;

  const bool rot = L.rotate_block == 128;
  if (rot) {
    return L.tiled_scales ? launch_impl<true, true, 3>(L, p, ksplit, stream)
                          : launch_impl<true, false, 3>(L, p, ksplit, stream);
  }
  return L.tiled_scales ? launch_impl<false, true, 3>(L, p, ksplit, stream)
                        : launch_impl<false, false, 3>(L, p, ksplit, stream);
}

}  // namespace svdq

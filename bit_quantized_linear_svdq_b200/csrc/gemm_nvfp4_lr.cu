// gemm_nvfp4_lr.cu -- block-scaled NVFP4 GEMM with the SVDQuant rank-R
// correction fused into its epilogue, for sm_100a tensor cores (tcgen05).
//
//   y[m, n] = bf16( alpha[n] * sum_k Q(x_hat)[m, k] Q(W)[n, k]  +  sum_r L[m, r] proj_up[n, r] )
//   alpha[n] = wcscales[n] * wtscale
//
// ("SVDQuant W4A4", vLLM-Omni svdquant.md: the NVFP4 GEMM followed by the
// bf16 rank correction of "Runtime support", fused here; shapes and scale
// layout from "Checkpoint contract".)
//
// Per CTA: one 128 x 128 output tile.
//   warp 0 lane 0   TMA producer: activation / weight code tiles (128 rows x
//                   256 K as 128 swizzled bytes), their scale atoms (bulk
//                   copies), and once per tile the L and proj_up tiles.
//   warp 1          owns 512 TMEM columns; lane 0 copies each stage's scale
//                   atoms to TMEM (tcgen05.cp) and issues the block-scaled
//                   MMAs (M=128, N=128, K=64, UE4M3 per 16) into accumulator
//                   columns [0,128); after the K loop it issues the bf16 MMAs
//                   L . proj_up^T (K = R) into a second accumulator [128,256).
//   warps 2-5       epilogue: TMEM -> registers, y = fma(alpha, acc, lr) ->
//                   bf16 -> global.
// Every wait is bounded; on expiry the CTA records an error, drains what it
// started, frees TMEM and exits.
#include <cuda_runtime.h>

#include "kcommon.cuh"
#include "svdq_kernels.h"

namespace svdq {
namespace {

constexpr int BM = 128, BN = 128;
constexpr int kKTileBytes = 128;                 // 256 FP4 elements per row per stage
constexpr int kStages = 4;
constexpr int kABytes = BM * kKTileBytes;        // 16 KB
constexpr int kBBytes = BN * kKTileBytes;        // 16 KB
constexpr int kSfaBytes = 4 * kSfAtomBytes;      // 4 K atoms x 128 rows
constexpr int kSfbBytes = (BN / 128) * 4 * kSfAtomBytes;
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;   // 36 KB
constexpr int kLrAtomBytesA = BM * 128;          // 64 bf16 of R per row
constexpr int kLrAtomBytesB = BN * 128;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColAcc = 0, kColLr = 128, kColSfa = 256, kColSfb = 288;   // SF: 2 buffers x 16

struct GParams {
  const uint8_t* sfa;
  const uint8_t* sfb;
  const float* alpha;
  __nv_bfloat16* y;
  unsigned* err;
  int M, N, R, k_tiles, ka_pad;
};

__global__ void __launch_bounds__(kThreads, 1)
    gemm_nvfp4_lr_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                         const __grid_constant__ CUtensorMap tm_l, const __grid_constant__ CUtensorMap tm_pu,
                         const GParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int RA = (p.R + 63) / 64;              // 64-wide swizzled boxes covering R
  uint8_t* stages = base;
  uint8_t* LT = stages + kStages * kStageBytes;
  uint8_t* PUT = LT + RA * kLrAtomBytesA;
  uint64_t* bars = reinterpret_cast<uint64_t*>(PUT + RA * kLrAtomBytesB);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* lr_full = bars + 2 * kStages;
  uint64_t* acc_full = bars + 2 * kStages + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nt = blockIdx.x, mt = blockIdx.y;
  const int n0 = nt * BN, m0 = mt * BM;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(lr_full), 1);
    mbar_init(smem_u32(acc_full), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  int issued = 0;
  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm_a);
      prefetch_tmap(&tm_b);
      prefetch_tmap(&tm_l);
      prefetch_tmap(&tm_pu);
      const uint32_t lb = smem_u32(lr_full);
      mbar_arrive_expect_tx(lb, (uint32_t)RA * (kLrAtomBytesA + kLrAtomBytesB));
      for (int a = 0; a < RA; ++a) {
        tma_load_2d(smem_u32(LT + a * kLrAtomBytesA), &tm_l, lb, 64 * a, m0);
        tma_load_2d(smem_u32(PUT + a * kLrAtomBytesB), &tm_pu, lb, 64 * a, n0);
      }
      for (int kt = 0; kt < p.k_tiles; ++kt) {
        const int s = kt % kStages;
        if (kt >= kStages &&
            !wait_bounded(smem_u32(&empty[s]), ((kt / kStages) - 1) & 1, abort_flag, p.err, kErrGemmTimeout))
          break;
        uint8_t* st = stages + s * kStageBytes;
        const uint32_t fb = smem_u32(&full[s]);
        mbar_arrive_expect_tx(fb, kStageBytes);
        tma_load_2d(smem_u32(st), &tm_a, fb, kt * kKTileBytes, m0);
        tma_load_2d(smem_u32(st + kABytes), &tm_b, fb, kt * kKTileBytes, n0);
        bulk_load(smem_u32(st + kABytes + kBBytes),
                  p.sfa + ((size_t)mt * p.ka_pad + (size_t)kt * 4) * kSfAtomBytes, kSfaBytes, fb);
        bulk_load(smem_u32(st + kABytes + kBBytes + kSfaBytes),
                  p.sfb + ((size_t)nt * p.ka_pad + (size_t)kt * 4) * kSfAtomBytes, kSfbBytes, fb);
        issued = kt + 1;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc_main = idesc_nvfp4(BM, BN);
      const uint32_t idesc_lr = idesc_bf16_f32(BM, BN);
      bool ok = true;
      for (int kt = 0; kt < p.k_tiles; ++kt) {
        const int s = kt % kStages;
        if (!wait_bounded(smem_u32(&full[s]), (kt / kStages) & 1, abort_flag, p.err, kErrGemmTimeout)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t st = smem_u32(stages + s * kStageBytes);
        const uint32_t sfa_col = kColSfa + (uint32_t)(kt & 1) * 16u;
        const uint32_t sfb_col = kColSfb + (uint32_t)(kt & 1) * 16u;
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
          tmem_cp_32x128b_x4(tmem + sfa_col + kb * 4, sdesc_sf_atom(st + kABytes + kBBytes + kb * kSfAtomBytes));
          tmem_cp_32x128b_x4(tmem + sfb_col + kb * 4,
                             sdesc_sf_atom(st + kABytes + kBBytes + kSfaBytes + kb * kSfAtomBytes));
        }
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
          mma_nvfp4(tmem + kColAcc, sdesc_kmajor_sw128(st + kb * 32), sdesc_kmajor_sw128(st + kABytes + kb * 32),
                    idesc_main, tmem + sfa_col + kb * 4, tmem + sfb_col + kb * 4, (kt | kb) != 0);
        }
        tc_commit(smem_u32(&empty[s]));
      }
      if (ok && wait_bounded(smem_u32(lr_full), 0, abort_flag, p.err, kErrGemmTimeout)) {
        tc_fence_after_sync();
        const uint32_t la = smem_u32(LT), pa = smem_u32(PUT);
        for (int kk = 0; kk < p.R / 16; ++kk) {
          mma_bf16(tmem + kColLr, sdesc_kmajor_sw128(la + (kk >> 2) * kLrAtomBytesA + (kk & 3) * 32),
                   sdesc_kmajor_sw128(pa + (kk >> 2) * kLrAtomBytesB + (kk & 3) * 32), idesc_lr, kk != 0);
        }
      }
      tc_commit(smem_u32(acc_full));
    }
    __syncwarp();
  } else {
    // Epilogue: warps 2..5 cover TMEM lane quadrants 2, 3, 0, 1.
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int m = m0 + row;
    const bool ok = wait_bounded(smem_u32(acc_full), 0, abort_flag, p.err, kErrGemmTimeout);
    tc_fence_after_sync();
    if (ok && !*abort_flag) {
      const bool vec_ok = (p.N & 7) == 0;
#pragma unroll 1
      for (int j = 0; j < BN / 32; ++j) {
        uint32_t acc[32], lr[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + kColAcc + j * 32, acc);
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + kColLr + j * 32, lr);
        tmem_ld_wait();
        const int n = n0 + j * 32;
        if (m < p.M && n < p.N) {
          const float4* al = reinterpret_cast<const float4*>(p.alpha + n);
          uint32_t packed[16];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float4 a4 = __ldg(al + c);
            const float y0 = fmaf(a4.x, __uint_as_float(acc[4 * c + 0]), __uint_as_float(lr[4 * c + 0]));
            const float y1 = fmaf(a4.y, __uint_as_float(acc[4 * c + 1]), __uint_as_float(lr[4 * c + 1]));
            const float y2 = fmaf(a4.z, __uint_as_float(acc[4 * c + 2]), __uint_as_float(lr[4 * c + 2]));
            const float y3 = fmaf(a4.w, __uint_as_float(acc[4 * c + 3]), __uint_as_float(lr[4 * c + 3]));
            packed[2 * c] = pack_bf16x2(y0, y1);
            packed[2 * c + 1] = pack_bf16x2(y2, y3);
          }
          __nv_bfloat16* dst = p.y + (size_t)m * p.N + n;
          if (vec_ok && n + 32 <= p.N) {
            uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
            for (int c = 0; c < 4; ++c)
              d4[c] = make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
          } else {
            const uint16_t* h = reinterpret_cast<const uint16_t*>(packed);
            uint16_t* d = reinterpret_cast<uint16_t*>(dst);
            for (int c = 0; c < 32 && n + c < p.N; ++c) d[c] = h[c];
          }
        }
      }
    }
  }

  // ---- cleanup
  if (warp == 0 && lane == 0 && *abort_flag) {
    for (int s = 0; s < kStages && s < issued; ++s) {
      const int last = s + ((issued - 1 - s) / kStages) * kStages;
      wait_for(smem_u32(&full[s]), (last / kStages) & 1, 100000000ull);
    }
    wait_for(smem_u32(lr_full), 0, 100000000ull);
  }
  if (warp == 1 && lane == 0) wait_for(smem_u32(acc_full), 0, kWaitTimeoutNs);
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_gemm_nvfp4_lr(const GemmLaunch& L, cudaStream_t stream) {
  if (L.M <= 0) return cudaSuccess;
  const int RA = (L.R + 63) / 64;
  const size_t smem = 1024 + (size_t)kStages * kStageBytes + (size_t)RA * (kLrAtomBytesA + kLrAtomBytesB) + 256;
  cudaError_t e = ensure_smem_limit(gemm_nvfp4_lr_kernel, smem);
  if (e != cudaSuccess) return e;
  GParams p;
  p.sfa = L.sfa;
  p.sfb = L.sfb;
  p.alpha = L.alpha;
  p.y = reinterpret_cast<__nv_bfloat16*>(L.y);
  p.err = L.err;
  p.M = L.M;
  p.N = L.N;
  p.R = L.R;
  p.k_tiles = L.k_tiles;
  p.ka_pad = L.ka_pad;
  dim3 grid((unsigned)((L.N + BN - 1) / BN), (unsigned)((L.M + BM - 1) / BM), 1);
  gemm_nvfp4_lr_kernel<<<grid, kThreads, smem, stream>>>(L.tm_a, L.tm_b, L.tm_l, L.tm_pu, p);
  return cudaGetLastError();
}

}  // namespace svdq

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
// Persistent kernel: one CTA per SM walks a static schedule of 128 x 128
// output tiles (tile = blockIdx.x + i * gridDim.x, M-tile fastest).
//   warp 0 lane 0   TMA producer: per K step (256 FP4 elements) the activation
//                   and weight code tiles (128 rows x 128 swizzled bytes) and
//                   their compact scale atoms (bulk copies) into a kStages
//                   ring; per tile the L and proj_up tiles.
//   warp 1          owns all 512 TMEM columns; lane 0 issues the block-scaled
//                   MMAs (M=128, N=128, K=64, UE4M3 per 16) into one of two
//                   accumulators, then the bf16 MMAs L . proj_up^T (K = R) into
//                   the rank-R accumulator.
//   warps 2-5       epilogue of tile i (TMEM -> registers, y = fma(alpha, acc,
//                   lr) -> bf16 -> global) while the tensor core runs tile i+1.
//   warps 6-9       scale warps: each writes the stage's scale factors into its
//                   own 32-lane TMEM sub-partition with tcgen05.st (every
//                   sub-partition needs all 128 rows' scales).  A register
//                   store does not occupy the tensor pipe, whereas a
//                   tcgen05.cp costs that pipe as much as a 128x128x64 MMA.
// TMEM columns: accumulators [0,128) and [128,256), rank-R accumulator
// [256,384), scale factors [384,512) (four buffers of 32 columns: A in
// +0..15, B in +16..31, 4 columns per K atom).
// Every wait is bounded; on expiry the CTA records an error, drains what it
// started, frees TMEM and exits.
#include <cuda_runtime.h>

#include "kcommon.cuh"
#include "svdq_kernels.h"

namespace svdq {
namespace {

constexpr int BM = 128, BN = 128;
constexpr int kKTileBytes = 128;                 // 256 FP4 elements per row per stage
constexpr int kMaxStages = 5;
constexpr int kABytes = BM * kKTileBytes;        // 16 KB
constexpr int kBBytes = BN * kKTileBytes;        // 16 KB
constexpr int kSfaBytes = 4 * kSfAtomBytes;      // 4 K atoms x 128 rows (2 KB)
constexpr int kSfbBytes = 4 * kSfAtomBytes;
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;   // 36 KB
constexpr int kLrAtomBytesA = BM * 128;          // 64 bf16 of R per row
constexpr int kLrAtomBytesB = BN * 128;
constexpr int kThreads = 320;
constexpr int kEpiWarps = 4;
constexpr int kSfWarp0 = 6, kSfWarps = 4;
constexpr int kSfBufs = 4;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColAcc = 0, kColLr = 256, kColSf = 384;

struct GParams {
  const uint8_t* sfa;
  const uint8_t* sfb;
  const float* alpha;
  __nv_bfloat16* y;
  unsigned* err;
  int M, N, R, k_tiles, ka_pad;
  int m_tiles, n_tiles;
  int lr_bufs;      // 2 when two L / proj_up tiles fit in shared memory, else 1
  int stages;       // depth of the K-step ring (4 or 5, as shared memory allows)
};

__device__ __forceinline__ void tile_coords(const GParams& p, int tile, int& mt, int& nt) {
  mt = tile % p.m_tiles;
  nt = tile / p.m_tiles;
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_nvfp4_lr_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                         const __grid_constant__ CUtensorMap tm_l, const __grid_constant__ CUtensorMap tm_pu,
                         const GParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // Round up to 1024 bytes by pointer arithmetic on the __shared__ array, so
  // every access below stays a shared-memory access (an integer round trip
  // would turn them into generic ones).
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int RA = (p.R + 63) / 64;              // 64-wide swizzled boxes covering R
  const int lr_buf_bytes = RA * (kLrAtomBytesA + kLrAtomBytesB);
  uint8_t* stages = base;
  uint8_t* LRB = stages + p.stages * kStageBytes;          // lr_bufs x {L tile, proj_up tile}
  uint64_t* bars = reinterpret_cast<uint64_t*>(LRB + p.lr_bufs * lr_buf_bytes);
  uint64_t* full = bars;                        // [p.stages] TMA landed
  uint64_t* empty = full + p.stages;             // [p.stages] MMAs done reading the stage
  uint64_t* sf_full = empty + p.stages;          // [kSfBufs] scale factors of a stage in TMEM
  uint64_t* lr_full = sf_full + kSfBufs;        // [2] L / proj_up tile landed
  uint64_t* lr_free = lr_full + 2;              // [2] rank-R MMAs done reading the L / proj_up tile
  uint64_t* acc_full = lr_free + 2;             // [2] accumulator (and rank-R accumulator) ready
  uint64_t* acc_free = acc_full + 2;            // [2] epilogue done reading accumulator
  uint64_t* lracc_free = acc_free + 2;          // [1] epilogue done reading the rank-R accumulator
  uint64_t* mma_done = lracc_free + 1;          // [1] every MMA of this CTA finished (teardown)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int num_tiles = p.m_tiles * p.n_tiles;

  if (tid == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < kSfBufs; ++b) mbar_init(smem_u32(&sf_full[b]), kSfWarps);
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&lr_full[b]), 1);
      mbar_init(smem_u32(&lr_free[b]), 1);
      mbar_init(smem_u32(&acc_full[b]), 1);
      mbar_init(smem_u32(&acc_free[b]), kEpiWarps);
    }
    mbar_init(smem_u32(lracc_free), kEpiWarps);
    mbar_init(smem_u32(mma_done), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // Everything above overlaps the previous kernel's tail (programmatic
  // dependent launch); nothing below runs before it has completed.
  griddep_wait();
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  if (tid == 0) griddep_launch_dependents();

  // Producer bookkeeping (for the drain after an abort).
  int issued = 0, lr_issued = 0;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm_a);
      prefetch_tmap(&tm_b);
      prefetch_tmap(&tm_l);
      prefetch_tmap(&tm_pu);
      int g = 0;   // k-stage counter across tiles
      int it = 0;
      bool stop = false;
      for (int tile = blockIdx.x; tile < num_tiles && !stop; tile += gridDim.x, ++it) {
        int mt, nt;
        tile_coords(p, tile, mt, nt);
        const int m0 = mt * BM, n0 = nt * BN;
        for (int kt = 0; kt < p.k_tiles; ++kt, ++g) {
          const int s = g % p.stages, n = g / p.stages;
          if (n >= 1 && !wait_bounded(smem_u32(&empty[s]), (n - 1) & 1, abort_flag, p.err, kErrGemmTimeout)) {
            stop = true;
            break;
          }
          uint8_t* st = stages + s * kStageBytes;
          const uint32_t fb = smem_u32(&full[s]);
          mbar_arrive_expect_tx(fb, kStageBytes);
          tma_load_2d(smem_u32(st), &tm_a, fb, kt * kKTileBytes, m0);
          tma_load_2d(smem_u32(st + kABytes), &tm_b, fb, kt * kKTileBytes, n0);
          bulk_load(smem_u32(st + kABytes + kBBytes),
                    p.sfa + ((size_t)mt * p.ka_pad + (size_t)kt * 4) * kSfAtomBytes, kSfaBytes, fb);
          bulk_load(smem_u32(st + kABytes + kBBytes + kSfaBytes),
                    p.sfb + ((size_t)nt * p.ka_pad + (size_t)kt * 4) * kSfAtomBytes, kSfbBytes, fb);
          issued = g + 1;
          if (kt == p.k_tiles - 1) {
            // L / proj_up tile of this output tile, read after its K loop.  It
            // is issued behind the tile's last K step so that, with a single
            // buffer, waiting for the previous tile's rank-R MMAs never holds
            // back the K-step ring.
            const int lb = p.lr_bufs == 2 ? (it & 1) : 0;
            const int use = p.lr_bufs == 2 ? (it >> 1) : it;
            if (use >= 1 &&
                !wait_bounded(smem_u32(&lr_free[lb]), (use - 1) & 1, abort_flag, p.err, kErrGemmTimeout)) {
              stop = true;
              break;
            }
            uint8_t* lt = LRB + lb * lr_buf_bytes;
            const uint32_t lf = smem_u32(&lr_full[lb]);
            mbar_arrive_expect_tx(lf, (uint32_t)lr_buf_bytes);
            for (int a = 0; a < RA; ++a) {
              tma_load_2d(smem_u32(lt + a * kLrAtomBytesA), &tm_l, lf, 64 * a, m0);
              tma_load_2d(smem_u32(lt + RA * kLrAtomBytesA + a * kLrAtomBytesB), &tm_pu, lf, 64 * a, n0);
            }
            lr_issued = it + 1;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc_main = idesc_nvfp4(BM, BN);
      const uint32_t idesc_lr = idesc_bf16_f32(BM, BN);
      int g = 0;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
        const int ab = it & 1;
        const uint32_t acc = tmem + kColAcc + (uint32_t)ab * BN;
        if (it >= 2 && !wait_bounded(smem_u32(&acc_free[ab]), ((it >> 1) - 1) & 1, abort_flag, p.err, kErrGemmTimeout)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        for (int kt = 0; kt < p.k_tiles; ++kt, ++g) {
          const int s = g % p.stages, b = g % kSfBufs;
          // The scale warps waited for the stage's data before writing its
          // scale factors, so their arrival also means the stage has landed.
          if (!wait_bounded(smem_u32(&sf_full[b]), (g / kSfBufs) & 1, abort_flag, p.err, kErrGemmTimeout)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t st = smem_u32(stages + s * kStageBytes);
          const uint32_t sf = tmem + kColSf + (uint32_t)b * 32u;
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            mma_nvfp4(acc, sdesc_kmajor_sw128(st + kb * 32), sdesc_kmajor_sw128(st + kABytes + kb * 32), idesc_main,
                      sf + kb * 4, sf + 16 + kb * 4, (kt | kb) != 0);
          }
          tc_commit(smem_u32(&empty[s]));
        }
        if (!ok) break;
        // rank-R correction into its own accumulator
        const int lb = p.lr_bufs == 2 ? (it & 1) : 0;
        const int use = p.lr_bufs == 2 ? (it >> 1) : it;
        if (!wait_bounded(smem_u32(&lr_full[lb]), use & 1, abort_flag, p.err, kErrGemmTimeout) ||
            (it >= 1 && !wait_bounded(smem_u32(lracc_free), (it - 1) & 1, abort_flag, p.err, kErrGemmTimeout))) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t la = smem_u32(LRB + lb * lr_buf_bytes);
        const uint32_t pa = la + RA * kLrAtomBytesA;
        for (int kk = 0; kk < p.R / 16; ++kk) {
          mma_bf16(tmem + kColLr, sdesc_kmajor_sw128(la + (kk >> 2) * kLrAtomBytesA + (kk & 3) * 32),
                   sdesc_kmajor_sw128(pa + (kk >> 2) * kLrAtomBytesB + (kk & 3) * 32), idesc_lr, kk != 0);
        }
        tc_commit(smem_u32(&lr_free[lb]));
        tc_commit(smem_u32(&acc_full[ab]));
      }
    }
    __syncwarp();
  } else if (warp >= kSfWarp0) {
    // Scale warps: stage g's scale atoms -> TMEM buffer g % kSfBufs of this
    // warp's lane quadrant.  Lane l's 16 bytes of an atom are the four columns
    // (rows l, l+32, l+64, l+96) of its TMEM lane.
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    int g = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      for (int kt = 0; kt < p.k_tiles; ++kt, ++g) {
        const int s = g % p.stages, b = g % kSfBufs;
        // Buffer b was last read by the MMAs of stage g - kSfBufs.  The whole
        // warp agrees on the outcome before the warp-wide TMEM store.
        bool w = true;
        if (g >= kSfBufs)
          w = wait_bounded(smem_u32(&empty[(g - kSfBufs) % p.stages]), ((g - kSfBufs) / p.stages) & 1, abort_flag,
                           p.err, kErrGemmTimeout);
        if (w) w = wait_bounded(smem_u32(&full[s]), (g / p.stages) & 1, abort_flag, p.err, kErrGemmTimeout);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t sfs = smem_u32(stages + s * kStageBytes + kABytes + kBBytes) + lane * 16;
        uint32_t v[32];
#pragma unroll
        for (int a = 0; a < 8; ++a) {      // atoms 0..3 of A, then 0..3 of B
          const uint4 q = ld_shared_v4(sfs + a * kSfAtomBytes);
          v[4 * a + 0] = q.x;
          v[4 * a + 1] = q.y;
          v[4 * a + 2] = q.z;
          v[4 * a + 3] = q.w;
        }
        tmem_st32(lane_base + kColSf + (uint32_t)b * 32u, v);
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sf_full[b]));
      }
    }
  } else {
    // Epilogue: warps 2..5 cover TMEM lane quadrants 2, 3, 0, 1.
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const bool vec_ok = (p.N & 7) == 0;
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      int mt, nt;
      tile_coords(p, tile, mt, nt);
      const int m = mt * BM + row, n0 = nt * BN;
      const int ab = it & 1;
      const bool w = wait_bounded(smem_u32(&acc_full[ab]), (it >> 1) & 1, abort_flag, p.err, kErrGemmTimeout);
      if (!__all_sync(0xffffffffu, w)) break;
      tc_fence_after_sync();
      const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
      for (int j = 0; j < BN / 32; ++j) {
        uint32_t acc[32], lr[32];
        tmem_ld32(lane_base + kColAcc + (uint32_t)ab * BN + j * 32, acc);
        tmem_ld32(lane_base + kColLr + j * 32, lr);
        tmem_ld_wait();
        if (j == BN / 32 - 1) {
          // Both accumulators of this tile are in registers: release them.
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(smem_u32(&acc_free[ab]));
            mbar_arrive(smem_u32(lracc_free));
          }
        }
        const int n = n0 + j * 32;
        if (m < p.M && n < p.N) {
          const float4* al = reinterpret_cast<const float4*>(p.alpha + n);
          __nv_bfloat16* dst = p.y + (size_t)m * p.N + n;
          if (vec_ok && n + 32 <= p.N) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const float4 a0 = __ldg(al + 2 * c), a1 = __ldg(al + 2 * c + 1);
              const int b = 8 * c;
              uint4 o;
              o.x = pack_bf16x2(fmaf(a0.x, __uint_as_float(acc[b + 0]), __uint_as_float(lr[b + 0])),
                                fmaf(a0.y, __uint_as_float(acc[b + 1]), __uint_as_float(lr[b + 1])));
              o.y = pack_bf16x2(fmaf(a0.z, __uint_as_float(acc[b + 2]), __uint_as_float(lr[b + 2])),
                                fmaf(a0.w, __uint_as_float(acc[b + 3]), __uint_as_float(lr[b + 3])));
              o.z = pack_bf16x2(fmaf(a1.x, __uint_as_float(acc[b + 4]), __uint_as_float(lr[b + 4])),
                                fmaf(a1.y, __uint_as_float(acc[b + 5]), __uint_as_float(lr[b + 5])));
              o.w = pack_bf16x2(fmaf(a1.z, __uint_as_float(acc[b + 6]), __uint_as_float(lr[b + 6])),
                                fmaf(a1.w, __uint_as_float(acc[b + 7]), __uint_as_float(lr[b + 7])));
              reinterpret_cast<uint4*>(dst)[c] = o;
            }
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              if (n + c < p.N) {
                const float v = fmaf(p.alpha[n + c], __uint_as_float(acc[c]), __uint_as_float(lr[c]));
                dst[c] = __float2bfloat16_rn(v);
              }
            }
          }
        }
      }
    }
  }

  // ---- cleanup
  if (warp == 0 && lane == 0 && *abort_flag) {
    for (int s = 0; s < p.stages && s < issued; ++s) {
      const int last = s + ((issued - 1 - s) / p.stages) * p.stages;
      wait_for(smem_u32(&full[s]), (last / p.stages) & 1, 100000000ull);
    }
    for (int b = 0; b < p.lr_bufs && b < lr_issued; ++b) {
      const int last_it = b + ((lr_issued - 1 - b) / p.lr_bufs) * p.lr_bufs;
      const int use = p.lr_bufs == 2 ? (last_it >> 1) : last_it;
      wait_for(smem_u32(&lr_full[b]), use & 1, 100000000ull);
    }
  }
  if (warp == 1 && lane == 0) {
    // No MMA may still be running when the tensor memory is released.
    tc_commit(smem_u32(mma_done));
    wait_for(smem_u32(mma_done), 0, kWaitTimeoutNs);
  }
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
  const int lr_buf_bytes = RA * (kLrAtomBytesA + kLrAtomBytesB);
  // Deepest ring that fits beside one L / proj_up buffer; a second buffer
  // only when the ring keeps its full depth.
  int stages = kMaxStages;
  while (stages > 2 && 1024 + (size_t)stages * kStageBytes + 256 + lr_buf_bytes > 227 * 1024) --stages;
  if (stages < kSfBufs) return cudaErrorInvalidValue;   // the scale warps' buffer reuse needs stages >= kSfBufs
  const size_t fixed = 1024 + (size_t)stages * kStageBytes + 256;
  const int lr_bufs = (fixed + 2 * (size_t)lr_buf_bytes <= 227 * 1024) ? 2 : 1;
  const size_t smem = fixed + (size_t)lr_bufs * lr_buf_bytes;
  cudaError_t e = ensure_smem_limit(gemm_nvfp4_lr_kernel, smem);
  if (e != cudaSuccess) return e;
  static int num_sms = 0;
  if (num_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (num_sms <= 0) num_sms = 148;
  }
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
  p.m_tiles = (L.M + BM - 1) / BM;
  p.n_tiles = (L.N + BN - 1) / BN;
  p.lr_bufs = lr_bufs;
  p.stages = stages;
  const int tiles = p.m_tiles * p.n_tiles;
  const int grid = tiles < num_sms ? tiles : num_sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gemm_nvfp4_lr_kernel, L.tm_a, L.tm_b, L.tm_l, L.tm_pu, p);
}

}  // namespace svdq

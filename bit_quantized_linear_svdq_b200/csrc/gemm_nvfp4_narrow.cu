// gemm_nvfp4_narrow.cu -- block-scaled NVFP4 GEMM with the SVDQuant rank-R
// correction for at most 32 token rows, for sm_100a tensor cores (tcgen05).
//
//   y[m, n] = bf16( alpha'[n] * ( sum_k Q(x_hat)[m, k] Q(W)[n, k] + sum_r L[m, r] proj_up'[n, r] ) )
//
// ("SVDQuant W4A4", vLLM-Omni svdquant.md: the NVFP4 GEMM followed by the
// bf16 rank correction of "Runtime support"; alpha folded into proj_up as in
// the 128 x 256 kernel.)  With so few rows the layer reads its weights once
// and little else.  Each tcgen05.mma costs the issuing thread about as much
// whatever its N, so the weights are the MMA's 128-row A operand (4 KB of
// weights per instruction) and the token rows its N = 32 B operand: the CTA
// computes y^T for 128 output columns over the whole of K, and no partial
// sums cross CTAs.  TMEM lane = output column n, TMEM column = token row m.
// Token rows at or beyond M are zero-filled by the TMA and carry zero scales
// (the quantizer writes zero scales for every row at or beyond M of a row
// tile), and their outputs are not stored.
//
// Persistent kernel, static schedule over 128-column tiles.  Roles:
//   warps 0-3       scale warps: per stage, tcgen05.st of the weight scales
//                   (128 rows, 4 columns per 64-element atom) and the token
//                   rows' scales (lane l holds row l's four bytes in the
//                   first of each atom's 4 columns) into their lane quadrant.
//   warps 4-7       epilogue, one per lane quadrant: alpha'[n] * acc -> bf16
//                   -> y[m, n] for m < M (32 consecutive n per store).
//   warp 8 lane 0   TMA producer: 128 weight rows and token rows 0..31 per K
//                   step (128-byte swizzle), the scale atoms; per tile the
//                   proj_up' and L rows.
//   warp 9          TMEM allocation; lane 0 issues the MMAs.
// Every wait is bounded; on expiry the CTA records an error, drains what it
// started, frees TMEM and exits.
#include <cuda_runtime.h>

#include "kcommon.cuh"
#include "svdq_kernels.h"

namespace svdq {
namespace {

constexpr int BM = 128, BN = 32;                       // output columns (weight rows), token rows
constexpr int kKTileBytes = 128;                       // 256 FP4 elements per row per stage
constexpr int kStages = 6;
constexpr int kAtoms = 4;                              // 64-element scale atoms per stage
constexpr int kWBytes = BM * kKTileBytes;              // 16 KB weight rows (A operand)
constexpr int kXBytes = BN * kKTileBytes;              // 4 KB token rows (B operand)
constexpr int kSfwBytes = kAtoms * kSfAtomBytes;       // 2 KB
constexpr int kSfxBytes = kAtoms * kSfAtomBytes;       // 2 KB: the 128-row atoms holding token rows 0..31
constexpr int kStageBytes = kWBytes + kXBytes + kSfwBytes + kSfxBytes;   // 24 KB
constexpr int kSfWarps = 4, kEpiWarp0 = 4, kEpiWarps = 4, kProdWarp = 8, kMmaWarp = 9;
constexpr int kThreads = 32 * 10;
constexpr int kSfBufs = kStages;
constexpr int kSfCols = 32;                            // per buffer: weight atoms 0..15, token atoms 16..31
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColAcc = 0, kColSf = 32;

struct NParams {
  const uint8_t* sfa;     // token-row scale atoms (row tile 0)
  const uint8_t* sfb;     // weight scale atoms
  const float* alpha;     // alpha' (folded), padded to a multiple of 256 columns
  __nv_bfloat16* y;
  unsigned* err;
  int M, N, R, k_tiles, ka_pad;
  int n_tiles;            // 128-column tiles
  int lr_row_bytes;       // bytes per row of the proj_up' / L tiles (32 or 64)
};

__device__ __forceinline__ uint64_t sdesc_rows(uint32_t saddr, int row_bytes) {
  const uint64_t layout = row_bytes == 128 ? 2ull : (row_bytes == 64 ? 4ull : 6ull);
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(16u >> 4) << 16) |
         ((uint64_t)((8u * (uint32_t)row_bytes) >> 4) << 32) | (1ull << 46) | (layout << 61);
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_nvfp4_narrow_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                             const __grid_constant__ CUtensorMap tm_pu, const __grid_constant__ CUtensorMap tm_l,
                             const NParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int pu_bytes = BM * p.lr_row_bytes, l_bytes = BN * p.lr_row_bytes;
  uint8_t* ring = base;
  uint8_t* LRB = ring + kStages * kStageBytes;                  // {proj_up' rows (A), L rows (B)}
  uint8_t* ALPHA = LRB + pu_bytes + l_bytes;                    // kEpiWarps x 32 floats
  uint64_t* bars = reinterpret_cast<uint64_t*>(ALPHA + kEpiWarps * 32 * 4);
  uint64_t* full = bars;                        // [kStages] TMA landed
  uint64_t* empty = full + kStages;             // [kStages] MMAs done reading the stage
  uint64_t* sf_full = empty + kStages;          // [kSfBufs] scales of a stage in TMEM
  uint64_t* lr_full = sf_full + kSfBufs;        // [1] proj_up' / L rows landed
  uint64_t* lr_free = lr_full + 1;              // [1] rank-R MMAs done reading them
  uint64_t* acc_full = lr_free + 1;             // [1] accumulator ready
  uint64_t* acc_free = acc_full + 1;            // [1] epilogue done reading it
  uint64_t* mma_done = acc_free + 1;            // [1] every MMA finished (teardown)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < kSfBufs; ++b) mbar_init(smem_u32(&sf_full[b]), kSfWarps);
    mbar_init(smem_u32(lr_full), 1);
    mbar_init(smem_u32(lr_free), 1);
    mbar_init(smem_u32(acc_full), 1);
    mbar_init(smem_u32(acc_free), kEpiWarps);
    mbar_init(smem_u32(mma_done), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // The weights (library-owned, written once at create time, which
  // synchronizes) do not depend on the previous kernel: the first tile's
  // first stages of weight codes and scale atoms start streaming now, while
  // that kernel (the activation quantizer) may still be running.  The stage
  // barriers are armed with the whole stage; the token half follows in the
  // producer loop.
  const int npre = (int)blockIdx.x < p.n_tiles ? min(kStages, p.k_tiles) : 0;
  if (tid == 0 && npre > 0) {
    const int n0 = (int)blockIdx.x * BM;
    prefetch_tmap(&tm_w);
    for (int i = 0; i < npre; ++i) {
      uint8_t* st = ring + i * kStageBytes;
      const uint32_t fb = smem_u32(&full[i]);
      mbar_arrive_expect_tx(fb, kStageBytes);
      tma_load_2d(smem_u32(st), &tm_w, fb, i * kKTileBytes, n0);
      bulk_load(smem_u32(st + kWBytes + kXBytes),
                p.sfb + ((size_t)blockIdx.x * p.ka_pad + (size_t)i * kAtoms) * kSfAtomBytes, kSfwBytes, fb);
    }
  }
  // Everything above overlaps the previous kernel's tail (programmatic
  // dependent launch); nothing below runs before it has completed.
  griddep_wait();
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  if (tid == 0) griddep_launch_dependents();

  int issued = 0, lr_issued = 0;
  if (warp == kProdWarp) {
    if (lane == 0) {
      prefetch_tmap(&tm_x);
      prefetch_tmap(&tm_pu);
      prefetch_tmap(&tm_l);
      int g = 0, it = 0;
      bool stop = false;
      for (int tile = blockIdx.x; tile < p.n_tiles && !stop; tile += gridDim.x, ++it) {
        const int n0 = tile * BM;
        for (int kt = 0; kt < p.k_tiles; ++kt, ++g) {
          const int s = g % kStages, n = g / kStages;
          if (n >= 1 && !wait_bounded(smem_u32(&empty[s]), (n - 1) & 1, abort_flag, p.err, kErrGemmTimeout)) {
            stop = true;
            break;
          }
          uint8_t* st = ring + s * kStageBytes;
          const uint32_t fb = smem_u32(&full[s]);
          if (g >= npre) {                         // else armed, weight half in flight since the prologue
            mbar_arrive_expect_tx(fb, kStageBytes);
            tma_load_2d(smem_u32(st), &tm_w, fb, kt * kKTileBytes, n0);
            bulk_load(smem_u32(st + kWBytes + kXBytes),
                      p.sfb + ((size_t)tile * p.ka_pad + (size_t)kt * kAtoms) * kSfAtomBytes, kSfwBytes, fb);
          }
          tma_load_2d(smem_u32(st + kWBytes), &tm_x, fb, kt * kKTileBytes, 0);
          bulk_load(smem_u32(st + kWBytes + kXBytes + kSfwBytes), p.sfa + (size_t)kt * kAtoms * kSfAtomBytes,
                    kSfxBytes, fb);
          issued = g + 1;
        }
        if (stop) break;
        // This tile's proj_up' rows and the L rows, read after its K loop.
        if (it >= 1 && !wait_bounded(smem_u32(lr_free), (it - 1) & 1, abort_flag, p.err, kErrGemmTimeout)) break;
        const uint32_t lf = smem_u32(lr_full);
        mbar_arrive_expect_tx(lf, (uint32_t)(pu_bytes + l_bytes));
        tma_load_2d(smem_u32(LRB), &tm_pu, lf, 0, n0);
        tma_load_2d(smem_u32(LRB + pu_bytes), &tm_l, lf, 0, 0);
        lr_issued = it + 1;
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      const uint32_t idesc_main = idesc_nvfp4(BM, BN);
      const uint32_t idesc_lr = idesc_bf16_f32(BM, BN);
      int g = 0, it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x, ++it) {
        if (it >= 1 && !wait_bounded(smem_u32(acc_free), (it - 1) & 1, abort_flag, p.err, kErrGemmTimeout)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        for (int kt = 0; kt < p.k_tiles; ++kt, ++g) {
          const int s = g % kStages, b = g % kSfBufs;
          // The scale warps waited for the stage's data before writing its
          // scales, so their arrival also means the stage has landed.
          if (!wait_bounded(smem_u32(&sf_full[b]), (g / kSfBufs) & 1, abort_flag, p.err, kErrGemmTimeout)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t st = smem_u32(ring + s * kStageBytes);
          const uint32_t sf = tmem + kColSf + (uint32_t)b * kSfCols;
          // One descriptor per operand and stage; a 32-byte K step inside the
          // swizzled row adds 2 to the address field (address >> 4).
          const uint64_t wd = sdesc_rows(st, kKTileBytes), xd = sdesc_rows(st + kWBytes, kKTileBytes);
#pragma unroll
          for (int kb = 0; kb < kAtoms; ++kb)
            mma_nvfp4(tmem + kColAcc, wd + 2 * kb, xd + 2 * kb, idesc_main, sf + 4 * kb, sf + 16 + 4 * kb,
                      (kt | kb) != 0);
          tc_commit(smem_u32(&empty[s]));
        }
        if (!ok) break;
        if (!wait_bounded(smem_u32(lr_full), it & 1, abort_flag, p.err, kErrGemmTimeout)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t pa = smem_u32(LRB), la = pa + pu_bytes;
        for (int kk = 0; kk < p.R / 16; ++kk)
          mma_bf16(tmem + kColAcc, sdesc_rows(pa + kk * 32, p.lr_row_bytes), sdesc_rows(la + kk * 32, p.lr_row_bytes),
                   idesc_lr, 1u);
        tc_commit(smem_u32(lr_free));
        tc_commit(smem_u32(acc_full));
      }
    }
    __syncwarp();
  } else if (warp < kSfWarps) {
    // Scale warps: stage g's scales -> TMEM buffer g % kSfBufs of this warp's
    // lane quadrant.  Weight atom a -> columns 4a..4a+3 (lane l: rows l,
    // l+32, l+64, l+96 of the tile); token atom a -> column 16 + 4a (lane l:
    // token row l's four bytes), the layout of a 128-row B block of which the
    // N = 32 MMA reads rows 0..31; columns 17 + 4a .. 19 + 4a are zero.
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    int g = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x) {
      for (int kt = 0; kt < p.k_tiles; ++kt, ++g) {
        const int s = g % kStages, b = g % kSfBufs;
        // Buffer b was last read by the MMAs of stage g - kSfBufs.  The whole
        // warp agrees on the outcome before the warp-wide TMEM store.
        bool w = true;
        if (g >= kSfBufs)
          w = wait_bounded(smem_u32(&empty[(g - kSfBufs) % kStages]), ((g - kSfBufs) / kStages) & 1, abort_flag,
                           p.err, kErrGemmTimeout);
        if (w) w = wait_bounded(smem_u32(&full[s]), (g / kStages) & 1, abort_flag, p.err, kErrGemmTimeout);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint8_t* sfs = ring + s * kStageBytes + kWBytes + kXBytes;
        uint32_t v[16], vx[16];
#pragma unroll
        for (int a = 0; a < kAtoms; ++a) {
          const uint4 qa = ld_shared_v4(smem_u32(sfs + a * kSfAtomBytes + lane * 16));
          v[4 * a + 0] = qa.x;
          v[4 * a + 1] = qa.y;
          v[4 * a + 2] = qa.z;
          v[4 * a + 3] = qa.w;
          vx[4 * a] = *reinterpret_cast<const uint32_t*>(sfs + kSfwBytes + a * kSfAtomBytes + lane * 16);
          vx[4 * a + 1] = vx[4 * a + 2] = vx[4 * a + 3] = 0u;
        }
        tmem_st16(lane_base + kColSf + (uint32_t)b * kSfCols, v);
        tmem_st16(lane_base + kColSf + (uint32_t)b * kSfCols + 16, vx);
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sf_full[b]));
      }
    }
  } else if (warp < kEpiWarp0 + kEpiWarps) {
    // Epilogue warp: lane quadrant q = warp & 3, output column n = n0 + 32q +
    // lane, TMEM columns = token rows.
    const int q = warp & 3;
    int it = 0;
    for (int tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x, ++it) {
      const int n = tile * BM + 32 * q + lane;
      const float a_n = __ldg(p.alpha + n);            // alpha' padded to a multiple of 256 columns
      const bool w = wait_bounded(smem_u32(acc_full), it & 1, abort_flag, p.err, kErrGemmTimeout);
      if (!__all_sync(0xffffffffu, w)) break;
      tc_fence_after_sync();
      uint32_t acc[32];
      tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + kColAcc, acc);
      tmem_ld_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(acc_free));
      if (n < p.N) {
#pragma unroll
        for (int m = 0; m < BN; ++m)
          if (m < p.M) p.y[(size_t)m * p.N + n] = __float2bfloat16_rn(a_n * __uint_as_float(acc[m]));
      }
    }
  }

  // ---- cleanup
  if (warp == kProdWarp && lane == 0 && *abort_flag) {
    for (int s = 0; s < kStages && s < issued; ++s) {
      const int last = s + ((issued - 1 - s) / kStages) * kStages;
      wait_for(smem_u32(&full[s]), (last / kStages) & 1, 100000000ull);
    }
    if (lr_issued > 0) wait_for(smem_u32(lr_full), (lr_issued - 1) & 1, 100000000ull);
  }
  if (warp == kMmaWarp && lane == 0) {
    // No MMA may still be running when the tensor memory is released.
    tc_commit(smem_u32(mma_done));
    wait_for(smem_u32(mma_done), 0, kWaitTimeoutNs);
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

size_t narrow_smem_bytes(int row_bytes) {
  return 1024 + (size_t)kStages * kStageBytes + (size_t)(BM + BN) * row_bytes + kEpiWarps * 32 * 4 + 512;
}

}  // namespace

// 9..32 rows.  At 1..8 rows the split-K kernel is faster (6.5 against 7.5 us
// at M = 1, K = N = 4096): this kernel's K loop is a chain of k_tiles x 4 MMAs
// issued by one thread (~80 cycles each whatever N), which split-K shortens.
bool gemm_narrow_applies(int M, int R) { return M > 8 && M <= BN && R <= 32; }

cudaError_t launch_gemm_nvfp4_narrow(const GemmLaunch& L, cudaStream_t stream) {
  if (L.M <= 0) return cudaSuccess;
  if (!gemm_narrow_applies(L.M, L.R)) return cudaErrorInvalidValue;
  const int row_bytes = gemm_n256_lr_row_bytes(L.R);
  const size_t smem = narrow_smem_bytes(row_bytes);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_limit(gemm_nvfp4_narrow_kernel, smem);
  if (e != cudaSuccess) return e;
  static int num_sms = 0;
  if (num_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (num_sms <= 0) num_sms = 148;
  }
  NParams p;
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
  p.n_tiles = (L.N + BM - 1) / BM;
  p.lr_row_bytes = row_bytes;
  const int grid = p.n_tiles < num_sms ? p.n_tiles : num_sms;
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
  // GemmLaunch: tm_b = weight rows {128, 128}, tm_a = token rows {128, 32},
  // tm_pu = proj_up' rows {row_bytes / 2, 128}, tm_l = L rows {row_bytes / 2, 32}.
  return cudaLaunchKernelEx(&cfg, gemm_nvfp4_narrow_kernel, L.tm_b, L.tm_a, L.tm_pu, L.tm_l, p);
}

}  // namespace svdq

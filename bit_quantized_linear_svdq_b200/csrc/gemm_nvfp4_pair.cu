// gemm_nvfp4_pair.cu -- block-scaled NVFP4 GEMM with the SVDQuant rank-R
// correction on 256 x 256 output tiles, each computed by a pair of CTAs (a
// 2-CTA cluster on two SMs) with tcgen05 .cta_group::2 MMAs, for sm_100a.
//
//   y[m, n] = bf16( alpha'[n] * ( sum_k Q(x_hat)[m, k] Q(W)[n, k] + sum_r L[m, r] proj_up'[n, r] ) )
//   proj_up'[n, r] = bf16(proj_up[n, r] / alpha[n]),  alpha[n] = wcscales[n] * wtscale
//
// ("SVDQuant W4A4", vLLM-Omni svdquant.md: the NVFP4 GEMM followed by the
// bf16 rank correction of "Runtime support"; alpha is folded into proj_up as
// in the 128 x 256 kernel.)  One pair MMA (M = 256, N = 256, K = 64) runs on
// the tensor cores of both SMs.  CTA r of the pair keeps output rows
// 128r .. 128r+127 of the tile in its own TMEM; per K step it holds its 128
// activation rows and weight rows 128r .. 128r+127 of the tile in shared
// memory, and each SM's tensor core reads the other weight half from the peer.
// Per SM and K step that is 32 KB of operands plus 6 KB of scales for the work
// the 128 x 256 kernel brings in 48 KB + 6 KB for: the K loop is bound by the
// bytes the L2 delivers to each SM, so the pair tile runs it faster.
//
// Persistent kernel, one pair per two SMs, static schedule over 256 x 256
// tiles (M-tile fastest).  Roles, in both CTAs unless stated:
//   warp 0 lane 0   producer: the A and B half-tiles with pair TMA loads whose
//                   bytes complete on the even CTA's `full` barrier (the even
//                   CTA expects both CTAs' bytes); the stage's scale atoms (A:
//                   this CTA's 128 rows, B: all 256 columns) with plain bulk
//                   loads on this CTA's `sf_ld` barrier; per tile the L rows
//                   and proj_up' half of this CTA, again on the even CTA.
//   warp 1          TMEM: a pair allocation of 512 columns (accumulator
//                   [0,256), four scale buffers of 48 columns from 256).  In
//                   the even CTA lane 0 issues the pair MMAs and commits them
//                   to the barriers of both CTAs.
//   warps 2-5       scale warps: tcgen05.st of each stage's scales into this
//                   CTA's TMEM (the pair MMA reads A scales of the CTA's own
//                   rows and B scales of all N columns from each SM's TMEM),
//                   then arrive on the even CTA's `sf_full`.
//   warps 6-9       epilogue of this CTA's 128 rows: TMEM -> alpha' * acc ->
//                   bf16 into shared-memory boxes -> TMA stores to y; each warp
//                   releases the accumulator on the even CTA's `acc_free`
//                   (eight arrivals: four warps in each CTA) after its last
//                   TMEM load.
// Every wait is bounded; on expiry the CTA records an error and skips its
// remaining work.  Both CTAs always reach the final cluster barrier, so
// neither exits while the other may still touch its shared memory.
//
// The MX instantiation serves the MXFP4 matmul of "Rotate in quantization and
// its vLLM implementation", section 3.3 (FP-Quant): E2M1 operands with one
// UE8M0 (power-of-two) scale per 32 K elements, stored in the same 512-byte
// atoms with the two block scales of each 64-element K step in bytes j = 0, 1
// (bytes 2, 3 zero), and no rank-R branch (R = 0): y = bf16(alpha * acc).
#include <cuda_runtime.h>

#include <map>
#include <mutex>

#include "kcommon.cuh"
#include "svdq_kernels.h"

namespace svdq {
namespace {

constexpr int BM = 256, BMC = 128, BN = 256;     // pair tile rows, rows per CTA, tile columns
constexpr int kKTileBytes = 128;                 // 256 FP4 elements per row per stage
constexpr int kMaxStages = 4;                    // ring depth: 4, or 3 when the rank-R tiles need the room
constexpr int kAtoms = 4;                        // 64-element scale atoms per stage
constexpr int kABytes = BMC * kKTileBytes;       // 16 KB: this CTA's activation rows
constexpr int kBBytes = (BN / 2) * kKTileBytes;  // 16 KB: this CTA's half of the weight rows
constexpr int kSfaBytes = kAtoms * kSfAtomBytes;      // 128 rows (2 KB)
constexpr int kSfbBytes = 2 * kAtoms * kSfAtomBytes;  // all 256 columns, two 128-row halves (4 KB)
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;   // 38 KB
constexpr int kSfWarp0 = 2, kSfWarps = 4;
constexpr int kEpiWarp0 = 6, kEpiWarps = 4;
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr int kSfCols = 48;
constexpr int kEpiCols = BN * 4 / kEpiWarps;     // columns per epilogue warp
constexpr int kStageOutBytes = 32 * 128;         // per epilogue warp: a 64-column x 32-row bf16 box
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColAcc = 0, kColSf = 256;
constexpr uint16_t kPairMask = 0x3;              // both CTAs of the cluster

struct PParams {
  const uint8_t* sfa;
  const uint8_t* sfb;
  const float* alpha;     // alpha' (folded), padded to a multiple of 256 columns
  __nv_bfloat16* y;
  unsigned* err;
  int M, N, R, k_tiles, ka_pad;
  int m_tiles;            // 256-row tiles
  int m_tiles128;         // 128-row scale tiles that exist in the workspace
  int n_tiles;            // 256-column tiles
  int lr_row_bytes;       // bytes per row of one L / proj_up' box in shared memory (32, 64 or 128)
  int lr_boxes;           // boxes of lr_row_bytes / 2 ranks per row (R <= 32: 1; else ceil(R / 64))
  int y_mode;             // 3: through shared-memory boxes and TMA stores (N % 8 == 0); 0: element stores
};

__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
// Two fp32 products, each rounded once (as two fmul.rn).
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ uint64_t sdesc_rows(uint32_t saddr, int row_bytes) {
  const uint64_t layout = row_bytes == 128 ? 2ull : (row_bytes == 64 ? 4ull : 6ull);
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(16u >> 4) << 16) |
         ((uint64_t)((8u * (uint32_t)row_bytes) >> 4) << 32) | (1ull << 46) | (layout << 61);
}

template <int kStages, bool MX>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_nvfp4_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                           const __grid_constant__ CUtensorMap tm_l, const __grid_constant__ CUtensorMap tm_pu,
                           const __grid_constant__ CUtensorMap tm_y, const PParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  constexpr int kSfBufs = kStages;
  const int lr_box_bytes = BMC * p.lr_row_bytes;                // 128 rows of one box
  const int lr_half_bytes = p.lr_boxes * lr_box_bytes;          // this CTA's L rows (or proj_up' rows)
  uint8_t* stages = base;
  uint8_t* OUT = stages + kStages * kStageBytes;                // kEpiWarps x 2 x kStageOutBytes
  uint8_t* ALPHA = OUT + kEpiWarps * 2 * kStageOutBytes;        // kEpiWarps x kEpiCols floats
  uint8_t* LRB = ALPHA + kEpiWarps * kEpiCols * 4;              // {L rows, proj_up' half} of this CTA
  uint64_t* bars = reinterpret_cast<uint64_t*>(LRB + 2 * lr_half_bytes);
  uint64_t* full = bars;                        // [stages] both CTAs' A/B landed (even CTA)
  uint64_t* empty = full + kMaxStages;          // [stages] pair MMAs done reading the stage
  uint64_t* sf_ld = empty + kMaxStages;         // [stages] this CTA's scale atoms landed
  uint64_t* sf_full = sf_ld + kMaxStages;       // [stages] scales in both TMEMs (even CTA)
  uint64_t* lr_full = sf_full + kMaxStages;     // [1] both CTAs' L / proj_up' landed (even CTA)
  uint64_t* lr_free = lr_full + 1;              // [1] rank-R MMAs done reading them
  uint64_t* acc_full = lr_free + 1;             // [1] accumulator ready
  uint64_t* acc_free = acc_full + 1;            // [1] both epilogues done reading (even CTA)
  uint64_t* mma_done = acc_free + 1;            // [1] every MMA finished (teardown)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();      // 0: even CTA (issues the MMAs), 1: its peer
  const bool leader = rank == 0;
  const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);
  const int num_tiles = p.m_tiles * p.n_tiles;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
      mbar_init(smem_u32(&sf_ld[s]), 1);
    }
    for (int b = 0; b < kSfBufs; ++b) mbar_init(smem_u32(&sf_full[b]), 2 * kSfWarps);
    mbar_init(smem_u32(lr_full), 1);
    mbar_init(smem_u32(lr_free), 1);
    mbar_init(smem_u32(acc_full), 1);
    mbar_init(smem_u32(acc_free), 2 * kEpiWarps);
    mbar_init(smem_u32(mma_done), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // The peer signals this CTA's barriers only after both have initialized them.
  cluster_sync();
  // Everything above overlaps the previous kernel's tail (programmatic
  // dependent launch); nothing below runs before it has completed.
  griddep_wait();
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  if (tid == 0) griddep_launch_dependents();

  int issued = 0, lr_issued = 0;
  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm_a);
      prefetch_tmap(&tm_b);
      prefetch_tmap(&tm_l);
      prefetch_tmap(&tm_pu);
      int g = 0, it = 0;
      bool stop = false;
      for (int tile = pair; tile < num_tiles && !stop; tile += npairs, ++it) {
        const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
        const int mrow0 = mt * BM + BMC * (int)rank;          // this CTA's activation rows
        const int mt128 = 2 * mt + (int)rank;
        const bool has_rows = mt128 < p.m_tiles128;           // else every row is beyond M
        const int nrow0 = nt * BN + (BN / 2) * (int)rank;     // this CTA's weight rows
        for (int kt = 0; kt < p.k_tiles; ++kt, ++g) {
          const int s = g % kStages, n = g / kStages;
          if (n >= 1 && !wait_bounded(smem_u32(&empty[s]), (n - 1) & 1, abort_flag, p.err, kErrGemmTimeout)) {
            stop = true;
            break;
          }
          uint8_t* st = stages + s * kStageBytes;
          const uint32_t fb = smem_u32(&full[s]);
          if (leader) mbar_arrive_expect_tx(fb, 2u * (kABytes + kBBytes));
          tma_load_2d_pair(smem_u32(st), &tm_a, fb, kt * kKTileBytes, mrow0);
          tma_load_2d_pair(smem_u32(st + kABytes), &tm_b, fb, kt * kKTileBytes, nrow0);
          const uint32_t sb = smem_u32(&sf_ld[s]);
          mbar_arrive_expect_tx(sb, (uint32_t)((has_rows ? kSfaBytes : 0) + kSfbBytes));
          if (has_rows)
            bulk_load(smem_u32(st + kABytes + kBBytes),
                      p.sfa + ((size_t)mt128 * p.ka_pad + (size_t)kt * kAtoms) * kSfAtomBytes, kSfaBytes, sb);
#pragma unroll
          for (int h = 0; h < 2; ++h)
            bulk_load(smem_u32(st + kABytes + kBBytes + kSfaBytes + h * (kSfbBytes / 2)),
                      p.sfb + ((size_t)(2 * nt + h) * p.ka_pad + (size_t)kt * kAtoms) * kSfAtomBytes, kSfbBytes / 2,
                      sb);
          issued = g + 1;
          if (kt == p.k_tiles - 1 && p.R > 0) {
            // This CTA's L rows and proj_up' half, read after the K loop.
            if (it >= 1 && !wait_bounded(smem_u32(lr_free), (it - 1) & 1, abort_flag, p.err, kErrGemmTimeout)) {
              stop = true;
              break;
            }
            const uint32_t lf = smem_u32(lr_full);
            if (leader) mbar_arrive_expect_tx(lf, (uint32_t)(4 * lr_half_bytes));
            for (int bx = 0; bx < p.lr_boxes; ++bx) {
              tma_load_2d_pair(smem_u32(LRB + bx * lr_box_bytes), &tm_l, lf, bx * (p.lr_row_bytes / 2), mrow0);
              tma_load_2d_pair(smem_u32(LRB + lr_half_bytes + bx * lr_box_bytes), &tm_pu, lf,
                               bx * (p.lr_row_bytes / 2), nrow0);
            }
            lr_issued = it + 1;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      const uint32_t idesc_main = MX ? idesc_mxfp4(BM, BN) : idesc_nvfp4(BM, BN);
      const uint32_t idesc_lr = idesc_bf16_f32(BM, BN);
      int g = 0, it = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += npairs, ++it) {
        if (it >= 1 &&
            !wait_bounded(smem_u32(acc_free), (it - 1) & 1, abort_flag, p.err, kErrGemmTimeout)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        for (int kt = 0; kt < p.k_tiles; ++kt, ++g) {
          const int s = g % kStages, b = g % kSfBufs;
          if (!wait_bounded(smem_u32(&full[s]), (g / kStages) & 1, abort_flag, p.err, kErrGemmTimeout) ||
              !wait_bounded(smem_u32(&sf_full[b]), (g / kSfBufs) & 1, abort_flag, p.err, kErrGemmTimeout)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t st = smem_u32(stages + s * kStageBytes);
          const uint32_t sf = tmem + kColSf + (uint32_t)b * kSfCols;
#pragma unroll
          for (int kb = 0; kb < kAtoms; ++kb) {
            if (MX)
              mma_mxfp4_pair(tmem + kColAcc, sdesc_rows(st + kb * 32, kKTileBytes),
                             sdesc_rows(st + kABytes + kb * 32, kKTileBytes), idesc_main, sf + 4 * kb,
                             sf + 16 + 8 * kb, (kt | kb) != 0);
            else
              mma_nvfp4_pair(tmem + kColAcc, sdesc_rows(st + kb * 32, kKTileBytes),
                             sdesc_rows(st + kABytes + kb * 32, kKTileBytes), idesc_main, sf + 4 * kb,
                             sf + 16 + 8 * kb, (kt | kb) != 0);
          }
          tc_commit_pair(smem_u32(&empty[s]), kPairMask);
        }
        if (!ok) break;
        if (p.R > 0) {                                       // no rank-R branch when R == 0
          if (!wait_bounded(smem_u32(lr_full), it & 1, abort_flag, p.err, kErrGemmTimeout)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t la = smem_u32(LRB), pa = la + lr_half_bytes;
          const int per_box = p.lr_row_bytes / 32;           // K = 16 bf16 = 32 bytes per MMA
          for (int kk = 0; kk < p.R / 16; ++kk) {
            const int off = (kk / per_box) * lr_box_bytes + (kk % per_box) * 32;
            mma_bf16_pair(tmem + kColAcc, sdesc_rows(la + off, p.lr_row_bytes),
                          sdesc_rows(pa + off, p.lr_row_bytes), idesc_lr, 1u);
          }
          tc_commit_pair(smem_u32(lr_free), kPairMask);
        }
        tc_commit_pair(smem_u32(acc_full), kPairMask);
      }
    }
    __syncwarp();
  } else if (warp < kSfWarp0 + kSfWarps) {
    // Scale warps: stage g's scale atoms -> TMEM buffer g % kSfBufs of this
    // warp's lane quadrant, in the layout of the 128 x 256 kernel (A atom a ->
    // columns 4a..4a+3; B atom kb -> 16+8kb..+3 for columns 0-127 of the tile,
    // +4..+7 for columns 128-255).
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    int g = 0;
    bool ok = true;
    for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
      for (int kt = 0; kt < p.k_tiles; ++kt, ++g) {
        const int s = g % kStages, b = g % kSfBufs;
        // Buffer b was last read by the pair MMAs of stage g - kSfBufs.  The
        // whole warp agrees on the outcome before the warp-wide TMEM store.
        bool w = true;
        if (g >= kSfBufs)
          w = wait_bounded(smem_u32(&empty[(g - kSfBufs) % kStages]), ((g - kSfBufs) / kStages) & 1, abort_flag,
                           p.err, kErrGemmTimeout);
        if (w) w = wait_bounded(smem_u32(&sf_ld[s]), (g / kStages) & 1, abort_flag, p.err, kErrGemmTimeout);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t sfs = smem_u32(stages + s * kStageBytes + kABytes + kBBytes) + lane * 16;
        uint32_t v0[32], v1[16];            // columns 0..31 and 32..47 of the buffer
#pragma unroll
        for (int i = 0; i < 12; ++i) {
          const uint32_t src = i < 4 ? sfs + i * kSfAtomBytes
                                     : sfs + kSfaBytes + ((i - 4) & 1) * (kSfbBytes / 2) + ((i - 4) >> 1) * kSfAtomBytes;
          const uint4 q = ld_shared_v4(src);
          if (i < 8) {
            v0[4 * i + 0] = q.x;
            v0[4 * i + 1] = q.y;
            v0[4 * i + 2] = q.z;
            v0[4 * i + 3] = q.w;
          } else {
            v1[4 * i - 32] = q.x;
            v1[4 * i - 31] = q.y;
            v1[4 * i - 30] = q.z;
            v1[4 * i - 29] = q.w;
          }
        }
        tmem_st32(lane_base + kColSf + (uint32_t)b * kSfCols, v0);
        tmem_st16(lane_base + kColSf + (uint32_t)b * kSfCols + 32, v1);
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive_on(smem_u32(&sf_full[b]), 0u);
      }
    }
  } else {
    // Epilogue warp e: TMEM lane quadrant q = warp & 3 (rows 32q..32q+31 of
    // this CTA's half of the tile), all 256 columns, in 64-column chunks.
    // Chunk pc + 1 is read from TMEM while chunk pc is converted.  With
    // y_mode 3 a chunk goes, as bf16, into one of the warp's two 64-column x
    // 32-row boxes (128-byte rows, 16-byte chunk c of row r at
    // r * 128 + (c ^ (r % 8)) * 16: the TMA 128-byte swizzle, conflict-free for
    // the row-per-lane writes) and leaves with a TMA store.  Nothing waits for
    // global memory before the accumulator is released: the release follows
    // the last TMEM load, and the stores drain while the pair starts the next
    // tile.
    const int e = warp - kEpiWarp0;
    const int q = warp & 3, hc = e >> 2;
    const int row = q * 32 + lane;
    uint8_t* outp = OUT + e * 2 * kStageOutBytes;
    float* alpha_w = reinterpret_cast<float*>(ALPHA + e * kEpiCols * 4);
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16) + kColAcc + (uint32_t)(hc * kEpiCols);
    if (p.y_mode == 3 && e == 0 && lane == 0) prefetch_tmap(&tm_y);
    int it = 0;
    for (int tile = pair; tile < num_tiles; tile += npairs, ++it) {
      const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
      const int m0 = mt * BM + BMC * (int)rank, m = m0 + row;
      const int nw = nt * BN + hc * kEpiCols;
      {
        float4 a[kEpiCols / 128];
#pragma unroll
        for (int i = 0; i < kEpiCols / 128; ++i) a[i] = __ldg(reinterpret_cast<const float4*>(p.alpha + nw) + 32 * i + lane);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < kEpiCols / 128; ++i) reinterpret_cast<float4*>(alpha_w)[32 * i + lane] = a[i];
        __syncwarp();
      }
      const bool w = wait_bounded(smem_u32(acc_full), it & 1, abort_flag, p.err, kErrGemmTimeout);
      if (!__all_sync(0xffffffffu, w)) break;
      tc_fence_after_sync();
      // Chunk pc + 1 is read from TMEM while chunk pc is converted.
      uint32_t acc[2][2][32];
      tmem_ld32(lane_base, acc[0][0]);
      tmem_ld32(lane_base + 32, acc[0][1]);
#pragma unroll
      for (int pc = 0; pc < kEpiCols / 64; ++pc) {
        const int nl0 = 64 * pc;
        tmem_ld_wait();
        if (pc + 1 < kEpiCols / 64) {
          tmem_ld32(lane_base + nl0 + 64, acc[(pc + 1) & 1][0]);
          tmem_ld32(lane_base + nl0 + 96, acc[(pc + 1) & 1][1]);
        } else {
          // Every TMEM load of this warp has completed: release the accumulator.
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive_on(smem_u32(acc_free), 0u);
        }
        uint8_t* box = outp + (pc & 1) * kStageOutBytes;
        if (p.y_mode == 3) {
          // The store issued from this box two chunks ago has read it.
          if (lane == 0) bulk_wait_read<1>();
          __syncwarp();
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int nl = nl0 + 32 * u;
          const uint32_t* a = acc[pc & 1][u];
          uint32_t o[16];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float4 a4 = reinterpret_cast<const float4*>(alpha_w)[(nl >> 2) + c];
            const uint64_t lo =
                mul_f32x2(pack_f32x2(a4.x, a4.y), pack_f32x2(__uint_as_float(a[4 * c]), __uint_as_float(a[4 * c + 1])));
            const uint64_t hi = mul_f32x2(pack_f32x2(a4.z, a4.w),
                                          pack_f32x2(__uint_as_float(a[4 * c + 2]), __uint_as_float(a[4 * c + 3])));
            o[2 * c] = pack_bf16x2(__uint_as_float((uint32_t)lo), __uint_as_float((uint32_t)(lo >> 32)));
            o[2 * c + 1] = pack_bf16x2(__uint_as_float((uint32_t)hi), __uint_as_float((uint32_t)(hi >> 32)));
          }
          if (p.y_mode == 3) {
            uint4* rowp = reinterpret_cast<uint4*>(box + lane * 128);
#pragma unroll
            for (int c = 0; c < 4; ++c)
              rowp[(4 * u + c) ^ (lane & 7)] = make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
          } else if (m < p.M) {
            __nv_bfloat16* dst = p.y + (size_t)m * p.N + nw + nl;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              if (nw + nl + c < p.N) {
                const uint32_t pr = o[c >> 1];
                dst[c] = __ushort_as_bfloat16((unsigned short)((c & 1) ? (pr >> 16) : (pr & 0xFFFFu)));
              }
            }
          }
        }
        if (p.y_mode == 3) {
          fence_proxy_async_smem();
          __syncwarp();
          // The tensor map clips the parts of the box beyond M and N; a box
          // that starts beyond them is not issued.
          if (lane == 0 && m0 + 32 * q < p.M && nw + nl0 < p.N) {
            tma_store_2d(&tm_y, smem_u32(box), nw + nl0, m0 + 32 * q);
            bulk_commit();
          }
        }
      }
    }
    if (p.y_mode == 3 && lane == 0) bulk_wait<0>();
  }

  // ---- cleanup
  if (warp == 0 && lane == 0 && *abort_flag) {
    // Wait (bounded) for the copies this CTA started: its scale atoms land on
    // its own barrier; the pair loads' bytes are counted by the even CTA.
    for (int s = 0; s < kStages && s < issued; ++s) {
      const int last = s + ((issued - 1 - s) / kStages) * kStages;
      wait_for(smem_u32(&sf_ld[s]), (last / kStages) & 1, 100000000ull);
      if (leader) wait_for(smem_u32(&full[s]), (last / kStages) & 1, 100000000ull);
    }
    if (leader && lr_issued > 0) wait_for(smem_u32(lr_full), (lr_issued - 1) & 1, 100000000ull);
  }
  if (warp == 1 && lane == 0) {
    // No pair MMA may still be running when the tensor memory is released.
    if (leader) tc_commit_pair(smem_u32(mma_done), kPairMask);
    wait_for(smem_u32(mma_done), 0, kWaitTimeoutNs);
  }
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

int pair_lr_boxes(int R) { return R <= 32 ? 1 : (R + 63) / 64; }

size_t pair_smem_bytes(int R, int stages) {
  return 1024 + (size_t)stages * kStageBytes + (size_t)kEpiWarps * (2 * kStageOutBytes + kEpiCols * 4) +
         (size_t)2 * pair_lr_boxes(R) * BMC * gemm_pair_lr_row_bytes(R) + 256;
}

// Deepest ring (4, else 3 stages) that fits beside the rank-R tiles.
int pair_stages(int R) { return pair_smem_bytes(R, kMaxStages) <= 227 * 1024 ? kMaxStages : kMaxStages - 1; }

// Pairs that can be resident at once (cached per device, ring depth and
// shared-memory size).
template <int kStages>
int max_active_pairs(size_t smem) {
  static std::mutex mu;
  static std::map<std::pair<int, size_t>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  auto key = std::make_pair(dev, smem);
  auto f = cache.find(key);
  if (f != cache.end()) return f->second;
  int n = 0;
  if (ensure_smem_limit(gemm_nvfp4_pair_kernel<kStages, false>, smem) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_nvfp4_pair_kernel<kStages, false>, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();   // clear a failed query
  cache[key] = n;
  return n;
}

int max_active_pairs_for(int R) {
  const size_t smem = pair_smem_bytes(R, pair_stages(R));
  return pair_stages(R) == kMaxStages ? max_active_pairs<kMaxStages>(smem) : max_active_pairs<kMaxStages - 1>(smem);
}

template <int kStages, bool MX>
cudaError_t launch_pair(const GemmLaunch& L, const PParams& p, size_t smem, int max_pairs, cudaStream_t stream) {
  cudaError_t e = ensure_smem_limit(gemm_nvfp4_pair_kernel<kStages, MX>, smem);
  if (e != cudaSuccess) return e;
  const int tiles = p.m_tiles * p.n_tiles;
  const int pairs = tiles < max_pairs ? tiles : max_pairs;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, gemm_nvfp4_pair_kernel<kStages, MX>, L.tm_a, L.tm_b, L.tm_l, L.tm_pu, L.tm_y, p);
}

}  // namespace

int gemm_pair_lr_row_bytes(int R) { return R <= 16 ? 32 : (R <= 32 ? 64 : 128); }

bool gemm_pair_available(int R) {
  return R <= 128 && pair_smem_bytes(R, pair_stages(R)) <= 227 * 1024 && max_active_pairs_for(R) > 0;
}

cudaError_t launch_gemm_nvfp4_pair(const GemmLaunch& L, cudaStream_t stream) {
  if (L.M <= 0) return cudaSuccess;
  if (L.R > 128 || L.R < 0) return cudaErrorInvalidValue;
  const int stages = pair_stages(L.R);
  const size_t smem = pair_smem_bytes(L.R, stages);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  const int max_pairs = max_active_pairs_for(L.R);
  if (max_pairs <= 0) return cudaErrorInvalidConfiguration;
  PParams p;
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
  p.m_tiles128 = (L.M + BMC - 1) / BMC;
  p.n_tiles = (L.N + BN - 1) / BN;
  p.lr_row_bytes = gemm_pair_lr_row_bytes(L.R);
  p.lr_boxes = pair_lr_boxes(L.R);
  p.y_mode = (L.N % 8) == 0 ? 3 : 0;
  if (L.mx)
    return stages == kMaxStages ? launch_pair<kMaxStages, true>(L, p, smem, max_pairs, stream)
                                : launch_pair<kMaxStages - 1, true>(L, p, smem, max_pairs, stream);
  return stages == kMaxStages ? launch_pair<kMaxStages, false>(L, p, smem, max_pairs, stream)
                              : launch_pair<kMaxStages - 1, false>(L, p, smem, max_pairs, stream);
}

}  // namespace svdq

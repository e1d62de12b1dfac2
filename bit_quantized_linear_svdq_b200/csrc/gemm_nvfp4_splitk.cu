// gemm_nvfp4_splitk.cu -- the SVDQuant W4A4 GEMM for few token rows, with K
// split over a thread-block cluster, for sm_100a tensor cores (tcgen05).
//
//   y[m, n] = bf16( alpha[n] * sum_k Q(x_hat)[m, k] Q(W)[n, k]  +  sum_r L[m, r] proj_up[n, r] )
//
// ("SVDQuant W4A4", vLLM-Omni svdquant.md: the NVFP4 GEMM followed by the
// bf16 rank correction of "Runtime support".)  With few rows the 128 x 256
// output tiles are too few to occupy the GPU and the time is the weight read,
// so each tile's K range is split over the S CTAs (S = 2, 4 or 8) of a
// cluster, every CTA reading 1/S of the tile's weights:
//   warp 0 lane 0   TMA producer for the CTA's K slice (128 rows of activation
//                   codes, 256 rows of weight codes, compact scale atoms; a
//                   3-stage ring of 54 KB).
//   warp 1          owns 512 TMEM columns: accumulator [0,256), scale factors
//                   [256,400); lane 0 issues the block-scaled MMAs (M=128,
//                   N=256, K=64, UE4M3 per 16).
//   warps 2-5       scale warps (tcgen05.st of each stage's scale factors).
//   warps 6-9       epilogue: after a cluster barrier (every K loop done, so
//                   the stage ring is free), each pushes the fp32 partial
//                   sums of its valid rows into the shared memory of the CTA
//                   that owns those columns (256/S columns per rank); after a
//                   second barrier each owner adds the S slots in rank order
//                   (a fixed order: results do not depend on timing), adds
//                   L . proj_up^T on CUDA cores, scales by alpha and stores bf16.
// Every wait is bounded; on expiry the CTA records an error, drains what it
// started, frees TMEM and exits (still passing both cluster barriers).
#include <cuda_runtime.h>

#include "kcommon.cuh"
#include "svdq_kernels.h"

namespace svdq {
namespace {

constexpr int BM = 128, BN = 256;
constexpr int kKTileBytes = 128;                 // 256 FP4 elements per row per stage
constexpr int kStages = 3;
constexpr int kAtoms = 4;
constexpr int kABytes = BM * kKTileBytes;        // 16 KB
constexpr int kBBytes = BN * kKTileBytes;        // 32 KB
constexpr int kSfaBytes = kAtoms * kSfAtomBytes;
constexpr int kSfbBytes = 2 * kAtoms * kSfAtomBytes;
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;   // 54 KB
constexpr int kSfWarp0 = 2, kSfWarps = 4;
constexpr int kEpiWarp0 = 6, kEpiWarps = 4;
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr int kSfBufs = kStages;
constexpr int kSfCols = 48;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColAcc = 0, kColSf = 256;
constexpr int kRecvBytes = BM * BN * 4;         // [S][128 rows][256/S] fp32 partial sums
static_assert(kRecvBytes <= kStages * kStageBytes, "receive buffer must fit in the stage ring");
// After the K loops, shared memory from the base holds: the receive buffer,
// then this tile's L rows (128 x R bf16) and the owner's proj_up rows
// (256/S x R bf16), then (past the ring when R is large) nothing else: the
// barriers follow the larger of the ring and this epilogue area.
__host__ __device__ constexpr int epi_bytes(int R) { return kRecvBytes + BM * R * 2 + BN * R * 2 + BN * 4; }
__host__ __device__ constexpr int body_bytes(int R) {
  return epi_bytes(R) > kStages * kStageBytes ? epi_bytes(R) : kStages * kStageBytes;
}

struct GParams {
  const uint8_t* sfa;
  const uint8_t* sfb;
  const float* alpha;             // (N padded) wcscales * wtscale
  const __nv_bfloat16* lowrank;   // L (M, R)
  const __nv_bfloat16* pu;        // proj_up (N, R)
  __nv_bfloat16* y;
  unsigned* err;
  int M, N, R, k_tiles, ka_pad;
  int m_tiles, n_tiles;           // n_tiles of 256 columns
  int S, kpc;                     // K slices per tile (cluster size), K tiles per slice
};

__global__ void __launch_bounds__(kThreads, 1)
    gemm_nvfp4_splitk_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                             const GParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* stages = base;
  float* recv = reinterpret_cast<float*>(base);            // after the K loops: [S][128 rows][256/S] fp32
  __nv_bfloat16* lrows = reinterpret_cast<__nv_bfloat16*>(base + kRecvBytes);       // [128][R]
  __nv_bfloat16* purows = lrows + BM * p.R;                                          // [R][256/S]
  float* alph = reinterpret_cast<float*>(purows + BN * p.R);                         // [256/S]
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + body_bytes(p.R));
  uint64_t* full = bars;                        // [kStages]
  uint64_t* empty = full + kStages;             // [kStages]
  uint64_t* sf_full = empty + kStages;          // [kSfBufs]
  uint64_t* acc_full = sf_full + kSfBufs;       // [1]
  uint64_t* mma_done = acc_full + 1;            // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x;
  const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
  const int m0 = mt * BM, n0 = nt * BN;
  const int rank = (int)cluster_ctarank();       // = K slice
  const int kt0 = rank * p.kpc;
  const int nk = min(p.kpc, p.k_tiles - kt0);    // >= 1 (host guarantees)
  const int mvalid = min(BM, p.M - m0);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < kSfBufs; ++b) mbar_init(smem_u32(&sf_full[b]), kSfWarps);
    mbar_init(smem_u32(acc_full), 1);
    mbar_init(smem_u32(mma_done), 1);
    *abort_flag = 0;
    fence_mbar_init();
    // The weights (library-owned, written once at create time, which
    // synchronizes) do not depend on the previous kernel: the first stages'
    // weight codes and scale atoms start streaming now, while that kernel
    // (the activation quantizer) may still be running.  Each stage's barrier
    // is armed with the whole stage; its activation half follows below.
    prefetch_tmap(&tm_b);
    for (int i = 0; i < min(nk, kStages); ++i) {
      uint8_t* st = stages + i * kStageBytes;
      const uint32_t fb = smem_u32(&full[i]);
      const int kt = kt0 + i;
      mbar_arrive_expect_tx(fb, kStageBytes);
      tma_load_2d(smem_u32(st + kABytes), &tm_b, fb, kt * kKTileBytes, n0);
#pragma unroll
      for (int h = 0; h < 2; ++h)
        bulk_load(smem_u32(st + kABytes + kBBytes + kSfaBytes + h * (kSfbBytes / 2)),
                  p.sfb + ((size_t)(2 * nt + h) * p.ka_pad + (size_t)kt * kAtoms) * kSfAtomBytes, kSfbBytes / 2, fb);
    }
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

  int issued = 0;
  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm_a);
      for (int i = 0; i < nk; ++i) {
        const int s = i % kStages, n = i / kStages, kt = kt0 + i;
        if (n >= 1 && !wait_bounded(smem_u32(&empty[s]), (n - 1) & 1, abort_flag, p.err, kErrGemmTimeout)) break;
        uint8_t* st = stages + s * kStageBytes;
        const uint32_t fb = smem_u32(&full[s]);
        if (n >= 1) {                              // the first kStages stages: armed, weights in flight
          mbar_arrive_expect_tx(fb, kStageBytes);
          tma_load_2d(smem_u32(st + kABytes), &tm_b, fb, kt * kKTileBytes, n0);
#pragma unroll
          for (int h = 0; h < 2; ++h)
            bulk_load(smem_u32(st + kABytes + kBBytes + kSfaBytes + h * (kSfbBytes / 2)),
                      p.sfb + ((size_t)(2 * nt + h) * p.ka_pad + (size_t)kt * kAtoms) * kSfAtomBytes, kSfbBytes / 2,
                      fb);
        }
        tma_load_2d(smem_u32(st), &tm_a, fb, kt * kKTileBytes, m0);
        bulk_load(smem_u32(st + kABytes + kBBytes),
                  p.sfa + ((size_t)mt * p.ka_pad + (size_t)kt * kAtoms) * kSfAtomBytes, kSfaBytes, fb);
        issued = i + 1;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_nvfp4(BM, BN);
      bool ok = true;
      for (int i = 0; i < nk; ++i) {
        const int s = i % kStages, b = i % kSfBufs;
        // The scale warps waited for the stage's data before writing its
        // scale factors, so their arrival also means the stage has landed.
        if (!wait_bounded(smem_u32(&sf_full[b]), (i / kSfBufs) & 1, abort_flag, p.err, kErrGemmTimeout)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t st = smem_u32(stages + s * kStageBytes);
        const uint32_t sf = tmem + kColSf + (uint32_t)b * kSfCols;
#pragma unroll
        for (int kb = 0; kb < kAtoms; ++kb)
          mma_nvfp4(tmem + kColAcc, sdesc_kmajor_sw128(st + kb * 32), sdesc_kmajor_sw128(st + kABytes + kb * 32), idesc,
                    sf + 4 * kb, sf + 16 + 8 * kb, (i | kb) != 0);
        tc_commit(smem_u32(&empty[s]));
      }
      if (ok) tc_commit(smem_u32(acc_full));
    }
    __syncwarp();
  } else if (warp < kSfWarp0 + kSfWarps) {
    // Scale warps: stage i's scale atoms -> TMEM buffer i % kSfBufs of this
    // warp's lane quadrant (columns: A atom a -> 4a..4a+3; B atom kb ->
    // 16+8kb+0..3 for rows 0-127, +4..7 for rows 128-255).
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    for (int i = 0; i < nk; ++i) {
      const int s = i % kStages, b = i % kSfBufs;
      bool w = true;
      if (i >= kSfBufs)
        w = wait_bounded(smem_u32(&empty[(i - kSfBufs) % kStages]), ((i - kSfBufs) / kStages) & 1, abort_flag, p.err,
                         kErrGemmTimeout);
      if (w) w = wait_bounded(smem_u32(&full[s]), (i / kStages) & 1, abort_flag, p.err, kErrGemmTimeout);
      if (!__all_sync(0xffffffffu, w)) break;
      tc_fence_after_sync();
      const uint32_t sfs = smem_u32(stages + s * kStageBytes + kABytes + kBBytes) + lane * 16;
      uint32_t v0[32], v1[16];
#pragma unroll
      for (int a = 0; a < 12; ++a) {
        const uint32_t src = a < 4 ? sfs + a * kSfAtomBytes
                                   : sfs + kSfaBytes + ((a - 4) & 1) * (kSfbBytes / 2) + ((a - 4) >> 1) * kSfAtomBytes;
        const uint4 q = ld_shared_v4(src);
        if (a < 8) {
          v0[4 * a + 0] = q.x;
          v0[4 * a + 1] = q.y;
          v0[4 * a + 2] = q.z;
          v0[4 * a + 3] = q.w;
        } else {
          v1[4 * a - 32] = q.x;
          v1[4 * a - 31] = q.y;
          v1[4 * a - 30] = q.z;
          v1[4 * a - 29] = q.w;
        }
      }
      tmem_st32(lane_base + kColSf + (uint32_t)b * kSfCols, v0);
      tmem_st16(lane_base + kColSf + (uint32_t)b * kSfCols + 32, v1);
      tmem_st_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sf_full[b]));
    }
  }

  // ---- cluster reduction of the S partial tiles
  const int cpo = BN / p.S;                      // columns owned by each rank (32, 64 or 128)
  bool acc_ok = true;
  if (warp >= kEpiWarp0) {
    const bool w = wait_bounded(smem_u32(acc_full), 0, abort_flag, p.err, kErrGemmTimeout);
    acc_ok = __all_sync(0xffffffffu, w);
    tc_fence_after_sync();
  }
  cluster_sync();                                // every CTA's MMAs are done: the stage rings are free
  // (warp-uniform: the TMEM loads below are warp-wide instructions)
  if (warp >= kEpiWarp0 && __all_sync(0xffffffffu, acc_ok && !*abort_flag)) {
    const int q = warp & 3;
    const int row = 32 * q + lane;
    if (32 * q < mvalid) {                       // this quadrant holds at least one existing row
      const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16) + kColAcc;
      const uint32_t recv_s = smem_u32(recv);
#pragma unroll 1
      for (int j = 0; j < BN; j += 32) {
        uint32_t a[32];
        tmem_ld32(lane_base + (uint32_t)j, a);
        tmem_ld_wait();
        if (row < mvalid) {
          const int owner = j / cpo;
          const uint32_t dst = mapa_shared(
              recv_s + (uint32_t)(((rank * BM + row) * cpo + (j - owner * cpo)) * 4), (uint32_t)owner);
#pragma unroll
          for (int t = 0; t < 8; ++t)
            st_shared_cluster_v4(dst + 16u * t, __uint_as_float(a[4 * t]), __uint_as_float(a[4 * t + 1]),
                                 __uint_as_float(a[4 * t + 2]), __uint_as_float(a[4 * t + 3]));
        }
      }
    }
  }
  // While the partials arrive: this tile's L rows ([row][R]) and this rank's
  // proj_up columns transposed ([R][cpo]) into shared memory, so that in the
  // sums below a warp reads one L row (broadcast) and 32 consecutive proj_up
  // entries (no bank conflict).
  {
    const int rv = p.R / 8;                      // 16-byte vectors per row (R is a multiple of 16)
    const uint4* lsrc = reinterpret_cast<const uint4*>(p.lowrank + (size_t)m0 * p.R);
    for (int i = tid; i < mvalid * rv; i += kThreads) reinterpret_cast<uint4*>(lrows)[i] = __ldg(lsrc + i);
    const int nown = max(0, min(cpo, p.N - (n0 + rank * cpo)));
    const uint4* psrc = reinterpret_cast<const uint4*>(p.pu + (size_t)(n0 + rank * cpo) * p.R);
    for (int i = tid; i < nown * rv; i += kThreads) {
      const int c = i / rv, r8 = 8 * (i % rv);
      const uint4 v = __ldg(psrc + i);
      const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
      for (int t = 0; t < 8; ++t) purows[(size_t)(r8 + t) * cpo + c] = e[t];
    }
    for (int c = tid; c < nown; c += kThreads) alph[c] = p.alpha[n0 + rank * cpo + c];
  }
  cluster_sync();                                // every partial has landed in its owner's buffer
  if (!*abort_flag) {
    // This rank's columns [n0 + rank * cpo, +cpo), one (row, column) per
    // thread (columns fastest): sum the slots in rank order, add
    // L . proj_up^T, scale by alpha, store bf16.
    for (int idx = tid; idx < mvalid * cpo; idx += kThreads) {
      const int row = idx / cpo, col = idx % cpo;
      const int m = m0 + row, n = n0 + rank * cpo + col;
      if (n >= p.N) continue;
      float acc = 0.f;
      for (int sl = 0; sl < p.S; ++sl) acc += recv[(size_t)(sl * BM + row) * cpo + col];
      // L . proj_up^T: 16 channels per step, four independent partial sums.
      const __nv_bfloat162* lrow = reinterpret_cast<const __nv_bfloat162*>(lrows + (size_t)row * p.R);
      const __nv_bfloat16* pcol = purows + col;
      float lr4[4] = {0.f, 0.f, 0.f, 0.f};
      for (int r0 = 0; r0 < p.R; r0 += 16) {
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const float2 l2 = __bfloat1622float2(lrow[r0 / 2 + t]);
          lr4[t & 3] = fmaf(l2.x, __bfloat162float(pcol[(size_t)(r0 + 2 * t) * cpo]), lr4[t & 3]);
          lr4[t & 3] = fmaf(l2.y, __bfloat162float(pcol[(size_t)(r0 + 2 * t + 1) * cpo]), lr4[t & 3]);
        }
      }
      const float lr = (lr4[0] + lr4[1]) + (lr4[2] + lr4[3]);
      p.y[(size_t)m * p.N + n] = __float2bfloat16_rn(fmaf(alph[col], acc, lr));
    }
  }

  // ---- cleanup
  if (warp == 0 && lane == 0 && *abort_flag) {
    for (int s = 0; s < kStages && s < issued; ++s) {
      const int last = s + ((issued - 1 - s) / kStages) * kStages;
      wait_for(smem_u32(&full[s]), (last / kStages) & 1, 100000000ull);
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

// Clusters of S CTAs of this kernel that the GPU can hold at once (0 if unknown).
int max_active_clusters(int S, int R) {
  static int cache[2][9] = {};
  const int ri = R <= 64 ? 0 : 1;
  if (cache[ri][S] == 0) {
    const size_t smem = 1024 + (size_t)body_bytes(R <= 64 ? 64 : 128) + 256;
    int n = 0;
    if (ensure_smem_limit(gemm_nvfp4_splitk_kernel, smem) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(1, (unsigned)S, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = smem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 1;
      attr[0].val.clusterDim.y = (unsigned)S;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, gemm_nvfp4_splitk_kernel, &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();
    cache[ri][S] = n > 0 ? n : -1;
  }
  return cache[ri][S];
}

int gemm_splitk_slices(int M, int N, int R, int k_tiles, int num_sms) {
  // Only for at most 32 rows: beyond that the partial sums pushed between
  // CTAs and the per-row epilogue cost more than the idle SMs save (measured:
  // faster at 1 and 16 rows, slower at 64).
  if (M > 32) return 1;
  const int tiles = (N + BN - 1) / BN;
  if (2 * tiles > num_sms) return 1;
  for (int s = 8; s >= 2; s >>= 1) {
    const int kpc = (k_tiles + s - 1) / s;
    if (tiles * s > num_sms || s > k_tiles || (s - 1) * kpc >= k_tiles) continue;
    if (max_active_clusters(s, R) < tiles) continue;   // every cluster must be resident at once
    return s;
  }
  return 1;
}

cudaError_t launch_gemm_nvfp4_splitk(const GemmLaunch& L, const void* lowrank, const void* proj_up, int S,
                                     cudaStream_t stream) {
  if (L.M <= 0) return cudaSuccess;
  if (S != 2 && S != 4 && S != 8) return cudaErrorInvalidValue;
  const size_t smem = 1024 + (size_t)body_bytes(L.R) + 256;
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_limit(gemm_nvfp4_splitk_kernel, smem);
  if (e != cudaSuccess) return e;
  GParams p;
  p.sfa = L.sfa;
  p.sfb = L.sfb;
  p.alpha = L.alpha;
  p.lowrank = reinterpret_cast<const __nv_bfloat16*>(lowrank);
  p.pu = reinterpret_cast<const __nv_bfloat16*>(proj_up);
  p.y = reinterpret_cast<__nv_bfloat16*>(L.y);
  p.err = L.err;
  p.M = L.M;
  p.N = L.N;
  p.R = L.R;
  p.k_tiles = L.k_tiles;
  p.ka_pad = L.ka_pad;
  p.m_tiles = (L.M + BM - 1) / BM;
  p.n_tiles = (L.N + BN - 1) / BN;
  p.S = S;
  p.kpc = (L.k_tiles + S - 1) / S;
  if ((S - 1) * p.kpc >= L.k_tiles) return cudaErrorInvalidValue;   // a slice would be empty
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(p.m_tiles * p.n_tiles), (unsigned)S, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = (unsigned)S;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, gemm_nvfp4_splitk_kernel, L.tm_a, L.tm_b, p);
}

}  // namespace svdq

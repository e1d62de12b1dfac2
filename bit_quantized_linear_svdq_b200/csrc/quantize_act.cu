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
// Inside a CTA (320 threads, one CTA per SM):
//   warp 8 lane 0   TMA producer: x chunk (128 rows x 128 K, two 128B-swizzled
//                   boxes), proj_down^T chunk (R x 128) and the smooth factors
//                   into a ring of up to 4 stages; warp 8 also owns the TMEM
//                   allocation.
//   warps 0-7       without rotation: each thread one 16-channel block of four
//                   rows; with rotation: four threads per row (32 K elements
//                   each, two rows per chunk in turn): smooth (+ rotate),
//                   quantize, write codes/scales to global, and write bf16(x_hat)
//                   back in place over x in shared memory -- exactly the
//                   128B-swizzled K-major layout the tensor core reads as A.
//   warp 9 lane 0   issues tcgen05.mma (M=128, N=R, K=16, bf16 -> fp32 TMEM)
//                   for L on each finished chunk, releasing the stage when done.
//
// Exact fp32 division without the divide unit: with y = RN(1/b),
//   q0 = RN(a*y), r = RN(a - b*q0) (fused), q1 = RN(q0 + r*y) (fused)
// is the correctly rounded a/b (Markstein's iteration; checked exhaustively
// for every significand pair that occurs here: bf16/bf16 for the smoothing,
// fp32/e4m3 and fp32/6 for the scale and codes).  The reciprocals come from
// create time (1/smooth) and a per-CTA table over the 127 e4m3 scales.  Two
// lanes run per instruction (fma.rn.f32x2).  Blocks whose values overflow or
// hold NaN take an IEEE-division slow path, so results equal the divide
// unit's in every case.
//
// Every wait is bounded (kWaitTimeoutNs); on expiry the CTA records an error,
// drains what it started, frees TMEM and exits.
#include <cuda_runtime.h>

#include <cstdlib>

#include "hadamard.cuh"
#include "kcommon.cuh"
#include "nvfp4_block.cuh"
#include "svdq_kernels.h"

namespace svdq {
namespace {

constexpr int kChunk = 128;                        // K elements per pipeline stage
constexpr int kRows = 128;                         // token rows per CTA (TMEM lanes)
constexpr int kMaxStages = 4;                     // ring depth: as many as shared memory allows
constexpr int kXStageBytes = kRows * kChunk * 2;   // 32 KB: two 64-wide swizzled boxes
constexpr int kXBoxBytes = kXStageBytes / 2;       // 16 KB
constexpr int kLamStageBytes = kChunk * 8;         // float4 {-s0,-s1,1/s0,1/s1} per channel pair
// Forward-layout outputs of one chunk are staged in shared memory and written
// with one TMA tensor store (codes, 128 rows x 64 bytes) and one bulk copy (the
// chunk's two adjacent scale atoms).
constexpr int kCodeStageBytes = kRows * kChunk / 2;   // 8 KB
constexpr int kSfStageBytes = 2 * kSfAtomBytes;       // 1 KB
// Thread layout: 8 compute warps, then the TMA producer warp and the MMA
// warp.  The unrotated path gives each thread four rows of one 16-channel
// block column (measured faster than 16 warps of two rows, which need fewer
// registers than the four-row chains want); the rotated path gives four
// threads to each row, two rows per chunk in turn: with ten warps a thread
// gets at most 168 registers (each SM sub-partition holds three of the warps),
// and a 64-value slice of the rotation block per thread spilled.
template <bool ROT>
struct QCfg {
  static constexpr int kComputeWarps = 8;
  static constexpr int kComputeThreads = 32 * kComputeWarps;
  static constexpr int kRowsPerThread = ROT ? 2 : 4;     // unrotated: rows r0 + (128 / 4) * rr; rotated: row4, row4 + 64
  static constexpr int kProducerWarp = kComputeWarps, kMmaWarp = kComputeWarps + 1;
  static constexpr int kThreads = 32 * (kComputeWarps + 2);
};
constexpr int kColRowsPerThread = QCfg<false>::kRowsPerThread;
constexpr int kColRowStride = kRows / kColRowsPerThread;   // 64

struct QParams {
  const float4* lam4;
  uint8_t* codes;
  uint8_t* scales;
  __nv_bfloat16* lowrank;
  unsigned* err;
  int M, K, Kp, R;
  int codes_pitch, scales_pitch, k_limit, ka_pad;
  int chunks_per_cta, n_chunks, ksplit;
  int stages;
};

// Byte offset, inside one stage's x tile, of the 16-byte group `c` (8 bf16,
// K elements 8c..8c+7 of the chunk) of row `row`: two 64-column boxes, each
// 128 rows x 128 bytes with the 128-byte swizzle (16B group index XOR row%8).
__device__ __forceinline__ uint32_t xoff(int row, int c) {
  return (uint32_t)((c >> 3) * kXBoxBytes + row * 128 + (((c & 7) ^ (row & 7)) << 4));
}

__device__ __forceinline__ void write_back_bf16(uint8_t* xs, int row, int c0, const uint64_t (&v)[8]) {
  uint4 o0, o1;
  o0.x = pack_bf16x2(lo2(v[0]), hi2(v[0])); o0.y = pack_bf16x2(lo2(v[1]), hi2(v[1]));
  o0.z = pack_bf16x2(lo2(v[2]), hi2(v[2])); o0.w = pack_bf16x2(lo2(v[3]), hi2(v[3]));
  o1.x = pack_bf16x2(lo2(v[4]), hi2(v[4])); o1.y = pack_bf16x2(lo2(v[5]), hi2(v[5]));
  o1.z = pack_bf16x2(lo2(v[6]), hi2(v[6])); o1.w = pack_bf16x2(lo2(v[7]), hi2(v[7]));
  *reinterpret_cast<uint4*>(xs + xoff(row, c0)) = o0;
  *reinterpret_cast<uint4*>(xs + xoff(row, c0 + 1)) = o1;
}

// Rotated path, one thread: the 32 consecutive K elements (quarter `qq` of the
// chunk) of row `row`; lanes 4r .. 4r+3 of a warp hold the four quarters of one
// row's 128-element rotation block (hadamard128_quarter).  Codes and the two
// scale bytes are returned in registers.
__device__ __forceinline__ void rotate_quarter(uint8_t* xs, const float4* lam4, const float2* srec, float y6, int row,
                                               int qq, uint32_t (&cw)[4], uint32_t& sbytes) {
  uint64_t v[16];
  float big = 0.0f;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 pw = *reinterpret_cast<const uint4*>(xs + xoff(row, 4 * qq + c));
    const uint32_t xin[4] = {pw.x, pw.y, pw.z, pw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 l = lam4[lam_slot(16 * qq + 4 * c + i)];
      v[4 * c + i] = div_rn2(bf16x2_to_f2(xin[i]), pk2(l.x, l.y), pk2(l.z, l.w));
      big = amax_nan(amax_nan(big, lo2(v[4 * c + i])), hi2(v[4 * c + i]));
    }
  }
  if (!(big < 3.0e38f)) {            // overflow / NaN (rare): redo with the divide unit
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 pw = *reinterpret_cast<const uint4*>(xs + xoff(row, 4 * qq + c));
      const uint32_t xin[4] = {pw.x, pw.y, pw.z, pw.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 l = lam4[lam_slot(16 * qq + 4 * c + i)];
        v[4 * c + i] = pk2(__fdiv_rn(__uint_as_float(xin[i] << 16), -l.x),
                           __fdiv_rn(__uint_as_float(xin[i] & 0xFFFF0000u), -l.y));
      }
    }
  }
  hadamard128_quarter(v, qq);
  sbytes = 0;
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    uint64_t blk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) blk[i] = v[8 * b + i];
    const uint32_t sb = quantize_any(blk, srec, y6, cw[2 * b], cw[2 * b + 1]);
    sbytes |= sb << (8 * b);
    write_back_bf16(xs, row, 4 * qq + 2 * b, blk);
  }
}

// Stage the codes (16 bytes) and two scale bytes of one rotated quarter.
__device__ __forceinline__ void stage_quarter(uint8_t* cst, uint8_t* sst, int row, int qq, const uint32_t (&cw)[4],
                                              uint32_t sbytes) {
  *reinterpret_cast<uint4*>(cst + row * (kChunk / 2) + qq * 16) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
  *reinterpret_cast<uint16_t*>(sst + (qq >> 1) * kSfAtomBytes + sf_atom_offset(row, 2 * (qq & 1))) =
      (uint16_t)sbytes;
}

// Row-major (caller layout) stores of one rotated quarter: 32 K elements from k.
__device__ __forceinline__ void store_quarter(const QParams& p, int m, int k, const uint32_t (&cw)[4],
                                              uint32_t sbytes) {
  uint8_t* dst = p.codes + (size_t)m * p.codes_pitch + (k >> 1);   // rows 8-byte aligned (K % 16 == 0)
#pragma unroll
  for (int j = 0; j < 2; ++j)
    if (k + 16 * j < p.k_limit) reinterpret_cast<uint2*>(dst)[j] = make_uint2(cw[2 * j], cw[2 * j + 1]);
  uint8_t* sd = p.scales + (size_t)m * p.scales_pitch + (k >> 4);
#pragma unroll
  for (int j = 0; j < 2; ++j)
    if (k + 16 * j < p.k_limit) sd[j] = (uint8_t)(sbytes >> (8 * j));
}

// Unrotated path, one thread: the 16-channel block column j = t & 7 of the
// chunk for rows t/8 + 32 i (i = 0..3), so the block's 8 smooth-factor
// operand pairs are loaded once for four rows.  NEG selects the negated
// layout (x / -smooth, written back negated; requires every smooth factor
// positive) over the sign-fixed one.
template <bool NEG>
__device__ __forceinline__ void smooth_cols(uint8_t* xs, const float4* lam4, const float2* srec, float y6, int t,
                                            uint32_t (&cw)[kColRowsPerThread][2], uint32_t (&sb)[kColRowsPerThread]) {
  constexpr int RPT = kColRowsPerThread;
  const int j = t & 7, r0 = t >> 3;
  uint64_t nb[8], yb[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 l = lam4[8 * i + j];                 // pair 8j + i (see lam_slot)
    nb[i] = pk2(l.x, l.y);
    yb[i] = pk2(l.z, l.w);
  }
  // The thread's rows are all loaded before any is written back, and the
  // common path has no per-row branch, so the rows' dependency chains
  // (divide, amax, scale, divide, convert) overlap.
  uint32_t xin[RPT][8];
#pragma unroll
  for (int rr = 0; rr < RPT; ++rr) {
    const int row = r0 + kColRowStride * rr;
    const uint4 p0 = *reinterpret_cast<const uint4*>(xs + xoff(row, 2 * j));
    const uint4 p1 = *reinterpret_cast<const uint4*>(xs + xoff(row, 2 * j + 1));
    xin[rr][0] = p0.x; xin[rr][1] = p0.y; xin[rr][2] = p0.z; xin[rr][3] = p0.w;
    xin[rr][4] = p1.x; xin[rr][5] = p1.y; xin[rr][6] = p1.z; xin[rr][7] = p1.w;
  }
  uint64_t v[RPT][8];
  float amax[RPT];
  bool finite = true;
#pragma unroll
  for (int rr = 0; rr < RPT; ++rr) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      v[rr][i] = NEG ? div_mk2(bf16x2_to_f2(xin[rr][i]), nb[i], yb[i]) : div_rn2(bf16x2_to_f2(xin[rr][i]), nb[i], yb[i]);
    amax[rr] = amax8(v[rr]);
    finite = finite && (amax[rr] < 3.0e38f);
  }
  if (finite) {
#pragma unroll
    for (int rr = 0; rr < RPT; ++rr) sb[rr] = quant_block<NEG>(v[rr], amax[rr], srec, y6, cw[rr][0], cw[rr][1]);
  } else {
    // A block holds +-inf or NaN (rare): such rows redo the divide with the
    // divide unit and quantize on the IEEE path.  (Fully unrolled, so the
    // per-row arrays stay in registers.)
#pragma unroll
    for (int rr = 0; rr < RPT; ++rr) {
      if (amax[rr] < 3.0e38f) {
        sb[rr] = quant_block<NEG>(v[rr], amax[rr], srec, y6, cw[rr][0], cw[rr][1]);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float s0 = NEG ? lo2(nb[i]) : -lo2(nb[i]), s1 = NEG ? hi2(nb[i]) : -hi2(nb[i]);
          v[rr][i] = pk2(__fdiv_rn(__uint_as_float(xin[rr][i] << 16), s0),
                         __fdiv_rn(__uint_as_float(xin[rr][i] & 0xFFFF0000u), s1));
        }
        sb[rr] = quant_block_slow(v[rr], cw[rr][0], cw[rr][1]);
        if (NEG) {
#pragma unroll
          for (int i = 0; i < 8; ++i) v[rr][i] ^= 0x8000000080000000ull;   // write back -x_hat
        }
      }
    }
  }
#pragma unroll
  for (int rr = 0; rr < RPT; ++rr) write_back_bf16(xs, r0 + kColRowStride * rr, 2 * j, v[rr]);
}

// smooth_cols for the last, ragged row tile: the thread's rows are handled one
// at a time and rows at or beyond `nvalid` (they do not exist; their shared
// memory was zero-filled by the TMA load) are skipped, with zero codes and
// scales staged for them.
template <bool NEG>
__device__ __noinline__ void smooth_cols_partial(uint8_t* xs, const float4* lam4, const float2* srec, float y6, int t,
                                                 int nvalid, uint32_t (&cw)[kColRowsPerThread][2],
                                                 uint32_t (&sb)[kColRowsPerThread]) {
  const int j = t & 7, r0 = t >> 3;
  uint64_t nb[8], yb[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 l = lam4[8 * i + j];
    nb[i] = pk2(l.x, l.y);
    yb[i] = pk2(l.z, l.w);
  }
#pragma unroll
  for (int rr = 0; rr < kColRowsPerThread; ++rr) {
    const int row = r0 + kColRowStride * rr;
    cw[rr][0] = cw[rr][1] = 0u;
    sb[rr] = 0u;
    if (row >= nvalid) continue;
    const uint4 p0 = *reinterpret_cast<const uint4*>(xs + xoff(row, 2 * j));
    const uint4 p1 = *reinterpret_cast<const uint4*>(xs + xoff(row, 2 * j + 1));
    const uint32_t xin[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
    uint64_t v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      v[i] = NEG ? div_mk2(bf16x2_to_f2(xin[i]), nb[i], yb[i]) : div_rn2(bf16x2_to_f2(xin[i]), nb[i], yb[i]);
    const float amax = amax8(v);
    if (amax < 3.0e38f) {
      sb[rr] = quant_block<NEG>(v, amax, srec, y6, cw[rr][0], cw[rr][1]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float s0 = NEG ? lo2(nb[i]) : -lo2(nb[i]), s1 = NEG ? hi2(nb[i]) : -hi2(nb[i]);
        v[i] = pk2(__fdiv_rn(__uint_as_float(xin[i] << 16), s0), __fdiv_rn(__uint_as_float(xin[i] & 0xFFFF0000u), s1));
      }
      sb[rr] = quant_block_slow(v, cw[rr][0], cw[rr][1]);
      if (NEG) {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] ^= 0x8000000080000000ull;
      }
    }
    write_back_bf16(xs, row, 2 * j, v);
  }
}

__device__ __forceinline__ void stage_cols(uint8_t* cst, uint8_t* sst, int t,
                                           const uint32_t (&cw)[kColRowsPerThread][2],
                                           const uint32_t (&sb)[kColRowsPerThread]) {
  const int j = t & 7, r0 = t >> 3;
#pragma unroll
  for (int rr = 0; rr < kColRowsPerThread; ++rr) {
    const int row = r0 + kColRowStride * rr;
    *reinterpret_cast<uint2*>(cst + row * (kChunk / 2) + j * 8) = make_uint2(cw[rr][0], cw[rr][1]);
    sst[(j >> 2) * kSfAtomBytes + sf_atom_offset(row, j & 3)] = (uint8_t)sb[rr];
  }
}

template <bool TILED>
__device__ __forceinline__ void store_cols(const QParams& p, int m0, int t, int kc,
                                           const uint32_t (&cw)[kColRowsPerThread][2],
                                           const uint32_t (&sb)[kColRowsPerThread]) {
  const int j = t & 7, r0 = t >> 3;
  const int k = kc + 16 * j;
  if (k >= p.k_limit) return;
#pragma unroll
  for (int rr = 0; rr < kColRowsPerThread; ++rr) {
    const int row = r0 + kColRowStride * rr, m = m0 + row;
    if (m >= p.M) continue;
    *reinterpret_cast<uint2*>(p.codes + (size_t)m * p.codes_pitch + (k >> 1)) = make_uint2(cw[rr][0], cw[rr][1]);
    if (TILED) {
      p.scales[((size_t)(m >> 7) * p.ka_pad + (k >> 6)) * kSfAtomBytes + sf_atom_offset(row, j & 3)] = (uint8_t)sb[rr];
    } else
      p.scales[(size_t)m * p.scales_pitch + (k >> 4)] = (uint8_t)sb[rr];
  }
}

template <bool ROT, bool NEG, bool TILED>
__global__ void __launch_bounds__(QCfg<ROT>::kThreads, 1)
    quantize_act_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_pdT,
                        const __grid_constant__ CUtensorMap tm_codes, const QParams p) {
  constexpr int kComputeThreads = QCfg<ROT>::kComputeThreads;
  constexpr int kProducerWarp = QCfg<ROT>::kProducerWarp, kMmaWarp = QCfg<ROT>::kMmaWarp;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // Round up to 1024 bytes by pointer arithmetic on the __shared__ array, so
  // every access below stays a shared-memory access (an integer round trip
  // would turn them into generic ones).
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int R = p.R;
  const int pd_stage_bytes = R * kChunk * 2;     // two 64-wide boxes of R rows x 128 B
  uint8_t* X = base;
  uint8_t* PD = X + p.stages * kXStageBytes;
  uint8_t* LAM = PD + p.stages * pd_stage_bytes;
  uint8_t* CST = LAM + p.stages * kLamStageBytes;       // code staging, one per stage
  uint8_t* SST = CST + p.stages * kCodeStageBytes;      // scale-atom staging, one per stage
  float* recv = reinterpret_cast<float*>(SST + p.stages * kSfStageBytes);   // [ksplit][128/ksplit rows][R]: partial L
  Tables* tabs = reinterpret_cast<Tables*>(reinterpret_cast<uint8_t*>(recv) + (size_t)kRows * R * 4);
  uint64_t* bars = reinterpret_cast<uint64_t*>(tabs + 1);
  uint64_t* full = bars;                    // TMA landed
  uint64_t* xready = bars + p.stages;        // x_hat written back (256 arrivals)
  uint64_t* empty = bars + 2 * p.stages;     // MMA finished reading the stage
  uint64_t* done = bars + 3 * p.stages;      // all MMAs of this CTA finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * p.stages + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * kRows;
  const int c_begin = blockIdx.y * p.chunks_per_cta;
  const int nch = min(p.chunks_per_cta, p.n_chunks - c_begin);
  const uint32_t tmem_cols = R <= 32 ? 32u : (R <= 64 ? 64u : 128u);

  if (tid == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&xready[s]), kComputeThreads);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(done), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (tid < 128) {
    const float s = e4m3_to_f32((uint32_t)tid);
    const float r = tid ? __frcp_rn(s) : 0.0f;
    tabs->srec[tid] = NEG ? make_float2(s, -r) : make_float2(-s, r);   // {-B, RN(1/B)}, B = -+s
  }
  // Everything above overlaps the previous kernel's tail (programmatic
  // dependent launch); nothing below runs before it has completed (its
  // output may be this kernel's x, and it may still read the buffers this
  // kernel writes).
  griddep_wait();
  if (warp == kProducerWarp) {
    tmem_alloc(smem_u32(tmem_slot), tmem_cols);
    tmem_relinquish();
    if (lane == 0) {
      prefetch_tmap(&tm_x);
      prefetch_tmap(&tm_pdT);
      if (TILED) prefetch_tmap(&tm_codes);
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  if (tid == 0) griddep_launch_dependents();

  int issued = 0;   // producer: loads issued
  if (warp == kProducerWarp) {
    if (lane == 0) {
      for (int i = 0; i < nch; ++i) {
        const int s = i % p.stages;
        if (i >= p.stages &&
            !wait_bounded(smem_u32(&empty[s]), ((i / p.stages) - 1) & 1, abort_flag, p.err, kErrQuantTimeout))
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
        bulk_load(smem_u32(LAM + s * kLamStageBytes), p.lam4 + kc / 2, kLamStageBytes, fb);
        issued = i + 1;
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, (uint32_t)R);
      for (int i = 0; i < nch; ++i) {
        const int s = i % p.stages;
        const uint32_t par = (i / p.stages) & 1;
        if (!wait_bounded(smem_u32(&full[s]), par, abort_flag, p.err, kErrQuantTimeout)) break;
        if (!wait_bounded(smem_u32(&xready[s]), par, abort_flag, p.err, kErrQuantTimeout)) break;
        tc_fence_after_sync();
        if (TILED) {
          // Every compute thread has staged its codes and scales (xready):
          // write the chunk's code tile and its two adjacent scale atoms.
          const int kc = (c_begin + i) * kChunk;
          tma_store_2d(&tm_codes, smem_u32(CST + s * kCodeStageBytes), kc / 2, m0);
          bulk_store(p.scales + ((size_t)blockIdx.x * p.ka_pad + kc / 64) * kSfAtomBytes,
                     smem_u32(SST + s * kSfStageBytes), kSfStageBytes);
          bulk_commit();
        }
        const uint32_t xa = smem_u32(X + s * kXStageBytes);
        const uint32_t pa = smem_u32(PD + s * pd_stage_bytes);
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk) {
          const uint64_t ad = sdesc_kmajor_sw128(xa + (kk >> 2) * kXBoxBytes + (kk & 3) * 32);
          const uint64_t bd = sdesc_kmajor_sw128(pa + (kk >> 2) * (R * 128) + (kk & 3) * 32);
          mma_bf16(tmem, ad, bd, idesc, (i | kk) != 0);
        }
        // The stage (and its staging buffers) is released only once the stores
        // have read the staging buffers.
        if (TILED) bulk_wait_read<0>();
        tc_commit(smem_u32(&empty[s]));
      }
      // Arrives when every MMA issued above has finished; waited on below
      // before the tensor memory is released.
      tc_commit(smem_u32(done));
      if (TILED) bulk_wait<0>();
    }
    __syncwarp();
  } else {
    // compute warps: the chunk's 128 rows x 128 channels
    const float y6 = __frcp_rn(6.0f);
    const int row4 = tid >> 2, qq = tid & 3;     // rotated mapping: four threads per row, rows row4 and row4 + 64
    const int nvalid = p.M - m0;                 // rows of this tile that exist (>= 1)
    for (int i = 0; i < nch; ++i) {
      const int s = i % p.stages;
      // Warp-uniform outcome: the rotated path uses full-warp shuffles.
      if (!__all_sync(0xffffffffu, wait_bounded(smem_u32(&full[s]), (i / p.stages) & 1, abort_flag, p.err,
                                                kErrQuantTimeout)))
        break;
      const int kc = (c_begin + i) * kChunk;
      uint8_t* xs = X + s * kXStageBytes;
      const float4* lam = reinterpret_cast<const float4*>(LAM + s * kLamStageBytes);
      uint32_t cwq[2][4], sq[2];                   // rotated mapping
      uint32_t cw[kColRowsPerThread][2], sb[kColRowsPerThread];   // column mapping
      if (ROT) {
        // rotate_quarter exchanges values between lanes with full-warp
        // shuffles, so only a whole warp may skip: all 8 of its rows of the
        // pass lie beyond M (rows beyond M that a warp does process are
        // zero-filled and rotate to zero).
#pragma unroll
        for (int ps = 0; ps < 2; ++ps) {
          if ((row4 & ~7) + 64 * ps < nvalid) {
            rotate_quarter(xs, lam, tabs->srec, y6, row4 + 64 * ps, qq, cwq[ps], sq[ps]);
          } else {                   // no row of this warp exists: zeros staged
#pragma unroll
            for (int c = 0; c < 4; ++c) cwq[ps][c] = 0u;
            sq[ps] = 0u;
          }
        }
      } else if (nvalid >= kRows) {
        smooth_cols<NEG>(xs, lam, tabs->srec, y6, tid, cw, sb);
      } else {
        smooth_cols_partial<NEG>(xs, lam, tabs->srec, y6, tid, nvalid, cw, sb);
      }
      if (TILED) {
        // The stores that last read this stage's staging buffers finished
        // before the stage was released for this chunk's load.
        uint8_t* cst = CST + s * kCodeStageBytes;
        uint8_t* sst = SST + s * kSfStageBytes;
        if (ROT) {
          stage_quarter(cst, sst, row4, qq, cwq[0], sq[0]);
          stage_quarter(cst, sst, row4 + 64, qq, cwq[1], sq[1]);
        } else
          stage_cols(cst, sst, tid, cw, sb);
      }
      fence_proxy_async_smem();                    // x_hat (and staging) -> async proxy
      mbar_arrive(smem_u32(&xready[s]));
      if (!TILED && ROT) {
        const int k0 = kc + 32 * qq;
#pragma unroll
        for (int ps = 0; ps < 2; ++ps) {
          const int m = m0 + row4 + 64 * ps;
          if (m < p.M && k0 < p.k_limit) store_quarter(p, m, k0, cwq[ps], sq[ps]);
        }
      } else if (!TILED) {
        store_cols<false>(p, m0, tid, kc, cw, sb);
      }
    }
    // The CTA that owns the last chunk zero-fills the scale atoms beyond Kp
    // (the GEMM's last K tile reads them and they must be finite).
    if (TILED && tid < kRows && m0 + tid < p.M && c_begin + nch == p.n_chunks) {
      for (int ka = p.Kp / 64; ka < p.ka_pad; ++ka) {
        uint8_t* atom = p.scales + ((size_t)((m0 + tid) >> 7) * p.ka_pad + ka) * kSfAtomBytes + sf_atom_offset(tid, 0);
        *reinterpret_cast<uint32_t*>(atom) = 0u;
      }
    }
  }

  // ---- rank-R down-projection: TMEM -> L (cluster reduction when K is split)
  // With K split over a cluster, rank q owns rows [q * 128/ksplit, (q+1) *
  // 128/ksplit) of the tile: every CTA pushes its partial sums of those rows
  // into slot (its rank) of the owner's receive buffer with DSMEM stores,
  // one cluster barrier publishes them, and each owner adds its slots in rank
  // order (a fixed order: the result does not depend on timing).
  const bool want_lr = p.lowrank != nullptr;
  const int rows_per = kRows / p.ksplit;
  if (want_lr && tid < kRows) {
    // warps 0-3 read TMEM lane quadrants 0-3: thread tid owns row tid.
    // Warp-uniform outcome: the TMEM loads below are warp-wide instructions.
    const bool ok = __all_sync(0xffffffffu, wait_bounded(smem_u32(done), 0, abort_flag, p.err, kErrQuantTimeout));
    tc_fence_after_sync();
    const int row = tid, m = m0 + row;
    const uint32_t owner = (uint32_t)(row / rows_per);
    const uint32_t dst0 = p.ksplit > 1 ? mapa_shared(smem_u32(recv) + (uint32_t)(((int)cluster_ctarank() * rows_per +
                                                                                  row % rows_per) * R * 4),
                                                     owner)
                                       : 0u;
    if (ok) {
      for (int j = 0; j < R; j += 16) {
        uint32_t r[16];
        tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)j, r);
        tmem_ld_wait();
        if (NEG) {                     // the negated layout accumulated -L
#pragma unroll
          for (int t = 0; t < 16; ++t) r[t] ^= 0x80000000u;
        }
        if (p.ksplit == 1) {
          if (m < p.M) {
            uint4* dst = reinterpret_cast<uint4*>(p.lowrank + (size_t)m * R + j);
            dst[0] = make_uint4(pack_bf16x2(__uint_as_float(r[0]), __uint_as_float(r[1])),
                                pack_bf16x2(__uint_as_float(r[2]), __uint_as_float(r[3])),
                                pack_bf16x2(__uint_as_float(r[4]), __uint_as_float(r[5])),
                                pack_bf16x2(__uint_as_float(r[6]), __uint_as_float(r[7])));
            dst[1] = make_uint4(pack_bf16x2(__uint_as_float(r[8]), __uint_as_float(r[9])),
                                pack_bf16x2(__uint_as_float(r[10]), __uint_as_float(r[11])),
                                pack_bf16x2(__uint_as_float(r[12]), __uint_as_float(r[13])),
                                pack_bf16x2(__uint_as_float(r[14]), __uint_as_float(r[15])));
          }
        } else {
#pragma unroll
          for (int t = 0; t < 4; ++t)
            st_shared_cluster_v4(dst0 + (uint32_t)(j + 4 * t) * 4u, __uint_as_float(r[4 * t]),
                                 __uint_as_float(r[4 * t + 1]), __uint_as_float(r[4 * t + 2]),
                                 __uint_as_float(r[4 * t + 3]));
        }
      }
    }
  }
  if (want_lr && p.ksplit > 1) {
    cluster_sync();                    // every partial has landed in its owner's buffer
    if (tid < kComputeThreads && !*abort_flag) {
      const uint32_t rank = cluster_ctarank();
      const int r4 = R / 4;
      for (int idx = tid; idx < rows_per * r4; idx += kComputeThreads) {
        const int rl = idx / r4, col = 4 * (idx % r4);
        const int m = m0 + (int)rank * rows_per + rl;
        if (m >= p.M) continue;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        for (int q = 0; q < p.ksplit; ++q) {
          const float4 v = *reinterpret_cast<const float4*>(recv + (size_t)(q * rows_per + rl) * R + col);
          a0 += v.x;
          a1 += v.y;
          a2 += v.z;
          a3 += v.w;
        }
        *reinterpret_cast<uint2*>(p.lowrank + (size_t)m * R + col) =
            make_uint2(pack_bf16x2(a0, a1), pack_bf16x2(a2, a3));
      }
    }
  }

  // ---- cleanup: after an abort, wait (bounded) for the copies this CTA started.
  if (warp == kProducerWarp && lane == 0 && *abort_flag) {
    for (int s = 0; s < p.stages && s < issued; ++s) {
      const int last = s + ((issued - 1 - s) / p.stages) * p.stages;
      wait_for(smem_u32(&full[s]), (last / p.stages) & 1, 100000000ull);
    }
  }
  if (warp == kMmaWarp && lane == 0) wait_for(smem_u32(done), 0, kWaitTimeoutNs);
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kProducerWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, tmem_cols);
  }
}

size_t smem_bytes(int R, int stages) {
  return 1024 + (size_t)stages * (kXStageBytes + R * kChunk * 2 + kLamStageBytes + kCodeStageBytes + kSfStageBytes) +
         (size_t)kRows * R * 4 +
         sizeof(Tables) + 256;
}

template <bool ROT, bool NEG, bool TILED>
cudaError_t launch_impl(const CUtensorMap& tm_x, const CUtensorMap& tm_pdT, const CUtensorMap& tm_codes,
                        const QParams& p, int row_tiles, int ksplit, cudaStream_t stream) {
  auto kern = quantize_act_kernel<ROT, NEG, TILED>;
  const size_t smem = smem_bytes(p.R, p.stages);
  cudaError_t e = ensure_smem_limit(kern, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)row_tiles, (unsigned)ksplit, 1);
  cfg.blockDim = dim3(QCfg<ROT>::kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = (unsigned)ksplit;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, tm_x, tm_pdT, tm_codes, p);
}

}  // namespace

cudaError_t launch_quantize_act(const QuantLaunch& L, cudaStream_t stream) {
  if (L.M <= 0) return cudaSuccess;
  const int n_chunks = L.Kp / kChunk;
  const int row_tiles = (L.M + kRows - 1) / kRows;
  const bool rot = L.rotate_block == 128;
  // Split K over a cluster (up to 8 CTAs) as far as one wave of one CTA per
  // SM allows.  Every CTA keeps at least one chunk.
  static int num_sms = 0;
  if (num_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (num_sms <= 0) num_sms = 148;
  }
  int ksplit = 1;
  for (int cand = 8; cand >= 2; cand >>= 1) {
    const int cpc = (n_chunks + cand - 1) / cand;
    if (cand <= n_chunks && (cand - 1) * cpc < n_chunks && row_tiles * cand <= num_sms) {
      ksplit = cand;
      break;
    }
  }
  // Tuning override: SVDQ_QUANT_KSPLIT=1|2|4|8 (applied when it keeps every CTA busy).
  static const int ks_env = [] {
    const char* e = getenv("SVDQ_QUANT_KSPLIT");
    return e ? atoi(e) : 0;
  }();
  if (ks_env == 1 || ks_env == 2 || ks_env == 4 || ks_env == 8) {
    const int cpc_env = (n_chunks + ks_env - 1) / ks_env;
    if (ks_env <= n_chunks && (ks_env - 1) * cpc_env < n_chunks) ksplit = ks_env;
  }
  const int cpc = (n_chunks + ksplit - 1) / ksplit;

  QParams p;
  p.lam4 = reinterpret_cast<const float4*>(L.lam4);
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
  // Deepest ring (up to kMaxStages) that fits in shared memory.
  p.stages = kMaxStages;
  while (p.stages > 2 && smem_bytes(L.R, p.stages) > 227 * 1024) --p.stages;

  if (rot) {
    return L.tiled_scales ? launch_impl<true, false, true>(L.tm_x, L.tm_pdT, L.tm_codes, p, row_tiles, ksplit, stream)
                          : launch_impl<true, false, false>(L.tm_x, L.tm_pdT, L.tm_codes, p, row_tiles, ksplit, stream);
  }
  if (L.lam_positive) {
    p.lam4 = reinterpret_cast<const float4*>(L.lam4_neg);
    return L.tiled_scales ? launch_impl<false, true, true>(L.tm_x, L.tm_pdT, L.tm_codes, p, row_tiles, ksplit, stream)
                          : launch_impl<false, true, false>(L.tm_x, L.tm_pdT, L.tm_codes, p, row_tiles, ksplit, stream);
  }
  return L.tiled_scales ? launch_impl<false, false, true>(L.tm_x, L.tm_pdT, L.tm_codes, p, row_tiles, ksplit, stream)
                        : launch_impl<false, false, false>(L.tm_x, L.tm_pdT, L.tm_codes, p, row_tiles, ksplit, stream);
}

}  // namespace svdq

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
//   L     = x_hat @ proj_down = x @ P,  P = diag(1/smooth) R^T proj_down   (tensor cores)
//
// The rank-R branch is reassociated: x_hat = (x / smooth) R^T, so
// x_hat proj_down = x (diag(1/smooth) R^T proj_down), and P is formed once, at
// create time, in double precision and rounded to bf16.  The tensor core then
// reads the raw x tile the TMA has just landed (it is exactly the K-major
// 128B-swizzled A operand), so the down-projection neither waits for the
// quantizer arithmetic nor needs x_hat written back to shared memory.
//
// Work decomposition.  A CTA owns 128 token rows and a contiguous slice of
// K; the K slices of one row tile form a thread-block cluster that reduces
// its partial L in distributed shared memory (fixed order, deterministic).
// Inside a CTA (640 threads, one CTA per SM):
//   warps 0-15      compute: without rotation each thread takes one 16-channel
//                   block column of two rows (t/8 and t/8 + 64); with rotation
//                   four threads share a row (32 K elements each).  Smooth
//                   (+ rotate), quantize, stage codes and scale atoms (or
//                   store them, in the caller's row-major layout).
//   warp 16 lane 0  TMA producer: x chunk (128 rows x 128 K, two 128B-swizzled
//                   boxes), P^T chunk (R x 128) and the smoothing operands into
//                   a ring of up to 4 stages; once the compute warps are done
//                   with a chunk it writes the chunk's staged codes (TMA
//                   store) and scale atoms (bulk store), and once those and the
//                   MMAs have read the stage it loads the chunk that reuses it.
//                   The warp owns the TMEM allocation.
//   warp 17 lane 0  issues tcgen05.mma (M=128, N=R, K=16, bf16 -> fp32 TMEM)
//                   for L as soon as a chunk has landed.
//   warps 16-19     once the last MMA has completed (while the compute warps
//                   finish their last chunks), read the rank-R partial sums of
//                   TMEM lane quadrants 0-3 and push them to their owner CTA.
// A stage is reloaded after both the MMAs and the stores have read it.
//
// Exact fp32 division without the divide unit.  With y = RZ(1/b) and
// y' = RN(1/b - y) carrying the sign of y, q = RN(a*y + RN(a*y')) -- one
// multiply and one fused multiply-add -- equals the correctly rounded a/b for
// every operand pair that occurs here (checked exhaustively: all bf16 x over
// every normal bf16 smoothing factor of magnitude below 2^117, where the only
// differences are quotients below 2^-19 that quantize to code +-0 and scale 0
// either way; all fp32 significands over the eight e4m3 significands for
// x_hat / scale and amax / 6), and rounding y toward zero gives zeros the
// sign of a/b.  The smoothing reciprocals come from create time, the scale
// reciprocals from a per-CTA table over the 127 e4m3 codes.  Two lanes run per
// instruction (f32x2).  Blocks whose values overflow or hold NaN take an
// IEEE-division path.
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
constexpr int kMaxStages = 4;                      // ring depth: as many as shared memory allows
constexpr int kXStageBytes = kRows * kChunk * 2;   // 32 KB: two 64-wide swizzled boxes
constexpr int kXBoxBytes = kXStageBytes / 2;       // 16 KB
constexpr int kLamStageBytes = kChunk * 8;         // float4 {yh_k, yh_k+1, yl_k, yl_k+1} per channel pair
// Forward-layout outputs of one chunk are staged in shared memory and written
// with one TMA tensor store (codes, 128 rows x 64 bytes) and one bulk copy (the
// chunk's two adjacent scale atoms).
constexpr int kCodeStageBytes = kRows * kChunk / 2;   // 8 KB
constexpr int kSfStageBytes = 2 * kSfAtomBytes;       // 1 KB
constexpr int kComputeWarps = 16;
constexpr int kComputeThreads = 32 * kComputeWarps;
// Warps 16-19 (TMEM lane quadrants 0-3) read out L; 16 and 17 first run the
// producer (with the stores) and the MMAs.  (Twenty warps: registers are allocated for
// blocks in groups of four warps, so a 21st would cost the 96-register budget.)
constexpr int kProducerWarp = kComputeWarps, kMmaWarp = kComputeWarps + 1, kLrWarp0 = kComputeWarps;
constexpr int kThreads = 32 * (kComputeWarps + 4);
// Unrotated mapping: thread t takes block column t % 8 of rows t/8 + kRowStride * i.
constexpr int kRowStride = kComputeThreads / 8;
constexpr int kRowsPerThread = kRows / kRowStride;
// Rotated mapping: four threads per row, kRotPasses rows per thread in turn.
constexpr int kRotRowsPerPass = kComputeThreads / 4;
constexpr int kRotPasses = kRows / kRotRowsPerPass;

struct QParams {
  const float4* lamq;       // smoothing reciprocal pairs, lam_slot order
  const float* lamf;        // smoothing factors (fp32), for the IEEE path
  uint8_t* codes;
  uint8_t* scales;
  __nv_bfloat16* lowrank;
  unsigned* err;
  int M, K, Kp, R;
  int codes_pitch, scales_pitch, k_limit, ka_pad;
  int chunks_per_cta, n_chunks, ksplit;
  int stages;
};

// e4m3 code -> {RZ(1/s), RN(1/s - RZ(1/s))}; code 0 -> {0, 0}.
struct QTables {
  float2 srec[128];
};

// Byte offset, inside one stage's x tile, of the 16-byte group `c` (8 bf16,
// K elements 8c..8c+7 of the chunk) of row `row`: two 64-column boxes, each
// 128 rows x 128 bytes with the 128-byte swizzle (16B group index XOR row%8).
__device__ __forceinline__ uint32_t xoff(int row, int c) {
  return (uint32_t)((c >> 3) * kXBoxBytes + row * 128 + (((c & 7) ^ (row & 7)) << 4));
}

// XOR mask on the 16-byte group index of a row of the partial-L receive
// buffer (R fp32 values, R a multiple of 16, so R/4 groups per row): 7 when
// the groups come in whole blocks of 8 (R a multiple of 32), else 3 (blocks
// of 4).  The swizzled index stays inside its aligned block, hence inside the
// row.
__device__ __forceinline__ int recv_swizzle(int R) { return (R / 4) % 8 == 0 ? 7 : 3; }

// One 16-element block of finite values -> scale byte + 16 codes (w0: 0-7, w1: 8-15).
__device__ __forceinline__ uint32_t quant_block_rr(const uint64_t (&v)[8], float amax, const float2* srec, float yh6,
                                                   float yl6, uint32_t& w0, uint32_t& w1) {
  const float q6 = fmaf(amax, yh6, amax * yl6);       // amax / 6, correctly rounded
  const uint32_t sb = cvt_e4m3(q6);
  // Branch-free: a zero scale (table entry {0, 0}) gives zero quotients and
  // the mask clears the codes.
  const float2 sr = srec[sb];
  const uint64_t yh = pk2(sr.x, sr.x), yl = pk2(sr.y, sr.y);
  uint64_t q[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) q[i] = div_rr2(v[i], yh, yl);
  const uint32_t keep = sb != 0u ? 0xFFFFFFFFu : 0u;
  w0 = keep & cvt_e2m1x8(lo2(q[0]), hi2(q[0]), lo2(q[1]), hi2(q[1]), lo2(q[2]), hi2(q[2]), lo2(q[3]), hi2(q[3]));
  w1 = keep & cvt_e2m1x8(lo2(q[4]), hi2(q[4]), lo2(q[5]), hi2(q[5]), lo2(q[6]), hi2(q[6]), lo2(q[7]), hi2(q[7]));
  return sb;
}

// The IEEE path of one unrotated block (values that overflowed or hold NaN),
// out of line so that the rare path stays out of the hot loop's instruction
// stream: it reloads the block's x from shared memory and returns the codes
// and the scale byte by value (passing the caller's register arrays would put
// them in local memory on the fast path too).
__device__ __noinline__ uint3 smooth_quant_block_ieee(const uint8_t* xs, int row, int j, const float* lamf, int k) {
  const uint4 p0 = *reinterpret_cast<const uint4*>(xs + xoff(row, 2 * j));
  const uint4 p1 = *reinterpret_cast<const uint4*>(xs + xoff(row, 2 * j + 1));
  const uint32_t xin[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
  uint64_t v[8];
  smooth_ieee(xin, lamf, k, v);
  uint3 r;
  r.z = quant_block_slow(v, r.x, r.y);
  return r;
}

// Unrotated path, one thread: 16-channel block column j = t & 7 of the chunk
// for rows t/8 and t/8 + 64; the block's smoothing operands are read once for
// both rows.  Rows at or beyond `nvalid` (zero-filled by the TMA) get zero
// codes and scales without being computed.
template <bool FULL>
__device__ __forceinline__ void smooth_rows(const uint8_t* xs, const float4* lam, const float2* srec, float yh6,
                                            float yl6, const float* lamf, int kc, int t, int nvalid,
                                            uint32_t (&cw)[kRowsPerThread][2], uint32_t (&sb)[kRowsPerThread]) {
  const int j = t & 7, r0 = t >> 3;
  bool live[kRowsPerThread];
  uint32_t xin[kRowsPerThread][8];
#pragma unroll
  for (int rr = 0; rr < kRowsPerThread; ++rr) {
    const int row = r0 + kRowStride * rr;
    live[rr] = FULL || row < nvalid;
    if (live[rr]) {
      const uint4 p0 = *reinterpret_cast<const uint4*>(xs + xoff(row, 2 * j));
      const uint4 p1 = *reinterpret_cast<const uint4*>(xs + xoff(row, 2 * j + 1));
      xin[rr][0] = p0.x; xin[rr][1] = p0.y; xin[rr][2] = p0.z; xin[rr][3] = p0.w;
      xin[rr][4] = p1.x; xin[rr][5] = p1.y; xin[rr][6] = p1.z; xin[rr][7] = p1.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) xin[rr][i] = 0u;
    }
  }
  uint64_t v[kRowsPerThread][8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 l = lam[8 * i + j];                  // pair 8j + i (see lam_slot)
    const uint64_t yh = pk2(l.x, l.y), yl = pk2(l.z, l.w);
#pragma unroll
    for (int rr = 0; rr < kRowsPerThread; ++rr) v[rr][i] = div_rr2(bf16x2_to_f2(xin[rr][i]), yh, yl);
  }
#pragma unroll
  for (int rr = 0; rr < kRowsPerThread; ++rr) {
    const float amax = amax8(v[rr]);
    if (amax < 3.0e38f) {
      sb[rr] = quant_block_rr(v[rr], amax, srec, yh6, yl6, cw[rr][0], cw[rr][1]);
    } else {
      // A block holds +-inf or NaN, or overflowed (rare): the divide unit.
      const uint3 r = smooth_quant_block_ieee(xs, r0 + kRowStride * rr, j, lamf, kc + 16 * j);
      cw[rr][0] = r.x;
      cw[rr][1] = r.y;
      sb[rr] = r.z;
    }
    if (!live[rr]) {
      cw[rr][0] = cw[rr][1] = 0u;
      sb[rr] = 0u;
    }
  }
}

__device__ __forceinline__ void stage_rows(uint8_t* cst, uint8_t* sst, int t, const uint32_t (&cw)[kRowsPerThread][2],
                                           const uint32_t (&sb)[kRowsPerThread]) {
  const int j = t & 7, r0 = t >> 3;
#pragma unroll
  for (int rr = 0; rr < kRowsPerThread; ++rr) {
    const int row = r0 + kRowStride * rr;
    *reinterpret_cast<uint2*>(cst + row * (kChunk / 2) + j * 8) = make_uint2(cw[rr][0], cw[rr][1]);
    sst[(j >> 2) * kSfAtomBytes + sf_atom_offset(row, j & 3)] = (uint8_t)sb[rr];
  }
}

// Row-major (caller layout) stores of the unrotated mapping.
__device__ __forceinline__ void store_rows(const QParams& p, int m0, int t, int kc,
                                           const uint32_t (&cw)[kRowsPerThread][2], const uint32_t (&sb)[kRowsPerThread]) {
  const int j = t & 7, r0 = t >> 3;
  const int k = kc + 16 * j;
  if (k >= p.k_limit) return;
#pragma unroll
  for (int rr = 0; rr < kRowsPerThread; ++rr) {
    const int m = m0 + r0 + kRowStride * rr;
    if (m >= p.M) continue;
    *reinterpret_cast<uint2*>(p.codes + (size_t)m * p.codes_pitch + (k >> 1)) = make_uint2(cw[rr][0], cw[rr][1]);
    p.scales[(size_t)m * p.scales_pitch + (k >> 4)] = (uint8_t)sb[rr];
  }
}

// Rotated path, one thread: the 32 consecutive K elements (quarter `qq`) of
// row `row`; lanes 4r .. 4r+3 of a warp hold the four quarters of one row's
// 128-element rotation block (hadamard128_quarter).  Codes and the two scale
// bytes are returned in registers.  Every lane of the warp must call it.
__device__ __forceinline__ void rotate_quarter(const uint8_t* xs, const float4* lam, const float2* srec, float yh6,
                                               float yl6, const float* lamf, int kc, int row, int qq,
                                               uint32_t (&cw)[4], uint32_t& sbytes) {
  uint64_t v[16];
  uint32_t xin[16];
  float big = 0.0f;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 pw = *reinterpret_cast<const uint4*>(xs + xoff(row, 4 * qq + c));
    xin[4 * c] = pw.x; xin[4 * c + 1] = pw.y; xin[4 * c + 2] = pw.z; xin[4 * c + 3] = pw.w;
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float4 l = lam[lam_slot(16 * qq + i)];
    v[i] = div_rr2(bf16x2_to_f2(xin[i]), pk2(l.x, l.y), pk2(l.z, l.w));
    big = amax_nan(amax_nan(big, lo2(v[i])), hi2(v[i]));
  }
  if (!(big < 3.0e38f)) {            // overflow / NaN (rare): the divide unit
    smooth_ieee(xin, lamf, kc + 32 * qq, v);
  }
  hadamard128_quarter(v, qq);
  sbytes = 0;
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    uint64_t blk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) blk[i] = v[8 * b + i];
    const float amax = amax8(blk);
    const uint32_t sb = amax < 3.0e38f ? quant_block_rr(blk, amax, srec, yh6, yl6, cw[2 * b], cw[2 * b + 1])
                                       : quant_block_slow(blk, cw[2 * b], cw[2 * b + 1]);
    sbytes |= sb << (8 * b);
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

template <bool ROT, bool TILED>
__global__ void __launch_bounds__(kThreads, 1)
    quantize_act_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_pdT,
                        const __grid_constant__ CUtensorMap tm_codes, const QParams p) {
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
  QTables* tabs = reinterpret_cast<QTables*>(reinterpret_cast<uint8_t*>(recv) + (size_t)kRows * R * 4);
  uint64_t* bars = reinterpret_cast<uint64_t*>(tabs + 1);
  uint64_t* full = bars;                     // TMA landed
  uint64_t* cdone = bars + p.stages;         // compute threads finished the stage (512 arrivals)
  uint64_t* empty = bars + 2 * p.stages;     // the MMAs have read the stage
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
      mbar_init(smem_u32(&cdone[s]), kComputeThreads);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(done), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (tid < 128) tabs->srec[tid] = tid ? recip_pair(e4m3_to_f32((uint32_t)tid)) : make_float2(0.0f, 0.0f);
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
      auto load = [&](int i) {
        const int s = i % p.stages;
        const int kc = (c_begin + i) * kChunk;
        const uint32_t fb = smem_u32(&full[s]);
        mbar_arrive_expect_tx(fb, kXStageBytes + pd_stage_bytes + kLamStageBytes);
        uint8_t* xs = X + s * kXStageBytes;
        uint8_t* pds = PD + s * pd_stage_bytes;
        tma_load_2d(smem_u32(xs), &tm_x, fb, kc, m0);
        tma_load_2d(smem_u32(xs + kXBoxBytes), &tm_x, fb, kc + 64, m0);
        tma_load_2d(smem_u32(pds), &tm_pdT, fb, kc, 0);
        tma_load_2d(smem_u32(pds + R * 128), &tm_pdT, fb, kc + 64, 0);
        bulk_load(smem_u32(LAM + s * kLamStageBytes), p.lamq + kc / 2, kLamStageBytes, fb);
        issued = i + 1;
      };
      // The first two chunks go out at once; the rest of the ring only once
      // chunk 0 has landed.  Every CTA asks for its first chunks at the same
      // moment, and requests for later stages queued beside them delay some
      // CTAs' first chunk (their cluster then waits for them at the end).
      const int first = min(nch, 2);
      for (int i = 0; i < first; ++i) load(i);
      if (nch > first && p.stages > first &&
          wait_bounded(smem_u32(&full[0]), 0, abort_flag, p.err, kErrQuantTimeout))
        for (int i = first; i < nch && i < p.stages; ++i) load(i);
      for (int j = 0; j < nch; ++j) {
        const int s = j % p.stages, par = (j / p.stages) & 1;
        // Chunk j's codes and scales are staged: write them.
        if (!wait_bounded(smem_u32(&cdone[s]), par, abort_flag, p.err, kErrQuantTimeout)) break;
        if (TILED) {
          const int kc = (c_begin + j) * kChunk;
          tma_store_2d(&tm_codes, smem_u32(CST + s * kCodeStageBytes), kc / 2, m0);
          bulk_store(p.scales + ((size_t)blockIdx.x * p.ka_pad + kc / 64) * kSfAtomBytes,
                     smem_u32(SST + s * kSfStageBytes), kSfStageBytes);
          bulk_commit();
        }
        if (j + p.stages < nch) {
          // The stage is reused once the stores and the MMAs have read it.
          if (TILED) bulk_wait_read<0>();
          if (!wait_bounded(smem_u32(&empty[s]), par, abort_flag, p.err, kErrQuantTimeout)) break;
          load(j + p.stages);
        }
      }
      // The staging buffers have been read; the stores themselves complete
      // at the end, after this warp's share of the rank-R read-out.
      if (TILED) bulk_wait_read<0>();
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, (uint32_t)R);
      for (int i = 0; i < nch; ++i) {
        const int s = i % p.stages;
        if (!wait_bounded(smem_u32(&full[s]), (i / p.stages) & 1, abort_flag, p.err, kErrQuantTimeout)) break;
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
  } else if (warp < kComputeWarps) {
    // compute warps: the chunk's 128 rows x 128 channels
    const float2 r6 = recip_pair(6.0f);
    const float yh6 = r6.x, yl6 = r6.y;
    const int row4 = tid >> 2, qq = tid & 3;     // rotated mapping: four threads per row (first pass)
    const int nvalid = p.M - m0;                 // rows of this tile that exist (>= 1)
    for (int i = 0; i < nch; ++i) {
      const int s = i % p.stages;
      // Warp-uniform outcome: the rotated path uses full-warp shuffles.
      if (!__all_sync(0xffffffffu, wait_bounded(smem_u32(&full[s]), (i / p.stages) & 1, abort_flag, p.err,
                                                kErrQuantTimeout)))
        break;
      const int kc = (c_begin + i) * kChunk;
      const uint8_t* xs = X + s * kXStageBytes;
      const float4* lam = reinterpret_cast<const float4*>(LAM + s * kLamStageBytes);
      uint32_t cwq[kRotPasses][4], sq[kRotPasses];                  // rotated mapping
      uint32_t cw[kRowsPerThread][2], sb[kRowsPerThread];           // column mapping
      if (ROT) {
        // Only a whole warp may skip (full-warp shuffles): all 8 of its rows
        // lie beyond M.  Rows beyond M that a warp does process are
        // zero-filled and rotate to zero.
#pragma unroll
        for (int ps = 0; ps < kRotPasses; ++ps) {
          sq[ps] = 0u;
          if ((row4 & ~7) + kRotRowsPerPass * ps < nvalid) {
            rotate_quarter(xs, lam, tabs->srec, yh6, yl6, p.lamf, kc, row4 + kRotRowsPerPass * ps, qq, cwq[ps], sq[ps]);
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) cwq[ps][c] = 0u;
          }
        }
      } else if (nvalid >= kRows) {
        smooth_rows<true>(xs, lam, tabs->srec, yh6, yl6, p.lamf, kc, tid, nvalid, cw, sb);
      } else {
        smooth_rows<false>(xs, lam, tabs->srec, yh6, yl6, p.lamf, kc, tid, nvalid, cw, sb);
      }
      if (TILED) {
        // The stores that last read this stage's staging buffers finished
        // before the stage was released for this chunk's load.
        uint8_t* cst = CST + s * kCodeStageBytes;
        uint8_t* sst = SST + s * kSfStageBytes;
        if (ROT) {
#pragma unroll
          for (int ps = 0; ps < kRotPasses; ++ps) stage_quarter(cst, sst, row4 + kRotRowsPerPass * ps, qq, cwq[ps], sq[ps]);
        } else {
          stage_rows(cst, sst, tid, cw, sb);
        }
      } else if (ROT) {
#pragma unroll
        for (int ps = 0; ps < kRotPasses; ++ps) {
          const int m = m0 + row4 + kRotRowsPerPass * ps, k0 = kc + 32 * qq;
          if (m < p.M && k0 < p.k_limit) store_quarter(p, m, k0, cwq[ps], sq[ps]);
        }
      } else {
        store_rows(p, m0, tid, kc, cw, sb);
      }
      fence_proxy_async_smem();                    // staging (and the reads of x) -> async proxy
      mbar_arrive(smem_u32(&cdone[s]));
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
  if (want_lr && warp >= kLrWarp0 && warp < kLrWarp0 + 4) {
    // Warps 16-19 read TMEM lane quadrants 0-3 (warp % 4): lane l of warp w
    // owns row 32 (w % 4) + l.  This runs as soon as the last MMA has
    // completed, while the compute warps may still be on their last chunks.
    // Warp-uniform outcome: the TMEM loads below are warp-wide instructions.
    const bool ok = __all_sync(0xffffffffu, wait_bounded(smem_u32(done), 0, abort_flag, p.err, kErrQuantTimeout));
    tc_fence_after_sync();
    const int row = 32 * (warp & 3) + lane, m = m0 + row;
    const uint32_t owner = (uint32_t)(row / rows_per);
    const uint32_t dst0 = p.ksplit > 1 ? mapa_shared(smem_u32(recv) + (uint32_t)(((int)cluster_ctarank() * rows_per +
                                                                                  row % rows_per) * R * 4),
                                                     owner)
                                       : 0u;
    // The receive buffer's 16-byte groups are XOR-swizzled by buffer row, so
    // the 32 lanes' stores of one column (32 rows) spread over every bank.
    const uint32_t gsw = (uint32_t)(((int)cluster_ctarank() * rows_per + row % rows_per) & recv_swizzle(R));
    if (ok) {
      for (int j = 0; j < R; j += 16) {
        uint32_t r[16];
        tmem_ld16(tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)j, r);
        tmem_ld_wait();
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
            st_shared_cluster_v4(dst0 + ((((uint32_t)(j + 4 * t) >> 2) ^ gsw) << 4), __uint_as_float(r[4 * t]),
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
          const int b = q * rows_per + rl;
          const float4 v = *reinterpret_cast<const float4*>(recv + (size_t)b * R + 4 * ((col >> 2) ^ (b & recv_swizzle(R))));
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
  if (TILED && warp == kProducerWarp && lane == 0) bulk_wait<0>();
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kProducerWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, tmem_cols);
  }
}

size_t smem_bytes(int R, int stages) {
  return 1024 + (size_t)stages * (kXStageBytes + R * kChunk * 2 + kLamStageBytes + kCodeStageBytes + kSfStageBytes) +
         (size_t)kRows * R * 4 + sizeof(QTables) + 256;
}

template <bool ROT, bool TILED>
cudaError_t launch_impl(const CUtensorMap& tm_x, const CUtensorMap& tm_pdT, const CUtensorMap& tm_codes,
                        const QParams& p, int row_tiles, int ksplit, cudaStream_t stream) {
  auto kern = quantize_act_kernel<ROT, TILED>;
  const size_t smem = smem_bytes(p.R, p.stages);
  cudaError_t e = ensure_smem_limit(kern, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)row_tiles, (unsigned)ksplit, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
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
  p.lamq = reinterpret_cast<const float4*>(L.lamq);
  p.lamf = L.lamf;
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

  if (rot)
    return L.tiled_scales ? launch_impl<true, true>(L.tm_x, L.tm_pdT, L.tm_codes, p, row_tiles, ksplit, stream)
                          : launch_impl<true, false>(L.tm_x, L.tm_pdT, L.tm_codes, p, row_tiles, ksplit, stream);
  return L.tiled_scales ? launch_impl<false, true>(L.tm_x, L.tm_pdT, L.tm_codes, p, row_tiles, ksplit, stream)
                        : launch_impl<false, false>(L.tm_x, L.tm_pdT, L.tm_codes, p, row_tiles, ksplit, stream);
}

}  // namespace svdq

// svdq_kernels.h -- host-side launch interface of the two hot-path kernels
// (internal to the library; the public boundary is include/svdq.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace svdq {

// Fused activation quantizer: x_hat = x / smooth (optionally block-Hadamard
// rotated), NVFP4 codes + e4m3 scales, and L = x_hat @ proj_down computed as
// x @ P with P = diag(1/smooth) R^T proj_down.
struct QuantLaunch {
  CUtensorMap tm_x;         // x bf16 (M, K): box {64, 128}, 128B swizzle
  CUtensorMap tm_pdT;       // P^T bf16 (R, Kp): box {64, R}, 128B swizzle
  CUtensorMap tm_codes;     // tiled_scales only: codes u8 (M, Kp/2): box {64, 128}, no swizzle (TMA store)
  const void* lamq;         // float4 (Kp/2): {yh_k, yh_k+1, yl_k, yl_k+1} per channel pair (yh = RZ(1/s),
                            // yl = RN(1/s - yh) with yh's sign), lam_slot order, padded with s = 1
  const float* lamf;        // (Kp) smooth factors as fp32, padded with 1 (IEEE path)
  uint8_t* codes;           // packed codes, row pitch codes_pitch bytes
  uint8_t* scales;          // row-major (pitch scales_pitch) or tensor-core tiles
  void* lowrank;            // bf16 (M, R) or nullptr
  unsigned* err;            // device error word
  int M, K, Kp, R;
  int codes_pitch;          // bytes per row of codes
  int scales_pitch;         // bytes per row of row-major scales
  int k_limit;              // codes/scales are written for k < k_limit only
  int ka_pad;               // tiled scales: 64-element K atoms per 128-row tile
  bool tiled_scales;        // scale layout: tensor-core tiles instead of row-major
  int rotate_block;         // 0 or 128
};
cudaError_t launch_quantize_act(const QuantLaunch& p, cudaStream_t stream);

// Grouped-Hadamard + MXFP4 quantizer (FP-Quant forward): x bf16 (M, K), K a
// multiple of 32 -> codes (row pitch codes_pitch) and E8M0 scales, either
// row-major (M, K/32) or in the GEMM's 512-byte atoms (two block scales per
// 64-element K step in bytes 0-1, bytes 2-3 zero), with codes and atoms zero
// up to Kp and ka_pad.  group: 0 (no rotation) or 32.
struct MxQuantLaunch {
  const void* x;
  uint8_t* codes;
  uint8_t* scales;
  int M, K, Kp;             // Kp: codes and atoms written up to Kp (tiled) or K (row-major)
  int codes_pitch, scales_pitch, ka_pad;
  int group;
  bool tiled;
};
cudaError_t launch_quantize_mx(const MxQuantLaunch& p, cudaStream_t stream);

// Back-to-back block-scaled FP4 MMAs on `ctas` CTAs (one per SM), operands in
// shared memory: the measured dense FP4 tensor rate.
cudaError_t launch_fp4_mma_loop(int iters, int ctas, unsigned* err, cudaStream_t stream);

// Standalone Walsh-Hadamard transform of rows of length 2^log2n (<= 2^15),
// in place; dtype 0 = bf16, 1 = fp16.
cudaError_t launch_hadamard_transform(void* x, int rows, int log2n, int dtype, cudaStream_t stream);

// Offline NVFP4 quantization of a dense bf16 weight (N, K) -> qweight (N, K/2),
// wscales (K/16, N), optional 128-block row rotation.
cudaError_t launch_quantize_weight(const void* w, int N, int K, int rotate_block, void* qweight, void* wscales,
                                   cudaStream_t stream);

// Block-scaled NVFP4 GEMM with the rank-R up-projection and the
// wcscales * wtscale scaling fused into the epilogue.
struct GemmLaunch {
  CUtensorMap tm_a;         // activation codes u8 (M, Kp/2): box {128, 128}, 128B swizzle
  CUtensorMap tm_b;         // weight codes u8 (N, Kp/2): box {128, 128}, 128B swizzle
  CUtensorMap tm_l;         // L bf16 (M, R): box {64, 128}, 128B swizzle
  CUtensorMap tm_pu;        // proj_up bf16 (N, R): box {64, 128}, 128B swizzle
  CUtensorMap tm_y;         // pair kernel with N % 8 == 0: y bf16 (M, N), box {64, 32}, 128B swizzle
  const uint8_t* sfa;       // activation scale tiles
  const uint8_t* sfb;       // weight scale tiles
  const float* alpha;       // (N padded to 128) wcscales * wtscale
  void* y;                  // bf16 (M, N)
  unsigned* err;
  int M, N, R;
  int k_tiles;              // Kp rounded up to 256, divided by 256
  int ka_pad;               // K atoms per 128-row scale tile (= 4 * k_tiles)
  bool mx;                  // pair kernel only: MXFP4 operands (UE8M0 scale per 32, bytes 0-1 of each atom word)
};
cudaError_t launch_gemm_nvfp4_lr(const GemmLaunch& p, cudaStream_t stream);

// The same product on 128 x 256 output tiles, with alpha folded into proj_up
// (y = alpha' * (acc + L proj_up'^T)); the GemmLaunch fields then hold:
//   tm_b   weight codes: box {128, 256}
//   tm_l   L: box {lr_row_bytes / 2, 128}, swizzle of lr_row_bytes (32 or 64)
//   tm_pu  proj_up' = bf16(proj_up / alpha) (N, R): box {lr_row_bytes / 2, 256}, same swizzle
//   sfb    weight scale tiles, an even number of 128-row tiles
//   alpha  alpha' (alpha, or 1 where alpha is 0)
// Requires R <= 32 (the L / proj_up' tile must fit beside the ring and staging).
int gemm_n256_lr_row_bytes(int R);

// Split-K variant for few rows (tiles too few to fill the GPU): 128 x 256
// tiles, each tile's K range split over an S-CTA cluster (S = 2, 4, 8);
// GemmLaunch as for the 128 x 256 kernel (tm_b box {128, 256}) but with the
// plain alpha; the rank-R term is read from `lowrank` (M, R) and `proj_up`
// (N, R) directly.  gemm_splitk_slices returns the S to use (1: do not split).
int gemm_splitk_slices(int M, int N, int R, int k_tiles, int num_sms);
cudaError_t launch_gemm_nvfp4_splitk(const GemmLaunch& p, const void* lowrank, const void* proj_up, int S,
                                     cudaStream_t stream);
cudaError_t launch_gemm_nvfp4_n256(const GemmLaunch& p, cudaStream_t stream);

// The same product for 9..32 rows (R <= 32, alpha folded), computed as
// y^T: 128 output columns (weight rows, the MMA's M) by the token rows (N =
// 32) over the whole of K per CTA (persistent), no cross-CTA sums.
// GemmLaunch fields:
//   tm_a   activation codes: box {128, 32} (rows 0..31)
//   tm_b   weight codes: box {128, 128}
//   tm_l   L: box {lr_row_bytes / 2, 32}, swizzle of lr_row_bytes
//   tm_pu  proj_up' (N, R): box {lr_row_bytes / 2, 128}, same swizzle
bool gemm_narrow_applies(int M, int R);

// 1..kGemvMaxRows token rows on CUDA cores (the product is a matrix-vector
// product bound by the weight read): weight codes (N, Kp/2), a row-major copy
// of the weight block scales (N, Kp/16), the activation codes and scale atoms
// the quantizer wrote, L (M, R), proj_up (N, R), the plain alpha (N).
constexpr int kGemvMaxRows = 4;
// The activation quantizer for 1..kGemvMaxRows rows on CUDA cores: one CTA
// per 128-channel slice writes codes (M, Kp/2), the scale atoms of row tile 0
// and the slice's fp32 partial L = x P into part[slice][M][R]; the
// matrix-vector kernel adds the partials in slice order.
struct FewQuantLaunch {
  const void* x;            // bf16 (M, K)
  const void* lamq;         // as QuantLaunch
  const float* lamf;
  const void* pdT;          // P^T bf16 (R, Kp)
  uint8_t* codes;
  uint8_t* sfa;
  float* part;
  int M, K, Kp, R, ka_pad, rotate_block;
};
cudaError_t launch_quantize_few(const FewQuantLaunch& p, cudaStream_t stream);
int quantize_few_slices(int Kp);

struct GemvLaunch {
  const uint8_t* qw;
  const uint8_t* sfr;
  const uint8_t* codes;
  const uint8_t* sfa;
  const void* lowrank;      // (M, R) bf16, used when lr_part is null
  const float* lr_part;     // [n_parts][M][R] fp32 partial L (the few-row quantizer's), or null
  int n_parts;
  const void* pu;
  const float* alpha;
  void* y;
  int M, N, K, Kp, R;
  int num_sms;
  unsigned* err;            // device error word (a bounded wait that expires sets kErrGemmTimeout)
};
size_t gemv_smem_bytes(int M, int Kp, int R);
bool gemv_applies(int M, int Kp, int R);
cudaError_t launch_gemv_nvfp4(const GemvLaunch& L, cudaStream_t stream);
cudaError_t launch_gemm_nvfp4_narrow(const GemmLaunch& p, cudaStream_t stream);

// The same product on 256 x 256 tiles, each computed by a 2-CTA cluster with
// pair (cta_group::2) MMAs; alpha folded as for the 128 x 256 kernel.  The
// GemmLaunch fields then hold:
//   tm_b   weight codes: box {128, 128} (each CTA loads its half of the tile)
//   tm_l   L: box {row_bytes / 2, 128}, swizzle of row_bytes = gemm_pair_lr_row_bytes(R)
//   tm_pu  proj_up' (N, R): box {row_bytes / 2, 128}, same swizzle
//   (for R > 32 the L / proj_up' boxes are {64, 128}, 128B swizzle, one per 64 ranks)
// gemm_pair_lr_row_bytes: bytes per row of one L / proj_up' box (32, 64 or 128).
// gemm_pair_available: R <= 128 and at least one pair fits on the device.
int gemm_pair_lr_row_bytes(int R);
bool gemm_pair_available(int R);
cudaError_t launch_gemm_nvfp4_pair(const GemmLaunch& p, cudaStream_t stream);

}  // namespace svdq

// quantize_mx.cu -- fused grouped-Hadamard rotation + MXFP4 quantization for
// sm_100a: the first half of the FP-Quant forward of "Rotate in quantization
// and its vLLM implementation", section 3.3 (the rotation and the FP4
// quantization in one kernel, so x is read once and no rotated copy is
// written), with the page's hadamard_group_size 32 and forward_method abs_max:
//
//   x_hat = fp32(butterfly_32(x) * fp32(1/sqrt(32)))     per 32-element group (optional)
//   e     = smallest integer with 2^e >= amax32(|x_hat|) / 6, clamped to [-127, 127]
//   scale = E8M0 byte e + 127 (255 for a block holding NaN, whose codes are 0)
//   code  = e2m1_rne_satfinite(x_hat * 2^-e)             (exact: a power-of-two scale)
//
// The butterfly runs stages h = 1, 2, 4, 8, 16 in that order, (a, b) -> (a + b,
// a - b) on pairs (i, i + h) with i & h == 0, each rounded to fp32, then one
// multiply by fp32(1/sqrt(32)) -- the order of the 128-block rotation.
//
// One thread per 32-element group: four 16-byte loads of x, the rotation in
// registers (16 packed fp32 pairs, f32x2 adds), 16 bytes of codes in one
// store.  Consecutive threads take consecutive groups of a row, so a warp's
// loads and code stores cover 2 KB and 512 contiguous bytes.  The exponent
// comes from amax's bits: amax = m * 2^E with m in [1, 2) gives
// ceil(log2(amax / 6)) = E - 2 + (m > 1.5), exactly.
#include <cuda_runtime.h>

#include "hadamard.cuh"
#include "kcommon.cuh"
#include "nvfp4_block.cuh"
#include "svdq_kernels.h"

namespace svdq {
namespace {

constexpr int kThreadsMx = 256;

struct MxParams {
  const uint32_t* x;      // bf16 pairs
  uint8_t* codes;
  uint8_t* scales;
  int M, K;
  int groups;             // groups per row written: Kp / 32 (tiled) or K / 32
  int codes_pitch, scales_pitch, ka_pad;
};

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// E8M0 exponent of the abs_max rule for a finite or infinite amax >= 0.
__device__ __forceinline__ int mx_exponent(float amax) {
  const uint32_t b = __float_as_uint(amax);
  const int E = (int)(b >> 23);            // sign bit is 0
  if (E == 0) return -127;                 // zero or below 2^-126: amax / 6 < 2^-128
  if (E == 255) return 127;                // infinity
  const int e = E - 127 - 2 + ((b & 0x7FFFFFu) > 0x400000u ? 1 : 0);
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

template <bool ROT, bool TILED>
__global__ void __launch_bounds__(kThreadsMx) quantize_mx_kernel(const MxParams p) {
  griddep_wait();            // x may be the previous kernel's output
  const long long total = (long long)p.M * p.groups;
  const long long stride = (long long)gridDim.x * blockDim.x;
  // Warp-uniform loop bound: every lane runs every iteration (the tiled scale
  // store pairs neighbouring lanes with a shuffle); lanes past the end idle.
  const long long warp0 = (long long)blockIdx.x * blockDim.x + (threadIdx.x & ~31);
  const int lane = threadIdx.x & 31;
  for (long long base = warp0; base < total; base += stride) {
    const long long gi = base + lane;
    const bool live = gi < total;
    const int m = live ? (int)(gi / p.groups) : 0;
    const int g = live ? (int)(gi % p.groups) : 0;
    const int k0 = 32 * g;
    uint32_t w[16];
    if (live && k0 < p.K) {
      const uint32_t* src = p.x + ((size_t)m * p.K + k0) / 2;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 q = ld_nc_v4(src + 4 * c);
        w[4 * c] = q.x; w[4 * c + 1] = q.y; w[4 * c + 2] = q.z; w[4 * c + 3] = q.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) w[i] = 0u;
    }
    uint64_t v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = bf16x2_to_f2(w[i]);
    if (ROT) {
      // h = 1: the two lanes of each word; regroup two words so each packed op
      // yields two results.
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint64_t a = pk2(lo2(v[2 * j]), lo2(v[2 * j + 1]));
        const uint64_t b = pk2(hi2(v[2 * j]), hi2(v[2 * j + 1]));
        const uint64_t sm = add2(a, b), df = sub2(a, b);
        v[2 * j] = pk2(lo2(sm), lo2(df));
        v[2 * j + 1] = pk2(hi2(sm), hi2(df));
      }
      // h = 2, 4, 8, 16: words (i, i + h/2).
#pragma unroll
      for (int st = 0; st < 4; ++st) {
        const int hp = 1 << st;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          if ((i & hp) == 0) {
            const uint64_t a = v[i], b = v[i + hp];
            v[i] = add2(a, b);
            v[i + hp] = sub2(a, b);
          }
        }
      }
      const float cn = 0.176776695296636881f;      // fp32(1/sqrt(32)) = 0x3E3504F3
      const uint64_t cn2 = pk2(cn, cn);
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = mul2(v[i], cn2);
    }
    uint64_t lo[8], hi[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      lo[i] = v[i];
      hi[i] = v[8 + i];
    }
    const float amax = amax3_nan(amax8(lo), amax8(hi), 0.0f);
    uint32_t sb, cw[4];
    if (amax != amax) {                       // NaN block: NaN scale, zero codes
      sb = 0xFFu;
#pragma unroll
      for (int i = 0; i < 4; ++i) cw[i] = 0u;
    } else {
      const int e = mx_exponent(amax);
      sb = (uint32_t)(e + 127);
      // 2^-e: a normal fp32 for e <= 126, the subnormal 2^-127 for e = 127.
      const float inv = e <= 126 ? __uint_as_float((uint32_t)(127 - e) << 23) : __uint_as_float(0x00400000u);
      const uint64_t inv2 = pk2(inv, inv);
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = mul2(v[i], inv2);
#pragma unroll
      for (int c = 0; c < 4; ++c)
        cw[c] = cvt_e2m1x8(lo2(v[4 * c]), hi2(v[4 * c]), lo2(v[4 * c + 1]), hi2(v[4 * c + 1]), lo2(v[4 * c + 2]),
                           hi2(v[4 * c + 2]), lo2(v[4 * c + 3]), hi2(v[4 * c + 3]));
    }
    if (k0 >= p.K) {                          // padding group: zero codes and scale
      sb = 0u;
#pragma unroll
      for (int i = 0; i < 4; ++i) cw[i] = 0u;
    }
    if (live)
      *reinterpret_cast<uint4*>(p.codes + (size_t)m * p.codes_pitch + 16 * g) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    if (TILED) {
      // Groups 2a and 2a + 1 of a row (neighbouring lanes: the group count per
      // row is even) share the 32-bit word of 64-element atom a: bytes 0, 1.
      const uint32_t other = __shfl_xor_sync(0xffffffffu, sb, 1);
      if (live && (g & 1) == 0) {
        const size_t atom = (size_t)(m >> 7) * p.ka_pad + (size_t)(g >> 1);
        *reinterpret_cast<uint32_t*>(p.scales + atom * kSfAtomBytes + sf_atom_offset(m & 127, 0)) = sb | (other << 8);
      }
      if (live && g == p.groups - 1) {
        // Atoms past the last code group (up to the GEMM's 256-element K tile) are zero.
        for (int a = p.groups / 2; a < p.ka_pad; ++a)
          *reinterpret_cast<uint32_t*>(p.scales + ((size_t)(m >> 7) * p.ka_pad + a) * kSfAtomBytes +
                                       sf_atom_offset(m & 127, 0)) = 0u;
      }
    } else if (live) {
      p.scales[(size_t)m * p.scales_pitch + g] = (uint8_t)sb;
    }
  }
  griddep_launch_dependents();
}

template <bool ROT, bool TILED>
cudaError_t launch_impl(const MxParams& p, int grid, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kThreadsMx, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, quantize_mx_kernel<ROT, TILED>, p);
}

}  // namespace

cudaError_t launch_quantize_mx(const MxQuantLaunch& L, cudaStream_t stream) {
  if (L.M <= 0) return cudaSuccess;
  MxParams p;
  p.x = static_cast<const uint32_t*>(L.x);
  p.codes = L.codes;
  p.scales = L.scales;
  p.M = L.M;
  p.K = L.K;
  p.groups = (L.tiled ? L.Kp : L.K) / 32;
  p.codes_pitch = L.codes_pitch;
  p.scales_pitch = L.scales_pitch;
  p.ka_pad = L.ka_pad;
  static int num_sms = 0;
  if (num_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (num_sms <= 0) num_sms = 148;
  }
  const long long total = (long long)L.M * p.groups;
  long long grid = (total + kThreadsMx - 1) / kThreadsMx;
  if (grid > 8LL * num_sms) grid = 8LL * num_sms;       // grid-stride beyond eight blocks per SM
  const bool rot = L.group == 32;
  if (rot) return L.tiled ? launch_impl<true, true>(p, (int)grid, stream) : launch_impl<true, false>(p, (int)grid, stream);
  return L.tiled ? launch_impl<false, true>(p, (int)grid, stream) : launch_impl<false, false>(p, (int)grid, stream);
}

}  // namespace svdq

// svdq_api.cu -- the C ABI of include/svdq.h: argument checking, create-time
// weight repacking into the layouts the kernels read, per-call tensor maps,
// and the two launches of the forward pass.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "svdq.h"
#include "kcommon.cuh"
#include "svdq_kernels.h"

struct svdq_linear {
  int device;
  int K, N, R, Kp, ka_pad, k_tiles, rotate_block;
  uint8_t* qw;            // (N, Kp/2) packed E2M1, rows zero-padded to Kp
  uint8_t* sfb;           // weight scale tiles: (ceil(N/128) rounded up to even) x ka_pad atoms of 512 B
  uint8_t* sfr;           // (N, Kp/16) the same scales row-major, zero beyond K/16 (few-row CUDA-core product)
  __nv_bfloat16* pdT;     // P^T (R, Kp), P = diag(1/smooth) R^T proj_down in bf16, zero-padded
  __nv_bfloat16* pu;      // proj_up (N, R)
  float4* lamq;           // (Kp/2) {yh_k, yh_k+1, yl_k, yl_k+1}: RZ(1/s) and RN(1/s - RZ(1/s)), padded with s = 1
  float* lamf;            // (Kp) smooth factors as fp32, padded with 1
  float* alpha;           // (roundup(N, 128)) wcscales * wtscale, zero-padded
  __nv_bfloat16* pu_fold; // proj_up' = bf16(proj_up / alpha) (N, R); proj_up where alpha = 0
  float* alpha_fold;      // (roundup(N, 256)) alpha, or 1 where alpha = 0
  bool n256;              // GEMM on 128 x 256 tiles with alpha folded into proj_up
  bool splitk;            // few rows: split-K GEMM over a cluster (unless SVDQ_SPLITK=0 at create)
  bool pair;              // more than 128 rows: 256 x 256 tiles on CTA pairs (unless SVDQ_GEMM_PAIR=0 at create)
  bool narrow;            // 9..32 rows: y^T on 128-column full-K tiles (unless SVDQ_GEMM_NARROW=0 at create)
  bool gemv;              // 1..4 rows: CUDA-core matrix-vector product (unless SVDQ_GEMV=0 at create)
  int lr_row_bytes;       // 128 x 256 GEMM: bytes per row of its L / proj_up' tiles
  int pair_row_bytes;     // pair GEMM: bytes per row of one L / proj_up' box
  unsigned* err;          // device error word
  // svdq_linear_forward_host: copy streams and events of its row-chunk pipeline.
  cudaStream_t s_in, s_out;
  cudaEvent_t ev_start, ev_out, ev_in[16], ev_comp[16];
  CUtensorMap tm_b, tm_pdT, tm_pu;
  CUtensorMap tm_b256, tm_pu_fold, tm_pu_fold128, tm_pu_fold_n128;
};

namespace {

thread_local std::string g_last_error;

svdq_status cuda_fail(cudaError_t e, const char* where) {
  g_last_error = std::string(where) + ": " + cudaGetErrorString(e);
  return SVDQ_ERR_CUDA;
}

#define SVDQ_CUDA(call)                                        \
  do {                                                         \
    cudaError_t e_ = (call);                                   \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call);        \
  } while (0)

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 2-D row-major tensor map (128-byte swizzle unless stated); out-of-bounds reads are zero,
// out-of-bounds parts of a stored box are skipped.
svdq_status make_tmap(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, uint64_t inner, uint64_t outer,
                      uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer,
                      CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    g_last_error = "cuTensorMapEncodeTiled unavailable";
    return SVDQ_ERR_CUDA;
  }
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    g_last_error = "cuTensorMapEncodeTiled failed with CUresult " + std::to_string((int)r);
    return SVDQ_ERR_CUDA;
  }
  return SVDQ_OK;
}

CUtensorMapSwizzle lr_swizzle(int row_bytes) {
  return row_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                         : (row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
}

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------- create-time repack kernels

// Weight scales into replicated tensor-core atoms, and row-major (N, Kp/16)
// for the few-row CUDA-core product.  Columns whose alpha is 0 get zero
// scales: their main product is multiplied by 0 anyway, and a zero there lets
// the 128 x 256 GEMM give them alpha' = 1 with y = L proj_up^T.
__global__ void repack_weight_scales(const uint8_t* __restrict__ wscales, const float* __restrict__ alpha,
                                     uint8_t* __restrict__ sfb, uint8_t* __restrict__ sfr, int K16, int N,
                                     int ka_pad, int sfr_pitch, unsigned* bad) {
  const long long total = (long long)K16 * N;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total; i += (long long)gridDim.x * blockDim.x) {
    const int kb = (int)(i / N), n = (int)(i % N);
    const uint8_t w = wscales[i];
    if ((w & 0x7F) == 0x7F) atomicOr(bad, 1u);       // e4m3 NaN
    const uint8_t b = alpha[n] == 0.0f ? 0 : w;
    sfb[((size_t)(n >> 7) * ka_pad + (kb >> 2)) * svdq::kSfAtomBytes + svdq::sf_atom_offset(n & 127, kb & 3)] = b;
    sfr[(size_t)n * sfr_pitch + kb] = b;
  }
}

// P^T (R, Kp) for the quantizer's down-projection, P = diag(1/s) R^T proj_down:
// x_hat proj_down = ((x / s) R^T) proj_down = x P, so the tensor core can read
// the raw x tile.  R = blockdiag(H_128 / sqrt(128)) (symmetric) or the
// identity.  Each entry in double precision (the rotation sum is exact in
// double for bf16 inputs up to rounding at 2^-53), then rounded to bf16.
// Padding channels are zero.  bad bit 32: an entry overflows bf16.
__global__ void prepare_proj_down(const __nv_bfloat16* __restrict__ pd, const __nv_bfloat16* __restrict__ sf,
                                  __nv_bfloat16* __restrict__ pdT, int K, int R, int Kp, int rot, unsigned* bad) {
  const long long total = (long long)R * Kp;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total; i += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(i / Kp), k = (int)(i % Kp);
    if (k >= K) {
      pdT[i] = __float2bfloat16_rn(0.0f);
      continue;
    }
    double acc;
    if (rot) {
      // (R proj_down)[k, r] = sum_t H[k % 128][t] proj_down[128 * (k / 128) + t, r] / sqrt(128),
      // H[a][b] = (-1)^popcount(a & b) (Sylvester).
      const int kb = k & ~127, kr = k & 127;
      acc = 0.0;
      for (int t = 0; t < 128; ++t) {
        const double v = (double)__bfloat162float(pd[(size_t)(kb + t) * R + r]);
        acc += (__popc(kr & t) & 1) ? -v : v;
      }
      acc /= sqrt(128.0);
    } else {
      acc = (double)__bfloat162float(pd[(size_t)k * R + r]);
    }
    const double val = acc / (double)__bfloat162float(sf[k]);
    const __nv_bfloat16 q = __float2bfloat16_rn(__double2float_rn(val));
    if (!isfinite(__bfloat162float(q))) atomicOr(bad, 32u);
    pdT[i] = q;
  }
}

// Per channel pair (k, k+1): the reciprocal pairs {yh_k, yh_k+1, yl_k, yl_k+1}
// with yh = RZ(1/s) and yl = RN(1/s - yh) (sign of yh), from which the
// quantizer forms the correctly rounded x / s as RN(x*yh + RN(x*yl)); stored in
// its bank-conflict-free order (svdq::lam_slot).  Also the factors themselves
// as fp32 (the IEEE path).  Padding channels get s = 1.  bad bit 2: a zero or
// non-finite factor; bit 16: a factor outside the magnitudes [2^-126, 2^117)
// for which that division is exact.
__global__ void prepare_smooth(const __nv_bfloat16* __restrict__ sf, float4* __restrict__ lamq, float* __restrict__ lamf,
                               int K, int Kp, unsigned* bad) {
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < Kp / 2; j += gridDim.x * blockDim.x) {
    float l[2] = {1.0f, 1.0f};
    if (2 * j < K) {                 // K is even, so channel 2j+1 exists too
      l[0] = __bfloat162float(sf[2 * j]);
      l[1] = __bfloat162float(sf[2 * j + 1]);
    }
    float yh[2], yl[2];
    for (int c = 0; c < 2; ++c) {
      const float a = fabsf(l[c]);
      if (!(isfinite(l[c]) && l[c] != 0.0f)) {
        atomicOr(bad, 2u);
        l[c] = 1.0f;
      } else if (a < 0x1p-126f || a >= 0x1p117f) {
        atomicOr(bad, 16u);
      }
      const double inv = 1.0 / (double)l[c];
      yh[c] = __double2float_rz(inv);
      yl[c] = copysignf(fabsf(__double2float_rn(inv - (double)yh[c])), yh[c]);
    }
    lamq[svdq::lam_slot(j)] = make_float4(yh[0], yh[1], yl[0], yl[1]);
    lamf[2 * j] = l[0];
    lamf[2 * j + 1] = l[1];
  }
}

__global__ void prepare_alpha(const __nv_bfloat16* __restrict__ wc, const __nv_bfloat16* __restrict__ wt, float* alpha,
                              int N, int Npad) {
  const float t = wt ? __bfloat162float(wt[0]) : 1.0f;
  for (int n = blockIdx.x * blockDim.x + threadIdx.x; n < Npad; n += gridDim.x * blockDim.x) {
    // bf16 x bf16 is exact in fp32.
    alpha[n] = n < N ? (wc ? __bfloat162float(wc[n]) : 1.0f) * t : 0.0f;
  }
}

// alpha' and proj_up' = bf16(proj_up / alpha) for the 128 x 256 GEMM, which
// computes y = alpha' (acc + L proj_up'^T).  bad bit 8: a column that cannot be
// folded without leaving the range where the quotient keeps bf16 precision
// (|alpha| outside [2^-24, 2^24], non-finite values, or a quotient that
// overflows or falls below the normal range); the layer then uses the
// 128 x 128 GEMM, which applies alpha in its epilogue.
__global__ void fold_alpha(const __nv_bfloat16* __restrict__ pu, const float* __restrict__ alpha,
                           __nv_bfloat16* __restrict__ pu_fold, float* __restrict__ alpha_fold, int N, int R,
                           int Npad256, unsigned* bad) {
  const long long total = (long long)Npad256 * R;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total; i += (long long)gridDim.x * blockDim.x) {
    const int n = (int)(i / R);
    const float a = n < N ? alpha[n] : 0.0f;
    if (i % R == 0) alpha_fold[n] = a == 0.0f ? 1.0f : a;
    if (n >= N) continue;
    if (a == 0.0f) {
      pu_fold[i] = pu[i];
      continue;
    }
    const float fa = fabsf(a);
    if (!(fa >= 0x1p-24f && fa <= 0x1p24f)) {         // also catches NaN
      atomicOr(bad, 8u);
      pu_fold[i] = pu[i];
      continue;
    }
    const float v = __bfloat162float(pu[i]);
    const __nv_bfloat16 q = __float2bfloat16_rn(__fdiv_rn(v, a));
    const float qf = __bfloat162float(q);
    if (!isfinite(qf) || (v != 0.0f && fabsf(qf) < 0x1p-126f)) atomicOr(bad, 8u);
    pu_fold[i] = q;
  }
}

int grid_for(long long n) {
  long long g = (n + 255) / 256;
  return (int)(g < 1 ? 1 : (g > 4096 ? 4096 : g));
}

svdq_status check_device(const svdq_linear* h) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev != h->device) {
    g_last_error = "current device differs from the device the handle was created on";
    return SVDQ_ERR_INVALID_ARG;
  }
  return SVDQ_OK;
}

void free_handle(svdq_linear* h) {
  if (!h) return;
  cudaFree(h->qw);
  cudaFree(h->sfb);
  cudaFree(h->sfr);
  cudaFree(h->pdT);
  cudaFree(h->pu);
  cudaFree(h->lamq);
  cudaFree(h->lamf);
  cudaFree(h->alpha);
  cudaFree(h->pu_fold);
  cudaFree(h->alpha_fold);
  cudaFree(h->err);
  if (h->s_in) cudaStreamDestroy(h->s_in);
  if (h->s_out) cudaStreamDestroy(h->s_out);
  if (h->ev_start) cudaEventDestroy(h->ev_start);
  if (h->ev_out) cudaEventDestroy(h->ev_out);
  for (int i = 0; i < 16; ++i) {
    if (h->ev_in[i]) cudaEventDestroy(h->ev_in[i]);
    if (h->ev_comp[i]) cudaEventDestroy(h->ev_comp[i]);
  }
  delete h;
}

struct WsLayout {
  size_t codes, sfa, lr, part, total;
};

// Workspace of one call: codes, scale atoms, L (bf16), and for at most
// kGemvMaxRows rows the few-row quantizer's fp32 partial L per 128-channel slice.
WsLayout ws_layout(const svdq_linear* h, int M) {
  WsLayout w;
  w.codes = 0;
  w.sfa = align256((size_t)M * (h->Kp / 2));
  w.lr = align256(w.sfa + (size_t)((M + 127) / 128) * h->ka_pad * svdq::kSfAtomBytes);
  w.part = align256(w.lr + (size_t)M * h->R * 2);
  const size_t part_bytes =
      M <= svdq::kGemvMaxRows ? (size_t)svdq::quantize_few_slices(h->Kp) * M * h->R * sizeof(float) : 0;
  w.total = align256(w.part + part_bytes);
  return w;
}

}  // namespace

extern "C" {

int svdq_version(void) { return (1 << 16) | 0; }

const char* svdq_status_string(svdq_status s) {
  switch (s) {
    case SVDQ_OK: return "ok";
    case SVDQ_ERR_INVALID_ARG: return "invalid argument";
    case SVDQ_ERR_SHAPE: return "unsupported shape";
    case SVDQ_ERR_UNSUPPORTED: return "unsupported device or configuration";
    case SVDQ_ERR_CUDA: return "CUDA error";
    case SVDQ_ERR_WORKSPACE: return "workspace missing or too small";
    case SVDQ_ERR_DEVICE: return "device-side error (bounded wait expired)";
  }
  return "unknown status";
}

const char* svdq_last_error(void) { return g_last_error.c_str(); }

svdq_status svdq_linear_create(svdq_linear** out, const svdq_linear_desc* d, void* stream_) {
  if (!out) return SVDQ_ERR_INVALID_ARG;
  *out = nullptr;
  if (!d || !d->qweight || !d->wscales || !d->proj_down || !d->proj_up || !d->smooth_factor)
    return SVDQ_ERR_INVALID_ARG;
  if (d->act_unsigned != 0) return SVDQ_ERR_UNSUPPORTED;
  if (d->K <= 0 || d->N <= 0 || d->K % 16 != 0) return SVDQ_ERR_SHAPE;
  if (d->R < 16 || d->R > 128 || d->R % 16 != 0) return SVDQ_ERR_SHAPE;
  if (d->rotate_block != 0 && d->rotate_block != 128) return SVDQ_ERR_SHAPE;
  if (d->rotate_block && d->K % d->rotate_block != 0) return SVDQ_ERR_SHAPE;
  if ((long long)d->K * d->N > (1LL << 40)) return SVDQ_ERR_SHAPE;

  int dev = 0, major = 0, minor = 0;
  SVDQ_CUDA(cudaGetDevice(&dev));
  SVDQ_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
  SVDQ_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
  if (major != 10 || minor != 0) {
    g_last_error = "requires an sm_100 (B200) device";
    return SVDQ_ERR_UNSUPPORTED;
  }
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);

  svdq_linear* h = new svdq_linear();
  std::memset(h, 0, sizeof(*h));
  h->device = dev;
  h->K = d->K;
  h->N = d->N;
  h->R = d->R;
  h->rotate_block = d->rotate_block;
  h->Kp = (d->K + 127) / 128 * 128;
  h->k_tiles = (h->Kp + 255) / 256;
  h->ka_pad = 4 * h->k_tiles;
  const int n_tiles = (d->N + 127) / 128;
  const int Npad = n_tiles * 128;
  const int n_tiles_even = (n_tiles + 1) & ~1;   // the 128 x 256 GEMM reads scale tiles in pairs
  const int Npad256 = n_tiles_even * 128;

  auto fail = [&](svdq_status s) {
    free_handle(h);
    return s;
  };
  cudaError_t e;
#define CREATE_CUDA(call)                         \
  do {                                            \
    e = (call);                                   \
    if (e != cudaSuccess) {                       \
      cuda_fail(e, #call);                        \
      return fail(SVDQ_ERR_CUDA);                 \
    }                                             \
  } while (0)

  CREATE_CUDA(cudaMalloc(&h->qw, (size_t)d->N * (h->Kp / 2)));
  CREATE_CUDA(cudaMalloc(&h->sfb, (size_t)n_tiles_even * h->ka_pad * svdq::kSfAtomBytes));
  // Row-major scales, padded to an even number of rows (the matrix-vector
  // product copies scale rows in pairs).
  CREATE_CUDA(cudaMalloc(&h->sfr, (size_t)((d->N + 1) & ~1) * (h->Kp / 16)));
  CREATE_CUDA(cudaMalloc(&h->pdT, (size_t)d->R * h->Kp * 2));
  CREATE_CUDA(cudaMalloc(&h->pu, (size_t)d->N * d->R * 2));
  CREATE_CUDA(cudaMalloc(&h->lamq, (size_t)(h->Kp / 2) * sizeof(float4)));
  CREATE_CUDA(cudaMalloc(&h->lamf, (size_t)h->Kp * sizeof(float)));
  CREATE_CUDA(cudaMalloc(&h->alpha, (size_t)Npad * sizeof(float)));
  CREATE_CUDA(cudaMalloc(&h->pu_fold, (size_t)d->N * d->R * 2));
  CREATE_CUDA(cudaMalloc(&h->alpha_fold, (size_t)Npad256 * sizeof(float)));
  CREATE_CUDA(cudaMalloc(&h->err, 2 * sizeof(unsigned)));   // [0] device error word, [1] create-time checks
  CREATE_CUDA(cudaStreamCreateWithFlags(&h->s_in, cudaStreamNonBlocking));
  CREATE_CUDA(cudaStreamCreateWithFlags(&h->s_out, cudaStreamNonBlocking));
  CREATE_CUDA(cudaEventCreateWithFlags(&h->ev_start, cudaEventDisableTiming));
  CREATE_CUDA(cudaEventCreateWithFlags(&h->ev_out, cudaEventDisableTiming));
  for (int i = 0; i < 16; ++i) {
    CREATE_CUDA(cudaEventCreateWithFlags(&h->ev_in[i], cudaEventDisableTiming));
    CREATE_CUDA(cudaEventCreateWithFlags(&h->ev_comp[i], cudaEventDisableTiming));
  }
  CREATE_CUDA(cudaMemsetAsync(h->err, 0, 2 * sizeof(unsigned), stream));

  CREATE_CUDA(cudaMemset2DAsync(h->qw, h->Kp / 2, 0, h->Kp / 2, d->N, stream));
  CREATE_CUDA(cudaMemcpy2DAsync(h->qw, h->Kp / 2, d->qweight, d->K / 2, d->K / 2, d->N, cudaMemcpyDeviceToDevice,
                                stream));
  CREATE_CUDA(cudaMemsetAsync(h->sfb, 0, (size_t)n_tiles_even * h->ka_pad * svdq::kSfAtomBytes, stream));
  CREATE_CUDA(cudaMemsetAsync(h->sfr, 0, (size_t)((d->N + 1) & ~1) * (h->Kp / 16), stream));
  prepare_alpha<<<grid_for(Npad), 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(d->wcscales),
                                                     static_cast<const __nv_bfloat16*>(d->wtscale), h->alpha, d->N,
                                                     Npad);
  CREATE_CUDA(cudaGetLastError());
  repack_weight_scales<<<grid_for((long long)(d->K / 16) * d->N), 256, 0, stream>>>(
      static_cast<const uint8_t*>(d->wscales), h->alpha, h->sfb, h->sfr, d->K / 16, d->N, h->ka_pad, h->Kp / 16,
      h->err + 1);
  CREATE_CUDA(cudaGetLastError());
  prepare_smooth<<<grid_for(h->Kp / 2), 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(d->smooth_factor), h->lamq,
                                                           h->lamf, d->K, h->Kp, h->err + 1);
  CREATE_CUDA(cudaGetLastError());
  prepare_proj_down<<<grid_for((long long)d->R * h->Kp), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(d->proj_down), static_cast<const __nv_bfloat16*>(d->smooth_factor), h->pdT,
      d->K, d->R, h->Kp, d->rotate_block == 128, h->err + 1);
  CREATE_CUDA(cudaGetLastError());
  CREATE_CUDA(cudaMemcpyAsync(h->pu, d->proj_up, (size_t)d->N * d->R * 2, cudaMemcpyDeviceToDevice, stream));
  fold_alpha<<<grid_for((long long)Npad256 * d->R), 256, 0, stream>>>(h->pu, h->alpha, h->pu_fold, h->alpha_fold,
                                                                      d->N, d->R, Npad256, h->err + 1);
  CREATE_CUDA(cudaGetLastError());
  unsigned bad = 0;
  CREATE_CUDA(cudaMemcpyAsync(&bad, h->err + 1, sizeof(unsigned), cudaMemcpyDeviceToHost, stream));
  CREATE_CUDA(cudaStreamSynchronize(stream));
  if (bad & (1u | 2u | 16u | 32u)) {
    g_last_error = (bad & 1u)    ? "wscales holds an e4m3 NaN"
                   : (bad & 2u)  ? "smooth_factor holds a zero or non-finite value"
                   : (bad & 16u) ? "smooth_factor holds a magnitude outside [2^-126, 2^117)"
                                 : "proj_down / smooth_factor overflows bf16";
    return fail(SVDQ_ERR_INVALID_ARG);
  }
  {
    // 128 x 256 tiles unless alpha cannot be folded, R > 32, or the
    // environment asks for the 128 x 128 GEMM (SVDQ_GEMM_TILE_N=128).
    const char* env = std::getenv("SVDQ_GEMM_TILE_N");
    const bool force128 = env && std::strcmp(env, "128") == 0;
    const bool foldable = !(bad & 8u) && !force128;
    h->n256 = foldable && d->R <= 32;
    const char* sk = std::getenv("SVDQ_SPLITK");
    h->splitk = !(sk && sk[0] == '0');
    // 256 x 256 pair tiles (2-CTA clusters) unless SVDQ_GEMM_PAIR=0.
    const char* pr = std::getenv("SVDQ_GEMM_PAIR");
    h->pair = foldable && !(pr && pr[0] == '0');
    const char* nw = std::getenv("SVDQ_GEMM_NARROW");
    h->narrow = h->n256 && !(nw && nw[0] == '0');
    const char* gv = std::getenv("SVDQ_GEMV");
    h->gemv = !(gv && gv[0] == '0');
    h->pair_row_bytes = svdq::gemm_pair_lr_row_bytes(d->R);
    h->lr_row_bytes = svdq::gemm_n256_lr_row_bytes(d->R);
  }
#undef CREATE_CUDA

  svdq_status s;
  if ((s = make_tmap(&h->tm_b, h->qw, CU_TENSOR_MAP_DATA_TYPE_UINT8, h->Kp / 2, d->N, h->Kp / 2, 128, 128)) != SVDQ_OK)
    return fail(s);
  if ((s = make_tmap(&h->tm_pdT, h->pdT, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, h->Kp, d->R, (uint64_t)h->Kp * 2, 64,
                     d->R)) != SVDQ_OK)
    return fail(s);
  if ((s = make_tmap(&h->tm_pu, h->pu, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d->R, d->N, (uint64_t)d->R * 2, 64, 128)) !=
      SVDQ_OK)
    return fail(s);
  // 256-row weight boxes: the 128 x 256 kernel and the split-K kernel for few rows.
  if ((s = make_tmap(&h->tm_b256, h->qw, CU_TENSOR_MAP_DATA_TYPE_UINT8, h->Kp / 2, d->N, h->Kp / 2, 128, 256)) !=
      SVDQ_OK)
    return fail(s);
  if (h->n256) {
    if ((s = make_tmap(&h->tm_pu_fold, h->pu_fold, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d->R, d->N, (uint64_t)d->R * 2,
                       h->lr_row_bytes / 2, 256, lr_swizzle(h->lr_row_bytes))) != SVDQ_OK)
      return fail(s);
  }
  if (h->narrow) {
    // 128-row proj_up' boxes: the few-row kernel's rank-R A operand.
    if ((s = make_tmap(&h->tm_pu_fold_n128, h->pu_fold, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d->R, d->N,
                       (uint64_t)d->R * 2, h->lr_row_bytes / 2, 128, lr_swizzle(h->lr_row_bytes))) != SVDQ_OK)
      return fail(s);
  }
  if (h->pair) {
    if ((s = make_tmap(&h->tm_pu_fold128, h->pu_fold, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d->R, d->N,
                       (uint64_t)d->R * 2, h->pair_row_bytes / 2, 128, lr_swizzle(h->pair_row_bytes))) != SVDQ_OK)
      return fail(s);
  }
  *out = h;
  return SVDQ_OK;
}

void svdq_linear_destroy(svdq_linear* h) {
  if (!h) return;
  cudaDeviceSynchronize();
  free_handle(h);
}

size_t svdq_workspace_bytes(const svdq_linear* h, int M) {
  if (!h || M <= 0) return 0;
  return ws_layout(h, M).total;
}

svdq_status svdq_quantize_act(const svdq_linear* h, const void* x, int M, void* codes, void* scales, void* lowrank,
                              void* stream_) {
  if (!h || M < 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!x || !codes || !scales) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || (lowrank && !aligned16(lowrank))) return SVDQ_ERR_INVALID_ARG;
  svdq_status s = check_device(h);
  if (s != SVDQ_OK) return s;
  svdq::QuantLaunch q;
  if ((s = make_tmap(&q.tm_x, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, h->K, M, (uint64_t)h->K * 2, 64, 128)) != SVDQ_OK)
    return s;
  q.tm_pdT = h->tm_pdT;
  q.tm_codes = q.tm_x;   // unused: the public layout is written directly
  q.lamq = h->lamq;
  q.lamf = h->lamf;
  q.codes = static_cast<uint8_t*>(codes);
  q.scales = static_cast<uint8_t*>(scales);
  q.lowrank = lowrank;
  q.err = h->err;
  q.M = M;
  q.K = h->K;
  q.Kp = h->Kp;
  q.R = h->R;
  q.codes_pitch = h->K / 2;
  q.scales_pitch = h->K / 16;
  q.k_limit = h->K;
  q.ka_pad = h->ka_pad;
  q.tiled_scales = false;
  q.rotate_block = h->rotate_block;
  cudaError_t e = svdq::launch_quantize_act(q, static_cast<cudaStream_t>(stream_));
  if (e != cudaSuccess) return cuda_fail(e, "quantize_act launch");
  return SVDQ_OK;
}

namespace {

svdq_status check_forward_args(const svdq_linear* h, int M, void* workspace) {
  if (!h || M < 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return SVDQ_ERR_WORKSPACE;
  return check_device(h);
}

enum class GemmKind { gemv, narrow, splitk, pair, n256, lr };
GemmKind pick_gemm(const svdq_linear* h, int M, int* S);

svdq_status forward_quantize(const svdq_linear* h, const void* x, int M, void* workspace, cudaStream_t stream) {
  const WsLayout w = ws_layout(h, M);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int S = 1;
  if (pick_gemm(h, M, &S) == GemmKind::gemv) {
    // 1..4 rows on the CUDA-core matrix-vector product: its own quantizer
    // (codes, scale atoms, per-slice partial L), no tensor-core tiles.
    svdq::FewQuantLaunch f;
    f.x = x;
    f.lamq = h->lamq;
    f.lamf = h->lamf;
    f.pdT = h->pdT;
    f.codes = ws + w.codes;
    f.sfa = ws + w.sfa;
    f.part = reinterpret_cast<float*>(ws + w.part);
    f.M = M;
    f.K = h->K;
    f.Kp = h->Kp;
    f.R = h->R;
    f.ka_pad = h->ka_pad;
    f.rotate_block = h->rotate_block;
    cudaError_t e = svdq::launch_quantize_few(f, stream);
    if (e != cudaSuccess) return cuda_fail(e, "quantize_few launch");
    return SVDQ_OK;
  }
  svdq::QuantLaunch q;
  svdq_status s;
  if ((s = make_tmap(&q.tm_x, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, h->K, M, (uint64_t)h->K * 2, 64, 128)) != SVDQ_OK)
    return s;
  q.tm_pdT = h->tm_pdT;
  if ((s = make_tmap(&q.tm_codes, ws + w.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, h->Kp / 2, M, h->Kp / 2, 64, 128,
                     CU_TENSOR_MAP_SWIZZLE_NONE)) != SVDQ_OK)
    return s;
  q.lamq = h->lamq;
  q.lamf = h->lamf;
  q.codes = ws + w.codes;
  q.scales = ws + w.sfa;
  q.lowrank = ws + w.lr;
  q.err = h->err;
  q.M = M;
  q.K = h->K;
  q.Kp = h->Kp;
  q.R = h->R;
  q.codes_pitch = h->Kp / 2;
  q.scales_pitch = 0;
  q.k_limit = h->Kp;
  q.ka_pad = h->ka_pad;
  q.tiled_scales = true;
  q.rotate_block = h->rotate_block;
  cudaError_t e = svdq::launch_quantize_act(q, stream);
  if (e != cudaSuccess) return cuda_fail(e, "quantize_act launch");
  return SVDQ_OK;
}

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

// Which GEMM kernel serves M rows on this handle (S: split-K cluster size).

GemmKind pick_gemm(const svdq_linear* h, int M, int* S) {
  *S = 1;
  // 1..4 rows: the weight read bounds the product; CUDA cores, no tiles.
  if (h->gemv && svdq::gemv_applies(M, h->Kp, h->R)) return GemmKind::gemv;
  // 9..32 rows (R <= 32): y^T on 128-column tiles over the whole of K.
  if (h->narrow && svdq::gemm_narrow_applies(M, h->R)) return GemmKind::narrow;
  // Few rows: split K over a cluster so the weight read is spread over the GPU.
  if (h->splitk) *S = svdq::gemm_splitk_slices(M, h->N, h->R, h->k_tiles, num_sms());
  if (*S > 1) return GemmKind::splitk;
  if (h->pair && M > 128 && svdq::gemm_pair_available(h->R)) return GemmKind::pair;
  if (h->n256) return GemmKind::n256;
  return GemmKind::lr;
}

svdq_status forward_gemm(const svdq_linear* h, int M, void* y, void* workspace, cudaStream_t stream) {
  const WsLayout w = ws_layout(h, M);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int S = 1;
  const GemmKind kind = pick_gemm(h, M, &S);
  if (kind == GemmKind::gemv) {
    svdq::GemvLaunch v;
    v.qw = h->qw;
    v.sfr = h->sfr;
    v.codes = ws + w.codes;
    v.sfa = ws + w.sfa;
    v.lowrank = ws + w.lr;
    v.lr_part = reinterpret_cast<const float*>(ws + w.part);
    v.n_parts = svdq::quantize_few_slices(h->Kp);
    v.pu = h->pu;
    v.alpha = h->alpha;
    v.y = y;
    v.M = M;
    v.N = h->N;
    v.K = h->K;
    v.Kp = h->Kp;
    v.R = h->R;
    v.num_sms = num_sms();
    v.err = h->err;
    cudaError_t e = svdq::launch_gemv_nvfp4(v, stream);
    if (e != cudaSuccess) return cuda_fail(e, "gemv launch");
    return SVDQ_OK;
  }
  svdq::GemmLaunch g;
  std::memset(&g, 0, sizeof(g));
  svdq_status s;
  if ((s = make_tmap(&g.tm_a, ws + w.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, h->Kp / 2, M, h->Kp / 2, 128, 128)) !=
      SVDQ_OK)
    return s;
  g.sfa = ws + w.sfa;
  g.sfb = h->sfb;
  g.y = y;
  g.err = h->err;
  g.M = M;
  g.N = h->N;
  g.R = h->R;
  g.k_tiles = h->k_tiles;
  g.ka_pad = h->ka_pad;
  if (kind == GemmKind::narrow) {
    if ((s = make_tmap(&g.tm_a, ws + w.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, h->Kp / 2, M, h->Kp / 2, 128, 32)) !=
        SVDQ_OK)
      return s;
    g.tm_b = h->tm_b;
    if ((s = make_tmap(&g.tm_l, ws + w.lr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, h->R, M, (uint64_t)h->R * 2,
                       h->lr_row_bytes / 2, 32, lr_swizzle(h->lr_row_bytes))) != SVDQ_OK)
      return s;
    g.tm_pu = h->tm_pu_fold_n128;
    g.alpha = h->alpha_fold;
    cudaError_t e = svdq::launch_gemm_nvfp4_narrow(g, stream);
    if (e != cudaSuccess) return cuda_fail(e, "gemm launch");
    return SVDQ_OK;
  }
  if (kind == GemmKind::splitk) {
    g.tm_b = h->tm_b256;
    g.alpha = h->alpha;
    cudaError_t e = svdq::launch_gemm_nvfp4_splitk(g, ws + w.lr, h->pu, S, stream);
    if (e != cudaSuccess) return cuda_fail(e, "gemm launch");
    return SVDQ_OK;
  }
  if (kind == GemmKind::pair) {
    g.tm_b = h->tm_b;
    if ((s = make_tmap(&g.tm_l, ws + w.lr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, h->R, M, (uint64_t)h->R * 2,
                       h->pair_row_bytes / 2, 128, lr_swizzle(h->pair_row_bytes))) != SVDQ_OK)
      return s;
    g.tm_pu = h->tm_pu_fold128;
    g.alpha = h->alpha_fold;
    if (h->N % 8 == 0 &&
        (s = make_tmap(&g.tm_y, y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, h->N, M, (uint64_t)h->N * 2, 64, 32)) != SVDQ_OK)
      return s;
    cudaError_t e = svdq::launch_gemm_nvfp4_pair(g, stream);
    if (e != cudaSuccess) return cuda_fail(e, "gemm launch");
    return SVDQ_OK;
  }
  if (kind == GemmKind::n256) {
    g.tm_b = h->tm_b256;
    if ((s = make_tmap(&g.tm_l, ws + w.lr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, h->R, M, (uint64_t)h->R * 2,
                       h->lr_row_bytes / 2, 128, lr_swizzle(h->lr_row_bytes))) != SVDQ_OK)
      return s;
    g.tm_pu = h->tm_pu_fold;
    g.alpha = h->alpha_fold;
    cudaError_t e = svdq::launch_gemm_nvfp4_n256(g, stream);
    if (e != cudaSuccess) return cuda_fail(e, "gemm launch");
    return SVDQ_OK;
  }
  g.tm_b = h->tm_b;
  if ((s = make_tmap(&g.tm_l, ws + w.lr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, h->R, M, (uint64_t)h->R * 2, 64, 128)) !=
      SVDQ_OK)
    return s;
  g.tm_pu = h->tm_pu;
  g.alpha = h->alpha;
  cudaError_t e = svdq::launch_gemm_nvfp4_lr(g, stream);
  if (e != cudaSuccess) return cuda_fail(e, "gemm launch");
  return SVDQ_OK;
}

}  // namespace

svdq_status svdq_hadamard_transform(void* x, int rows, int n, int dtype, void* stream) {
  if (rows < 0 || (dtype != 0 && dtype != 1)) return SVDQ_ERR_INVALID_ARG;
  if (n < 1 || n > 32768 || (n & (n - 1)) != 0) return SVDQ_ERR_SHAPE;
  if (rows == 0) return SVDQ_OK;
  if (!x || (reinterpret_cast<uintptr_t>(x) & 1u) != 0) return SVDQ_ERR_INVALID_ARG;
  int log2n = 0;
  while ((1 << log2n) < n) ++log2n;
  cudaError_t e = svdq::launch_hadamard_transform(x, rows, log2n, dtype, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "hadamard_transform launch");
  return SVDQ_OK;
}

svdq_status svdq_quantize_weight(const void* w, int N, int K, int rotate_block, void* qweight, void* wscales,
                                 void* stream) {
  if (!w || !qweight || !wscales || !aligned16(w) || (reinterpret_cast<uintptr_t>(qweight) & 7u) != 0)
    return SVDQ_ERR_INVALID_ARG;
  if (N < 1 || K < 16 || K % 16 != 0) return SVDQ_ERR_SHAPE;
  if (rotate_block != 0 && (rotate_block != 128 || K % 128 != 0)) return SVDQ_ERR_SHAPE;
  cudaError_t e = svdq::launch_quantize_weight(w, N, K, rotate_block, qweight, wscales,
                                               static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "quantize_weight launch");
  return SVDQ_OK;
}

svdq_status svdq_linear_forward_quantize(const svdq_linear* h, const void* x, int M, void* workspace, void* stream) {
  svdq_status s = check_forward_args(h, M, workspace);
  if (s != SVDQ_OK || M == 0) return s;
  if (!x || !aligned16(x)) return SVDQ_ERR_INVALID_ARG;
  return forward_quantize(h, x, M, workspace, static_cast<cudaStream_t>(stream));
}

const char* svdq_linear_gemm_kernel(const svdq_linear* h, int M) {
  if (!h || M <= 0) return "";
  int S = 1;
  switch (pick_gemm(h, M, &S)) {
    case GemmKind::gemv: return "gemv_nvfp4_kernel (CUDA cores, 1-4 rows)";
    case GemmKind::narrow: return "gemm_nvfp4_narrow_kernel (y^T on 128 x 32 tiles over the whole of K)";
    case GemmKind::splitk:
      return S == 8 ? "gemm_nvfp4_splitk_kernel (128 x 256 tiles, K split over 8-CTA clusters)"
                    : (S == 4 ? "gemm_nvfp4_splitk_kernel (128 x 256 tiles, K split over 4-CTA clusters)"
                              : "gemm_nvfp4_splitk_kernel (128 x 256 tiles, K split over 2-CTA clusters)");
    case GemmKind::pair:
      return "gemm_nvfp4_pair_kernel (256 x 256 tiles on 2-CTA clusters, tcgen05 cta_group::2, alpha folded)";
    case GemmKind::n256: return "gemm_nvfp4_n256_kernel (128 x 256 tiles, alpha folded)";
    case GemmKind::lr: return "gemm_nvfp4_lr_kernel (128 x 128 tiles)";
  }
  return "";
}

svdq_status svdq_linear_forward_gemm(const svdq_linear* h, int M, void* y, void* workspace, void* stream) {
  svdq_status s = check_forward_args(h, M, workspace);
  if (s != SVDQ_OK || M == 0) return s;
  if (!y || !aligned16(y)) return SVDQ_ERR_INVALID_ARG;
  return forward_gemm(h, M, y, workspace, static_cast<cudaStream_t>(stream));
}

svdq_status svdq_linear_forward(const svdq_linear* h, const void* x, int M, void* y, void* workspace, void* stream_) {
  if (!h || M < 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!x || !y || !aligned16(x) || !aligned16(y)) return SVDQ_ERR_INVALID_ARG;
  svdq_status s = check_forward_args(h, M, workspace);
  if (s != SVDQ_OK) return s;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if ((s = forward_quantize(h, x, M, workspace, stream)) != SVDQ_OK) return s;
  return forward_gemm(h, M, y, workspace, stream);
}

svdq_status svdq_linear_forward_host(const svdq_linear* h, const void* x_host, int M, void* y_host, void* x_dev,
                                     void* y_dev, void* workspace, void* stream_) {
  if (!h || M < 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!x_host || !y_host) return SVDQ_ERR_INVALID_ARG;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  // Row chunks: one for M < 1024, else six with boundaries at 1/16, 4/16,
  // 8/16, 12/16 and 15/16 of M (rounded down to 128 rows).  The host-to-device
  // copy of chunk i+1 (stream s_in), the layer on chunk i (the caller's
  // stream) and the device-to-host copy of chunk i-1 (stream s_out) run at the
  // same time; the short first and last chunks keep the start (copy in, no
  // copy out yet) and the end (copy out only) short.  Few large copies: PCIe
  // moves less in both directions together when the copies are many and
  // small.  Chunks run in order on the caller's stream and share the
  // workspace.  Every chunk but the last is a multiple of 128 rows and the
  // last has at least M/16 rows, so no chunk takes the few-row GEMM when M
  // does not.
  int bounds[7];
  int n_chunks = 0;
  bounds[0] = 0;
  if (M < 1024) {
    bounds[++n_chunks] = M;
  } else {
    static const int cum16[5] = {1, 4, 8, 12, 15};
    for (int i = 0; i < 5; ++i) {
      const int b = (int)(((int64_t)M * cum16[i] / 16) & ~127);
      if (b > bounds[n_chunks]) bounds[++n_chunks] = b;
    }
    bounds[++n_chunks] = M;
  }
  const size_t xrow = (size_t)h->K * 2, yrow = (size_t)h->N * 2;
  SVDQ_CUDA(cudaEventRecord(h->ev_start, stream));          // work queued before this call
  SVDQ_CUDA(cudaStreamWaitEvent(h->s_in, h->ev_start, 0));
  SVDQ_CUDA(cudaStreamWaitEvent(h->s_out, h->ev_start, 0));
  for (int c = 0; c < n_chunks; ++c) {
    const int r0 = bounds[c], rc = bounds[c + 1] - bounds[c];
    SVDQ_CUDA(cudaMemcpyAsync(static_cast<uint8_t*>(x_dev) + r0 * xrow, static_cast<const uint8_t*>(x_host) + r0 * xrow,
                              (size_t)rc * xrow, cudaMemcpyHostToDevice, h->s_in));
    SVDQ_CUDA(cudaEventRecord(h->ev_in[c], h->s_in));
  }
  svdq_status s = SVDQ_OK;
  for (int c = 0; c < n_chunks; ++c) {
    const int r0 = bounds[c], rc = bounds[c + 1] - bounds[c];
    SVDQ_CUDA(cudaStreamWaitEvent(stream, h->ev_in[c], 0));
    s = svdq_linear_forward(h, static_cast<const uint8_t*>(x_dev) + r0 * xrow, rc,
                            static_cast<uint8_t*>(y_dev) + r0 * yrow, workspace, stream_);
    if (s != SVDQ_OK) break;
    SVDQ_CUDA(cudaEventRecord(h->ev_comp[c], stream));
    SVDQ_CUDA(cudaStreamWaitEvent(h->s_out, h->ev_comp[c], 0));
    SVDQ_CUDA(cudaMemcpyAsync(static_cast<uint8_t*>(y_host) + r0 * yrow, static_cast<const uint8_t*>(y_dev) + r0 * yrow,
                              (size_t)rc * yrow, cudaMemcpyDeviceToHost, h->s_out));
  }
  // The caller's stream ends after every copy (also on an error above).
  SVDQ_CUDA(cudaEventRecord(h->ev_out, h->s_out));
  SVDQ_CUDA(cudaStreamWaitEvent(stream, h->ev_out, 0));
  SVDQ_CUDA(cudaEventRecord(h->ev_start, h->s_in));
  SVDQ_CUDA(cudaStreamWaitEvent(stream, h->ev_start, 0));
  SVDQ_CUDA(cudaStreamSynchronize(stream));
  return s;
}

svdq_status svdq_device_status(const svdq_linear* h, int* flags) {
  if (!h) return SVDQ_ERR_INVALID_ARG;
  svdq_status s = check_device(h);
  if (s != SVDQ_OK) return s;
  SVDQ_CUDA(cudaDeviceSynchronize());
  unsigned v = 0;
  SVDQ_CUDA(cudaMemcpy(&v, h->err, sizeof(unsigned), cudaMemcpyDeviceToHost));
  if (v) SVDQ_CUDA(cudaMemset(h->err, 0, sizeof(unsigned)));
  if (flags) *flags = (int)v;
  return v ? SVDQ_ERR_DEVICE : SVDQ_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- MXFP4 with a grouped Hadamard (FP-Quant)

struct svdq_mxfp4 {
  int device;
  int K, N, Kp, k_tiles, ka_pad, group;
  float alpha;
  uint8_t* qw;            // (N, Kp/2) packed E2M1, rows zero-padded to Kp
  uint8_t* sfb;           // weight E8M0 scale atoms ((ceil(N/128) rounded up to even) x ka_pad x 512 B)
  float* alpha_v;         // (roundup(N, 256)) alpha for every column
  unsigned* err;          // [0] device error word, [1] create-time checks
  CUtensorMap tm_b;       // qw: box {128, 128}, 128B swizzle
};

namespace {

// (N, K/32) row-major E8M0 bytes -> the GEMM's atoms: the two block scales of
// each 64-element K step in bytes 0, 1 of the row's 32-bit atom word (bytes 2,
// 3 and every atom past K stay zero from the memset).  bad bit 1: a NaN byte.
__global__ void repack_mx_scales(const uint8_t* __restrict__ ws, uint8_t* __restrict__ sfb, int N, int G, int ka_pad,
                                 unsigned* bad) {
  const long long total = (long long)N * G;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total; i += (long long)gridDim.x * blockDim.x) {
    const int n = (int)(i / G), g = (int)(i % G);
    const uint8_t b = ws[i];
    if (b == 0xFF) atomicOr(bad, 1u);
    sfb[((size_t)(n >> 7) * ka_pad + (g >> 1)) * svdq::kSfAtomBytes + svdq::sf_atom_offset(n & 127, g & 1)] = b;
  }
}

__global__ void fill_f32(float* p, float v, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) p[i] = v;
}

void free_mx(svdq_mxfp4* h) {
  if (!h) return;
  cudaFree(h->qw);
  cudaFree(h->sfb);
  cudaFree(h->alpha_v);
  cudaFree(h->err);
  delete h;
}

struct MxWs {
  size_t codes, sfa, total;
};
MxWs mx_ws_layout(const svdq_mxfp4* h, int M) {
  MxWs w;
  w.codes = 0;
  w.sfa = align256((size_t)M * (h->Kp / 2));
  w.total = align256(w.sfa + (size_t)((M + 127) / 128) * h->ka_pad * svdq::kSfAtomBytes);
  return w;
}

}  // namespace

extern "C" {

svdq_status svdq_mxfp4_create(svdq_mxfp4** out, const svdq_mxfp4_desc* d, void* stream_) {
  if (!out) return SVDQ_ERR_INVALID_ARG;
  *out = nullptr;
  if (!d || !d->qweight || !d->wscales) return SVDQ_ERR_INVALID_ARG;
  if (d->K <= 0 || d->N <= 0 || d->K % 32 != 0) return SVDQ_ERR_SHAPE;
  if (d->hadamard_group != 0 && d->hadamard_group != 32) return SVDQ_ERR_SHAPE;
  if ((long long)d->K * d->N > (1LL << 40)) return SVDQ_ERR_SHAPE;
  if (!std::isfinite(d->alpha)) return SVDQ_ERR_INVALID_ARG;
  int dev = 0, major = 0, minor = 0;
  SVDQ_CUDA(cudaGetDevice(&dev));
  SVDQ_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
  SVDQ_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
  if (major != 10 || minor != 0) {
    g_last_error = "requires an sm_100 (B200) device";
    return SVDQ_ERR_UNSUPPORTED;
  }
  if (!svdq::gemm_pair_available(0)) {
    g_last_error = "the pair GEMM does not fit on this device";
    return SVDQ_ERR_UNSUPPORTED;
  }
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  svdq_mxfp4* h = new svdq_mxfp4();
  std::memset(h, 0, sizeof(*h));
  h->device = dev;
  h->K = d->K;
  h->N = d->N;
  h->group = d->hadamard_group;
  h->alpha = d->alpha;
  h->Kp = (d->K + 127) / 128 * 128;
  h->k_tiles = (h->Kp + 255) / 256;
  h->ka_pad = 4 * h->k_tiles;
  const int n_tiles_even = (((d->N + 127) / 128) + 1) & ~1;
  const int Npad256 = (d->N + 255) / 256 * 256;
  cudaError_t e;
  auto fail = [&](svdq_status st) {
    free_mx(h);
    return st;
  };
#define MX_CUDA(call)                             \
  do {                                            \
    e = (call);                                   \
    if (e != cudaSuccess) {                       \
      cuda_fail(e, #call);                        \
      return fail(SVDQ_ERR_CUDA);                 \
    }                                             \
  } while (0)
  MX_CUDA(cudaMalloc(&h->qw, (size_t)d->N * (h->Kp / 2)));
  MX_CUDA(cudaMalloc(&h->sfb, (size_t)n_tiles_even * h->ka_pad * svdq::kSfAtomBytes));
  MX_CUDA(cudaMalloc(&h->alpha_v, (size_t)Npad256 * sizeof(float)));
  MX_CUDA(cudaMalloc(&h->err, 2 * sizeof(unsigned)));
  MX_CUDA(cudaMemsetAsync(h->err, 0, 2 * sizeof(unsigned), stream));
  MX_CUDA(cudaMemset2DAsync(h->qw, h->Kp / 2, 0, h->Kp / 2, d->N, stream));
  MX_CUDA(cudaMemcpy2DAsync(h->qw, h->Kp / 2, d->qweight, d->K / 2, d->K / 2, d->N, cudaMemcpyDeviceToDevice, stream));
  MX_CUDA(cudaMemsetAsync(h->sfb, 0, (size_t)n_tiles_even * h->ka_pad * svdq::kSfAtomBytes, stream));
  repack_mx_scales<<<grid_for((long long)d->N * (d->K / 32)), 256, 0, stream>>>(
      static_cast<const uint8_t*>(d->wscales), h->sfb, d->N, d->K / 32, h->ka_pad, h->err + 1);
  MX_CUDA(cudaGetLastError());
  fill_f32<<<grid_for(Npad256), 256, 0, stream>>>(h->alpha_v, d->alpha, Npad256);
  MX_CUDA(cudaGetLastError());
  unsigned bad = 0;
  MX_CUDA(cudaMemcpyAsync(&bad, h->err + 1, sizeof(unsigned), cudaMemcpyDeviceToHost, stream));
  MX_CUDA(cudaStreamSynchronize(stream));
#undef MX_CUDA
  if (bad & 1u) {
    g_last_error = "wscales holds an E8M0 NaN (0xFF)";
    return fail(SVDQ_ERR_INVALID_ARG);
  }
  svdq_status s;
  if ((s = make_tmap(&h->tm_b, h->qw, CU_TENSOR_MAP_DATA_TYPE_UINT8, h->Kp / 2, d->N, h->Kp / 2, 128, 128)) != SVDQ_OK)
    return fail(s);
  *out = h;
  return SVDQ_OK;
}

void svdq_mxfp4_destroy(svdq_mxfp4* h) {
  if (!h) return;
  cudaDeviceSynchronize();
  free_mx(h);
}

size_t svdq_mxfp4_workspace_bytes(const svdq_mxfp4* h, int M) {
  if (!h || M <= 0) return 0;
  return mx_ws_layout(h, M).total;
}

svdq_status svdq_mxfp4_quantize(const void* x, int M, int K, int hadamard_group, void* codes, void* scales,
                                void* stream) {
  if (M < 0 || K <= 0 || K % 32 != 0) return M < 0 ? SVDQ_ERR_INVALID_ARG : SVDQ_ERR_SHAPE;
  if (hadamard_group != 0 && hadamard_group != 32) return SVDQ_ERR_SHAPE;
  if (M == 0) return SVDQ_OK;
  if (!x || !codes || !scales || !aligned16(x) || !aligned16(codes)) return SVDQ_ERR_INVALID_ARG;
  svdq::MxQuantLaunch q;
  q.x = x;
  q.codes = static_cast<uint8_t*>(codes);
  q.scales = static_cast<uint8_t*>(scales);
  q.M = M;
  q.K = K;
  q.Kp = K;
  q.codes_pitch = K / 2;
  q.scales_pitch = K / 32;
  q.ka_pad = 0;
  q.group = hadamard_group;
  q.tiled = false;
  cudaError_t e = svdq::launch_quantize_mx(q, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "quantize_mx launch");
  return SVDQ_OK;
}

svdq_status svdq_mxfp4_forward(const svdq_mxfp4* h, const void* x, int M, void* y, void* workspace, void* stream_) {
  if (!h || M < 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!x || !y || !aligned16(x) || !aligned16(y)) return SVDQ_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return SVDQ_ERR_WORKSPACE;
  int dev = -1;
  SVDQ_CUDA(cudaGetDevice(&dev));
  if (dev != h->device) {
    g_last_error = "current device differs from the device the handle was created on";
    return SVDQ_ERR_INVALID_ARG;
  }
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  const MxWs w = mx_ws_layout(h, M);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  svdq::MxQuantLaunch q;
  q.x = x;
  q.codes = ws + w.codes;
  q.scales = ws + w.sfa;
  q.M = M;
  q.K = h->K;
  q.Kp = h->Kp;
  q.codes_pitch = h->Kp / 2;
  q.scales_pitch = 0;
  q.ka_pad = h->ka_pad;
  q.group = h->group;
  q.tiled = true;
  cudaError_t e = svdq::launch_quantize_mx(q, stream);
  if (e != cudaSuccess) return cuda_fail(e, "quantize_mx launch");
  svdq::GemmLaunch g;
  std::memset(&g, 0, sizeof(g));
  svdq_status s;
  if ((s = make_tmap(&g.tm_a, ws + w.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, h->Kp / 2, M, h->Kp / 2, 128, 128)) !=
      SVDQ_OK)
    return s;
  g.tm_b = h->tm_b;
  g.tm_l = h->tm_b;      // no rank-R branch: the L and proj_up maps are never read
  g.tm_pu = h->tm_b;
  if (h->N % 8 == 0 &&
      (s = make_tmap(&g.tm_y, y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, h->N, M, (uint64_t)h->N * 2, 64, 32)) != SVDQ_OK)
    return s;
  else if (h->N % 8 != 0)
    g.tm_y = h->tm_b;
  g.sfa = ws + w.sfa;
  g.sfb = h->sfb;
  g.alpha = h->alpha_v;
  g.y = y;
  g.err = h->err;
  g.M = M;
  g.N = h->N;
  g.R = 0;
  g.k_tiles = h->k_tiles;
  g.ka_pad = h->ka_pad;
  g.mx = true;
  e = svdq::launch_gemm_nvfp4_pair(g, stream);
  if (e != cudaSuccess) return cuda_fail(e, "mxfp4 gemm launch");
  return SVDQ_OK;
}

svdq_status svdq_mxfp4_device_status(const svdq_mxfp4* h, int* flags) {
  if (!h) return SVDQ_ERR_INVALID_ARG;
  unsigned v = 0;
  SVDQ_CUDA(cudaDeviceSynchronize());
  SVDQ_CUDA(cudaMemcpy(&v, h->err, sizeof(unsigned), cudaMemcpyDeviceToHost));
  SVDQ_CUDA(cudaMemset(h->err, 0, sizeof(unsigned)));
  if (flags) *flags = (int)v;
  return v ? SVDQ_ERR_DEVICE : SVDQ_OK;
}

}  // extern "C"

/*
 * svdq.h -- C ABI of the B200 (sm_100a) SVDQuant W4A4 linear layer.
 *
 * The layer ("SVDQuant W4A4", vLLM-Omni svdquant.md, sections "Overview",
 * "Checkpoint contract", "Runtime support") computes, for bf16 activations
 * x[M, K] and an offline-quantized checkpoint,
 *
 *   x_hat = x / smooth_factor                      (per input channel k)
 *   x_hat = x_hat R^T   (optional: R = blockdiag(H_128 / sqrt(128)), the
 *                        normalized Sylvester Hadamard of "Rotate in
 *                        quantization and its vLLM implementation",
 *                        sections 2.1-2.2; the weight was rotated offline)
 *   y     = wcscales (.) wtscale * (Q(x_hat) Q(W)^T) + (x_hat proj_down) proj_up^T
 *
 * in bf16, where Q() is NVFP4: E2M1 codes {0,.5,1,1.5,2,3,4,6} x sign, two
 * per byte (element 2j in the low nibble of byte j), one e4m3 (OCP FP8
 * E4M3FN) scale per 16 consecutive K elements.  Activations are quantized
 * online with scale = e4m3_rne_satfinite(fp32(amax/6)) and
 * code = e2m1_rne_satfinite(fp32(x_hat / scale)) (a block whose scale rounds
 * to zero gets scale 0 and codes 0).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers (cudaMalloc'd or otherwise
 *    device-accessible) unless a name ends in _host.  All tensors are dense,
 *    row-major, with no padding between rows.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Work is enqueued asynchronously on it; nothing synchronizes unless stated.
 *  - Functions return an svdq_status and never throw across the ABI.  On
 *    SVDQ_ERR_CUDA the CUDA error text is available from svdq_last_error().
 *  - The device must be compute capability 10.0 (B200, sm_100a); create()
 *    checks the current device.
 *  - A handle is used on the device that was current at create().  The calls
 *    that take a caller workspace (svdq_quantize_act, svdq_linear_forward and
 *    its two stages) may run on one handle from several host threads at once:
 *    they only read the handle, so it is safe as long as their workspaces and
 *    outputs differ.  Two calls are exceptions: svdq_linear_forward_host uses
 *    copy streams and events owned by the handle, so its calls on one handle
 *    must not overlap; svdq_linear_forward_noalloc shares one scratch array
 *    per device among all its calls, so calls whose kernels can overlap on
 *    the GPU race (see each declaration).
 */
#ifndef SVDQ_H_
#define SVDQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SVDQ_API __attribute__((visibility("default")))
#else
#define SVDQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,   /* null pointer, bad flag, misaligned pointer, M < 0 */
  SVDQ_ERR_SHAPE = 2,         /* K % 16 != 0, R not in {16..128} step 16, rotate block does not divide K */
  SVDQ_ERR_UNSUPPORTED = 3,   /* not an sm_100 device, act_unsigned != 0, precision other than nvfp4 */
  SVDQ_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed (see svdq_last_error) */
  SVDQ_ERR_WORKSPACE = 5,     /* workspace NULL or too small for M */
  SVDQ_ERR_DEVICE = 6         /* a kernel reported a device-side error (bounded wait expired) */
} svdq_status;

/* Opaque handle: library-owned, repacked copies of one layer's weights. */
typedef struct svdq_linear svdq_linear;

/*
 * Layer description at create time.  Shapes and dtypes are the checkpoint
 * contract of "SVDQuant W4A4" (section "Checkpoint contract"); K must be a
 * multiple of 16 (same section).  The library reads rank / precision /
 * act_unsigned of the checkpoint's quantization_config through K, N, R and
 * act_unsigned; precision is always "nvfp4".
 */
typedef struct {
  int K;                      /* input features, multiple of 16 (and of rotate_block if set) */
  int N;                      /* output features, >= 1 */
  int R;                      /* low-rank correction rank: 16, 32, ..., 128 */
  int rotate_block;           /* 0 = no online rotation, 128 = block Hadamard of size 128 */
  int act_unsigned;           /* must be 0 (signed activations) */
  const void* qweight;        /* (N, K/2)  int8: packed E2M1, element 2j in low nibble of byte j */
  const void* wscales;        /* (K/16, N) float8_e4m3fn: wscales[k/16, n] scales W[n, k] */
  const void* proj_down;      /* (K, R)    bf16 */
  const void* proj_up;        /* (N, R)    bf16 */
  const void* smooth_factor;  /* (K,)      bf16, finite, magnitude in [2^-126, 2^117) */
  const void* wcscales;       /* (N,)      bf16, or NULL meaning all ones */
  const void* wtscale;        /* (1,)      bf16, or NULL meaning 1.0 */
} svdq_linear_desc;

/*
 * svdq_linear_create -- validate the description and copy + repack the
 * weights into library-owned device memory (FP4 weight rows padded for TMA,
 * scale factors re-tiled into the tensor-core scale layout, the down-projection
 * folded with the smoothing and the rotation as P = diag(1/smooth_factor) R^T
 * proj_down in bf16 (so that x_hat proj_down = x P), reciprocal pairs of the
 * smoothing factors for the exact division, alpha[n] = wcscales[n] * wtscale
 * precomputed in fp32).  Returns SVDQ_ERR_INVALID_ARG for a wscales NaN, a
 * smoothing factor that is zero, non-finite or of magnitude outside
 * [2^-126, 2^117) (the range in which the quantizer's division is exact), or a
 * P entry that overflows bf16; svdq_last_error() names which.
 * The source tensors may be freed once this returns: it synchronizes `stream`.
 * On success *out receives the handle; on failure *out is set to NULL.
 * Shape errors are reported here (the pages' fail-at-load convention,
 * "SVDQuant W4A4" section "Runtime support").
 */
SVDQ_API svdq_status svdq_linear_create(svdq_linear** out, const svdq_linear_desc* desc, void* stream);

/* Free the handle and its device memory.  NULL is a no-op.  Synchronizes the device. */
SVDQ_API void svdq_linear_destroy(svdq_linear* h);

/* Bytes of device workspace svdq_linear_forward needs for M rows (0 for M == 0). */
SVDQ_API size_t svdq_workspace_bytes(const svdq_linear* h, int M);

/*
 * svdq_quantize_act -- the fused activation quantizer alone (smooth, optional
 * rotation, NVFP4 quantize, and the rank-R down-projection from the same read
 * of x).
 *   x       (M, K)    bf16, input
 *   codes   (M, K/2)  uint8 output: packed E2M1 codes, low nibble = even k
 *   scales  (M, K/16) uint8 output: e4m3 scale bytes, row-major
 *   lowrank (M, R)    bf16 output L = x_hat proj_down, computed as x P with
 *                     P = bf16(diag(1/smooth_factor) R^T proj_down) (fp32
 *                     accumulate on the tensor cores), or NULL to skip it
 * M == 0 is a no-op.  Pointers must be 16-byte aligned.
 */
SVDQ_API svdq_status svdq_quantize_act(const svdq_linear* h, const void* x, int M,
                              void* codes, void* scales, void* lowrank, void* stream);

/*
 * svdq_linear_forward -- y (M, N) bf16 = the full layer on x (M, K) bf16.
 * Two kernels on `stream`: the fused quantizer (writes codes, tensor-core
 * scale tiles and L into `workspace`) and the block-scaled FP4 GEMM whose
 * epilogue adds the rank-R up-projection and applies wcscales * wtscale.
 * workspace: >= svdq_workspace_bytes(h, M) bytes of device memory, 256-byte
 * aligned, owned by the caller, not shared by concurrent calls.
 */
SVDQ_API svdq_status svdq_linear_forward(const svdq_linear* h, const void* x, int M, void* y,
                                void* workspace, void* stream);

/*
 * The two stages of svdq_linear_forward, callable separately (same
 * arguments; together they are exactly svdq_linear_forward):
 *   svdq_linear_forward_quantize -- the fused quantizer: x -> codes, scale
 *       tiles and L inside `workspace`.
 *   svdq_linear_forward_gemm     -- the GEMM + rank-R epilogue: workspace -> y.
 * The workspace written by the first call must be passed unchanged, with the
 * same M, to the second; stream order between them is the caller's.
 */
SVDQ_API svdq_status svdq_linear_forward_quantize(const svdq_linear* h, const void* x, int M,
                                                  void* workspace, void* stream);
SVDQ_API svdq_status svdq_linear_forward_gemm(const svdq_linear* h, int M, void* y,
                                              void* workspace, void* stream);

/*
 * svdq_linear_gemm_kernel -- static text naming the kernel that
 * svdq_linear_forward_gemm launches for M rows on this handle ("" for a NULL
 * handle or M <= 0).  The choice depends on M, N, K, R, the create-time
 * switches and the device's SM count, and is made by the same function the
 * launch uses.  Host-only; launches nothing.
 */
SVDQ_API const char* svdq_linear_gemm_kernel(const svdq_linear* h, int M);

/*
 * svdq_linear_forward_host -- end-to-end call on HOST buffers: copies x_host
 * (M, K bf16) to x_dev, runs svdq_linear_forward into y_dev, copies y_dev to
 * y_host (M, N bf16) and synchronizes `stream` before returning.  The copies
 * and the layer are pipelined over row chunks (two copy streams owned by the
 * handle), so calls on one handle must not overlap.  Host buffers should be
 * pinned (required for the overlap).  x_dev / y_dev / workspace are
 * caller-owned device buffers as in svdq_linear_forward.
 */
SVDQ_API svdq_status svdq_linear_forward_host(const svdq_linear* h, const void* x_host, int M, void* y_host,
                                     void* x_dev, void* y_dev, void* workspace, void* stream);

/*
 * svdq_linear_forward_noalloc -- svdq_linear_forward without a caller
 * workspace and without allocating anything.  The pages have no counterpart:
 * this is a library convenience for callers that cannot allocate device memory
 * when they run the layer -- hosts that pass a kernel its inputs and outputs
 * but no scratch buffer (plugin interfaces, runtimes that own all device
 * memory), and latency-bound loops that must not call cudaMalloc, which can
 * block on and synchronize with work already queued on the device.
 *   x (M, K) bf16 in, y (M, N) bf16 out: caller-owned device memory, 16-byte
 *   aligned, exactly as for svdq_linear_forward.
 * The intermediates go to a library-owned device array of
 * SVDQ_NOALLOC_SCRATCH_BYTES (32 MiB) per device, held from the first call on
 * that device until the process exits.  M whose svdq_workspace_bytes(h, M)
 * exceeds it returns SVDQ_ERR_WORKSPACE before anything is launched (about
 * 14,000 rows at K = 3072, R = 32); use svdq_linear_forward for larger M.
 * The first call on each device (made with that device current) looks up the
 * array's device address and caches it; make that first call before any
 * stream capture begins.  The cache is tied to the device's context: after a
 * cudaDeviceReset the next call finds a new context and looks the address up
 * again (the array then starts over in the new context).  The call itself
 * allocates and frees nothing.
 * Every call on a device -- any handle, thread or stream -- shares the one
 * array, which keeps the previous call's contents: calls whose kernels can
 * overlap on the GPU race and corrupt each other's results, so order them (one
 * stream, or events).  Nothing in the array needs to start at zero: every
 * byte the GEMM reads is written earlier in the same call.
 */
#define SVDQ_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
SVDQ_API svdq_status svdq_linear_forward_noalloc(const svdq_linear* h, const void* x, int M, void* y,
                                                 void* stream);

/*
 * svdq_hadamard_transform -- the standalone in-place Walsh-Hadamard transform
 * x <- x H_n / sqrt(n) of every row ("Rotate in quantization and its vLLM
 * implementation", section 3.1, the Hadacore transform: Sylvester recursion,
 * no stored matrix; H symmetric, so the operation is its own inverse).
 *   x      (rows, n) bf16 (dtype 0) or fp16 (dtype 1), row-major, 2-byte aligned,
 *          transformed in place
 *   n      power of two, 1 <= n <= 32768 (else SVDQ_ERR_SHAPE)
 *   rows   >= 0; rows == 0 is a no-op
 * Arithmetic in fp32: butterfly stages h = 1, 2, ..., n/2 in that order
 * ((x[i], x[i+h]) -> (x[i] + x[i+h], x[i] - x[i+h]) for i & h == 0), one
 * multiply by fp32(1/sqrt(n)), then round to nearest even in the storage type.
 * Caller-owned device memory; asynchronous on `stream`.
 */
SVDQ_API svdq_status svdq_hadamard_transform(void* x, int rows, int n, int dtype, void* stream);

/*
 * svdq_quantize_weight -- offline NVFP4 quantization of a dense weight on the
 * GPU (the checkpoint's weight tensors from a bf16 W), with the optional
 * rotation of every row by blockdiag(H_128 / sqrt(128)) ("Rotate in
 * quantization and its vLLM implementation", section 2.1: the offline W' = R W,
 * which in the checkpoint's (N, K) orientation rotates each row like an
 * activation row).  Same rules as the activation quantizer: fp32 butterfly,
 * scale = e4m3_rne_satfinite(fp32(amax/6)), code = e2m1_rne_satfinite(fp32(w/scale)).
 *   w        (N, K)    bf16 in, 16-byte aligned
 *   qweight  (N, K/2)  uint8 out: packed E2M1, element 2j in the low nibble of byte j; 8-byte aligned
 *   wscales  (K/16, N) uint8 out: e4m3 scale bytes, wscales[k/16, n] scales w[n, k]
 * K must be a positive multiple of 16 (of 128 when rotate_block == 128), N >= 1,
 * rotate_block 0 or 128 (else SVDQ_ERR_SHAPE).  Caller-owned device buffers;
 * asynchronous on `stream`.  The outputs are svdq_linear_desc's qweight and
 * wscales.
 */
SVDQ_API svdq_status svdq_quantize_weight(const void* w, int N, int K, int rotate_block, void* qweight,
                                          void* wscales, void* stream);

/*
 * svdq_device_status -- synchronize the handle's device and read + clear its
 * device error word (nonzero when a kernel's bounded wait expired: the kernel
 * then skipped its remaining work, released its tensor memory and returned).
 * *flags receives the word (bit 0: quantizer, bit 1: GEMM).  Returns
 * SVDQ_ERR_DEVICE when it was nonzero.
 */
SVDQ_API svdq_status svdq_device_status(const svdq_linear* h, int* flags);

/*
 * ---------------------------------------------------------------------------
 * MXFP4 with a grouped Hadamard rotation: the FP-Quant forward of "Rotate in
 * quantization and its vLLM implementation", section 3.3 (FPQuantConfig with
 * hadamard_group_size 32, forward_dtype "mxfp4", forward_method "abs_max";
 * the fused rotate-and-quantize step followed by the MXFP4 matmul to bf16):
 *
 *   x_hat = x R^T        R = blockdiag(H_32 / sqrt(32)) (or the identity, group 0)
 *   y     = bf16( alpha * Q(x_hat) Q(W')^T )      W' = W R^T, quantized offline
 *
 * Q() is MXFP4: E2M1 codes, two per byte (element 2j in the low nibble of byte
 * j), one E8M0 scale byte per 32 consecutive K elements (value 2^(byte - 127),
 * 255 = NaN).  The page names the method "abs_max" without its formula; this
 * library takes, for each block, the smallest power of two s with
 * amax(|x_hat|) / s <= 6 (the largest E2M1 magnitude), exponent clamped to
 * [-127, 127] (a zero block gets byte 0, a block holding NaN byte 255 and zero
 * codes), and code = e2m1_rne_satfinite(x_hat / s).  Rotation arithmetic is
 * fp32: butterfly stages h = 1, 2, 4, 8, 16, then one multiply by
 * fp32(1/sqrt(32)).  There is no smoothing and no rank-R branch.
 * ---------------------------------------------------------------------------
 */
typedef struct svdq_mxfp4 svdq_mxfp4;

typedef struct {
  int K;                      /* input features, a positive multiple of 32 */
  int N;                      /* output features, >= 1 */
  int hadamard_group;         /* 32: the rotation above; 0: none */
  const void* qweight;        /* (N, K/2)  uint8: packed E2M1 of the rotated weight W' (device) */
  const void* wscales;        /* (N, K/32) uint8: E8M0 scale bytes of W', row-major (device); 255 is refused */
  float alpha;                /* the matmul's output scale (finite) */
} svdq_mxfp4_desc;

/*
 * svdq_mxfp4_create -- copy the weight codes (rows padded for TMA) and re-tile
 * the weight scales into the tensor-core scale layout in library-owned device
 * memory; synchronizes `stream`, after which the sources may be freed.
 * SVDQ_ERR_SHAPE for K % 32 != 0 or a group other than 0 / 32;
 * SVDQ_ERR_INVALID_ARG for a NaN scale byte or a non-finite alpha.
 */
SVDQ_API svdq_status svdq_mxfp4_create(svdq_mxfp4** out, const svdq_mxfp4_desc* desc, void* stream);

/* Free the handle and its device memory.  NULL is a no-op.  Synchronizes the device. */
SVDQ_API void svdq_mxfp4_destroy(svdq_mxfp4* h);

/* Bytes of device workspace svdq_mxfp4_forward needs for M rows (0 for M == 0). */
SVDQ_API size_t svdq_mxfp4_workspace_bytes(const svdq_mxfp4* h, int M);

/*
 * svdq_mxfp4_quantize -- the fused rotate-and-quantize step alone, in the
 * public layout (no handle; also the offline weight quantizer: pass W's rows).
 *   x       (M, K)    bf16 in, 16-byte aligned; K a positive multiple of 32
 *   codes   (M, K/2)  uint8 out: packed E2M1, element 2j in the low nibble; 16-byte aligned
 *   scales  (M, K/32) uint8 out: E8M0 bytes, row-major
 *   hadamard_group    32 or 0
 * M == 0 is a no-op.  Caller-owned device buffers; asynchronous on `stream`.
 */
SVDQ_API svdq_status svdq_mxfp4_quantize(const void* x, int M, int K, int hadamard_group, void* codes, void* scales,
                                         void* stream);

/*
 * svdq_mxfp4_forward -- y (M, N) bf16 = alpha * Q(x R^T) Q(W')^T: the fused
 * rotate-and-quantize kernel writes codes and scale tiles into `workspace`,
 * then the block-scaled MXFP4 GEMM (tcgen05, 256 x 256 tiles on CTA pairs)
 * writes y.  x 16-byte aligned; workspace >= svdq_mxfp4_workspace_bytes(h, M)
 * bytes, 256-byte aligned, caller-owned, not shared by concurrent calls.
 */
SVDQ_API svdq_status svdq_mxfp4_forward(const svdq_mxfp4* h, const void* x, int M, void* y, void* workspace,
                                        void* stream);

/* As svdq_device_status, for an MXFP4 handle (bit 1: the GEMM's bounded wait expired). */
SVDQ_API svdq_status svdq_mxfp4_device_status(const svdq_mxfp4* h, int* flags);

/*
 * svdq_fp4_mma_loop -- a measurement utility, with no counterpart in the pages:
 * the dense block-scaled FP4 tensor-core rate of the current device, which the
 * GEMM's roofline fraction divides by.  Launches one CTA per SM on `stream`;
 * each issues `iters` x 4 back-to-back tcgen05.mma kind::mxf4nvf4 (NVFP4,
 * M = 128, N = 256, K = 64) from shared memory with no loads in the loop.
 * *ctas receives the number of CTAs; the launch performs
 * (*ctas) * iters * 4 * 2 * 128 * 256 * 64 flops.  Time it with CUDA events on
 * `stream`.  1 <= iters <= 2^20 (at most about a quarter of a second).
 * svdq_fp4_mma_loop_status synchronizes the device and reads + clears the
 * loop's error word (nonzero when its bounded wait expired).
 */
SVDQ_API svdq_status svdq_fp4_mma_loop(int iters, int* ctas, void* stream);
SVDQ_API svdq_status svdq_fp4_mma_loop_status(int* flags);

/* Static text for a status code. */
SVDQ_API const char* svdq_status_string(svdq_status s);

/* Text of the last CUDA error seen by this thread ("" if none). */
SVDQ_API const char* svdq_last_error(void);

/* ABI version: (major << 16) | minor. */
SVDQ_API int svdq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_H_ */

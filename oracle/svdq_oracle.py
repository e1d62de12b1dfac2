"""CPU oracle for the SVDQuant W4A4 linear layer (test infrastructure only).

THIS IS TEST INFRASTRUCTURE.  Only the test suite, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
or run anything in this package.  The product (the CUDA library and its Python
binding) never calls it and shares no code, table or constant with it.

It is a plain, slow, literal restatement of what the layer computes, written in
numpy: fp64 for the matrix products, and exact IEEE fp32 emulation (numpy
float32 ops are correctly rounded) where the method rounds to fp32 before a
discrete decision (the 4-bit codes and the e4m3 scales).  Sources:

* "SVDQuant W4A4" (vLLM-Omni svdquant.md), section "Checkpoint contract":
  tensor names, shapes and dtypes (qweight (N, K/2) int8 with two packed FP4
  values per byte, wscales (K/16, N) float8_e4m3fn, proj_down (K, R),
  proj_up (N, R), smooth_factor (K,), wcscales (N,), wtscale (1,)); K is a
  multiple of 16; wcscales of ones means no per-output correction.
* same page, section "Runtime support": the layer takes bf16 inputs, runs the
  NVFP4 product and then the bf16 rank-R correction (added to the output).
* "Rotate in quantization and its vLLM implementation" (vllm_quantization_
  rotate.md), section 2.1 (math): y = x W = (x R^T)(R W) for orthogonal R;
  section 2.2: the Sylvester Hadamard recursion H_2n = [[H, H], [H, -H]],
  symmetric, H H^T = n I, so H / sqrt(n) is orthogonal and its own inverse;
  section 3.2: the Hadamard is applied per block of the hidden dimension;
  section 1 (background and Q&A): the absmax integer quantizer used in its
  worked examples (scale = max|x| / (2^(n-1) - 1) signed, / (2^n - 1)
  unsigned; q = round(x / scale); x_hat = q * scale).

Conventions the pages leave open (each is a reading of them, taken as the
plainest one the rest of the text supports):

* NVFP4 = E2M1 codes {0, 0.5, 1, 1.5, 2, 3, 4, 6} with a sign bit (bit 3);
  byte j of a row holds element 2j in its low nibble and 2j+1 in its high one.
* One e4m3 (OCP FP8 E4M3FN) scale per 16 consecutive K elements; activation
  scale s = e4m3_rne_satfinite(fp32(amax / 6)); code = rne_satfinite onto the
  E2M1 grid of fp32(x_hat / s), ties to the even code, sign kept (a negative
  value that rounds to zero is code 0x8).  A block whose scale rounds to zero
  gets scale byte 0x00 and codes 0x0.
* x_hat = fp32(x / smooth_factor), then, if rotating, a fp32 Walsh-Hadamard
  butterfly per block (stages h = 1, 2, 4, ... in that order, (a, b) ->
  (a + b, a - b) on pairs (i, i + h) with i & h == 0) followed by one fp32
  multiply by fp32(1 / sqrt(block)).
* The rank-R branch is applied to the same x_hat (smoothed and rotated).
* y = wcscales[n] * wtscale * (Q(x_hat) Q(W)^T)[m, n] + (x_hat proj_down proj_up^T)[m, n].

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(page examples, closed forms, library routines, brute force, invariants).  The
layer's composition -- divide by smooth_factor, then rotate, and the same x_hat
in both branches -- is pinned by a hand-derived case with non-unit smoothing
factors, by exact recovery of an on-grid x_hat through smoothing and a 4- or
16-block rotation, and by the rotation identity y = (x R^T)(R W) through the
rank-R branch and through the dense main product at block 128.
"""
from __future__ import annotations

import numpy as np

# ----------------------------------------------------------------------------
# Number formats
# ----------------------------------------------------------------------------

#: Magnitudes of the eight E2M1 codes 0..7 (sign is bit 3).
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 (exact: bf16 is the top half of fp32)."""
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def e4m3_decode(bits: np.ndarray) -> np.ndarray:
    """OCP FP8 E4M3FN byte -> float64 value.

    Sign bit 7, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 encodes
    subnormals m/8 * 2^-6; S.1111.111 is NaN; there is no infinity.  The
    checkpoint's wscales dtype is float8_e4m3fn ("SVDQuant W4A4", section
    "Checkpoint contract").
    """
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = b & 0x7
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return sign * val


def _e4m3_positive_table():
    codes = np.arange(0, 127, dtype=np.uint8)          # 0x00 .. 0x7E, all finite >= 0
    return codes, e4m3_decode(codes)


def e4m3_encode_rne_satfinite(v: np.ndarray) -> np.ndarray:
    """float -> E4M3FN byte, round to nearest (ties to even mantissa), saturating.

    Finite magnitudes above the largest finite value 448 saturate to 448; NaN
    maps to 0x7F.  The decision is taken on the exact value of ``v`` (float64
    holds every fp32 input and every e4m3 value and midpoint exactly).
    """
    v = np.asarray(v, dtype=np.float64)
    codes, table = _e4m3_positive_table()               # ascending
    a = np.abs(v)
    a_cl = np.minimum(a, table[-1])
    hi = np.searchsorted(table, a_cl, side="left")      # table[hi] >= a
    hi = np.clip(hi, 0, len(table) - 1)
    lo = np.clip(hi - 1, 0, len(table) - 1)
    d_lo = a_cl - table[lo]
    d_hi = table[hi] - a_cl
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ((codes[hi] & 1) == 0))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(a_cl == table[hi], hi, idx)
    out = codes[idx].astype(np.uint8)
    out = np.where(np.signbit(v) & (out != 0), out | 0x80, out).astype(np.uint8)
    out = np.where(np.isnan(v), np.uint8(0x7F), out).astype(np.uint8)
    return out


def e2m1_decode(nibbles: np.ndarray) -> np.ndarray:
    """E2M1 code (low 4 bits) -> float64: magnitude table, sign in bit 3."""
    n = np.asarray(nibbles).astype(np.int64) & 0xF
    mag = E2M1_MAGNITUDES[n & 7]
    return np.where(n & 8, -mag, mag)


def e2m1_encode_rne_satfinite(v: np.ndarray) -> np.ndarray:
    """float -> E2M1 code, round to nearest (ties to the even code), saturating at 6.

    "Even" is the code whose mantissa bit (bit 0) is 0, i.e. ties go to
    0, 1, 2, 4 (not 0.5, 1.5, 3, 6).  The sign bit follows the sign of ``v``
    (a negative value that rounds to magnitude 0 becomes code 0x8).
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), 6.0)
    hi = np.searchsorted(E2M1_MAGNITUDES, a, side="left")
    hi = np.clip(hi, 0, 7)
    lo = np.clip(hi - 1, 0, 7)
    d_lo = a - E2M1_MAGNITUDES[lo]
    d_hi = E2M1_MAGNITUDES[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ((hi & 1) == 0))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(a == E2M1_MAGNITUDES[hi], hi, idx)
    return (idx | np.where(np.signbit(v), 8, 0)).astype(np.uint8)


def pack_e2m1(codes: np.ndarray) -> np.ndarray:
    """(rows, K) codes -> (rows, K/2) bytes; element 2j -> low nibble of byte j."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] & 0xF) | ((c[:, 1::2] & 0xF) << 4)


def unpack_e2m1(packed: np.ndarray) -> np.ndarray:
    """(rows, K/2) bytes -> (rows, K) codes; inverse of :func:`pack_e2m1`."""
    p = np.asarray(packed).view(np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


# ----------------------------------------------------------------------------
# Hadamard rotation (vllm_quantization_rotate.md sections 2.1, 2.2, 3.1, 3.2)
# ----------------------------------------------------------------------------

def sylvester_hadamard(n: int) -> np.ndarray:
    """Unnormalised Sylvester Hadamard H_n (entries +-1), by the section 2.2 recursion."""
    if n < 1 or n & (n - 1):
        raise ValueError("n must be a power of two")
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def hadamard_butterfly(v: np.ndarray, block: int, dtype=np.float32) -> np.ndarray:
    """Unnormalised blockwise Walsh-Hadamard transform along the last axis.

    Fast O(n log n) form (section 3.1: the recursion, no stored matrix).  Each
    stage h = 1, 2, 4, ..., block/2 replaces the pair (v[i], v[i+h]) with
    i & h == 0 by (v[i] + v[i+h], v[i] - v[i+h]), every add rounded to
    ``dtype``.  The result equals v @ H_block (H symmetric) per block.
    """
    v = np.array(v, dtype=dtype, copy=True)
    lead = v.shape[:-1]
    K = v.shape[-1]
    if K % block:
        raise ValueError("last dimension must be a multiple of the block")
    w = v.reshape(*lead, K // block, block)
    h = 1
    while h < block:
        w = w.reshape(*lead, K // block, block // (2 * h), 2, h)
        a = w[..., 0, :].copy()
        b = w[..., 1, :].copy()
        w[..., 0, :] = a + b
        w[..., 1, :] = a - b
        h *= 2
    return w.reshape(*lead, K)


def rotate_rows_fp32(v32: np.ndarray, block: int) -> np.ndarray:
    """x_hat <- fp32(butterfly(x_hat) * fp32(1/sqrt(block))), the online rotation x R^T."""
    c = np.float32(1.0 / np.sqrt(np.float64(block)))
    return (hadamard_butterfly(v32, block, np.float32) * c).astype(np.float32)


def rotate_rows_f64(v: np.ndarray, block: int) -> np.ndarray:
    """Exact-arithmetic (fp64) x R^T with R = blockdiag(H_block / sqrt(block))."""
    return hadamard_butterfly(np.asarray(v, np.float64), block, np.float64) / np.sqrt(block)


def f32_to_bf16_bits(v32: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest, ties to even (NaN -> 0x7FC0 with its sign)."""
    v32 = np.asarray(v32, dtype=np.float32)
    u = v32.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    nan = np.isnan(v32)
    r[nan] = (np.uint16(0x7FC0) | ((u[nan] >> 16) & 0x8000).astype(np.uint16))
    return r


def hadamard_transform(x_bits: np.ndarray, n: int, dtype: str = "bf16") -> np.ndarray:
    """The standalone Walsh-Hadamard transform of each length-n row (n = 2^k):
    x <- x H_n / sqrt(n), in fp32 as the online rotation (the butterfly stages
    h = 1, 2, ..., n/2 in that order, then one multiply by fp32(1/sqrt(n))),
    rounded to the storage type (round to nearest, ties to even).

    "Rotate in quantization and its vLLM implementation", section 3.1: the
    Hadacore transform uses the Sylvester recursion with no stored matrix, and
    since H is symmetric the same operation is its own inverse.  dtype is
    "bf16" or "fp16"; x_bits are the row-major (rows, n) bit patterns.
    """
    x_bits = np.asarray(x_bits, dtype=np.uint16)
    if dtype == "bf16":
        x32 = bf16_to_f32(x_bits)
    elif dtype == "fp16":
        x32 = x_bits.view(np.float16).astype(np.float32)
    else:
        raise ValueError(dtype)
    r = rotate_rows_fp32(x32, n)
    if dtype == "bf16":
        return f32_to_bf16_bits(r)
    return r.astype(np.float16).view(np.uint16)


# ----------------------------------------------------------------------------
# Activation path
# ----------------------------------------------------------------------------

def smooth_and_rotate(x_bits: np.ndarray, smooth_bits: np.ndarray, rotate_block: int) -> np.ndarray:
    """x_hat in fp32: fp32(x / smooth_factor), then the optional block rotation."""
    x = bf16_to_f32(x_bits)
    lam = bf16_to_f32(smooth_bits)
    xh = (x / lam[None, :]).astype(np.float32)
    if rotate_block:
        xh = rotate_rows_fp32(xh, rotate_block)
    return xh


def quantize_nvfp4_rows(v32: np.ndarray):
    """NVFP4 quantization of fp32 rows: one e4m3 scale per 16 consecutive elements.

    scale s = e4m3_rne_satfinite(fp32(amax / 6)) with amax = max |v| over the
    block; code = e2m1_rne_satfinite(fp32(v / s)); a block whose s is zero gets
    codes 0.  Returns (packed codes (rows, K/2) uint8, scale bytes (rows, K/16)
    uint8).
    """
    v32 = np.asarray(v32, dtype=np.float32)
    rows, K = v32.shape
    blk = v32.reshape(rows, K // 16, 16)
    amax = np.max(np.abs(blk), axis=2)                                  # exact
    s_f32 = (amax / np.float32(6.0)).astype(np.float32)                 # fp32 divide
    s_bits = e4m3_encode_rne_satfinite(s_f32)
    s = e4m3_decode(s_bits).astype(np.float32)                          # exact in fp32
    safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        q = (blk / safe[:, :, None]).astype(np.float32)                 # fp32 divide
    codes = e2m1_encode_rne_satfinite(q)
    codes = np.where((s > 0)[:, :, None], codes, np.uint8(0)).astype(np.uint8)
    return pack_e2m1(codes.reshape(rows, K)), s_bits


def quantize_act(x_bits, smooth_bits, rotate_block: int = 0):
    """Activation quantizer: returns (codes (M, K/2), scale bytes (M, K/16), x_hat fp32)."""
    xh = smooth_and_rotate(x_bits, smooth_bits, rotate_block)
    codes, scales = quantize_nvfp4_rows(xh)
    return codes, scales, xh


def dequantize_nvfp4(codes: np.ndarray, scale_bytes: np.ndarray) -> np.ndarray:
    """Packed codes (rows, K/2) + scale bytes (rows, K/16) -> float64 (rows, K)."""
    c = e2m1_decode(unpack_e2m1(codes))
    s = e4m3_decode(scale_bytes)
    return c * np.repeat(s, 16, axis=1)


def dequantize_weight(qweight: np.ndarray, wscales: np.ndarray) -> np.ndarray:
    """Q(W) (N, K) float64 from qweight (N, K/2) and wscales (K/16, N).

    Note the checkpoint's scale tensor is K-block-major: wscales[k // 16, n]
    scales W[n, k] ("SVDQuant W4A4", section "Checkpoint contract").
    """
    return dequantize_nvfp4(np.asarray(qweight).view(np.uint8), np.asarray(wscales).view(np.uint8).T)


def lowrank_down(xh32: np.ndarray, proj_down_bits: np.ndarray) -> np.ndarray:
    """x_hat @ proj_down in float64 ((M, R))."""
    return np.asarray(xh32, np.float64) @ bf16_to_f32(proj_down_bits).astype(np.float64)


def linear_forward(ck, qweight=None, wscales=None, rows=None) -> np.ndarray:
    """y (M, N) float64 for a checkpoint-like object (attributes as in the contract).

    y = wcscales * wtscale * (Q(x_hat) @ Q(W)^T) + (x_hat @ proj_down) @ proj_up^T.
    ``rows`` optionally restricts the computation to a subset of token rows.
    """
    qweight = ck.qweight if qweight is None else qweight
    wscales = ck.wscales if wscales is None else wscales
    x_bits = ck.x if rows is None else ck.x[rows]
    codes, scales, xh = quantize_act(x_bits, ck.smooth_factor, ck.rotate_block)
    xq = dequantize_nvfp4(codes, scales)
    wq = dequantize_weight(qweight, wscales)
    acc = xq @ wq.T
    alpha = bf16_to_f32(ck.wcscales).astype(np.float64) * np.float64(bf16_to_f32(ck.wtscale)[0])
    lr = lowrank_down(xh, ck.proj_down) @ bf16_to_f32(ck.proj_up).astype(np.float64).T
    return alpha[None, :] * acc + lr


# ----------------------------------------------------------------------------
# Offline weight quantization (rotation page section 2.1: W' = R W, done once)
# ----------------------------------------------------------------------------

def quantize_weight_nvfp4(dense_bits: np.ndarray, rotate_block: int = 0):
    """Dense bf16 W (N, K) -> (qweight (N, K/2), wscales (K/16, N)).

    The checkpoint stores W as (N, K), so R W in the page's (K, N) orientation
    rotates each weight row exactly like an activation row.  Rotation and
    quantization are the activation path's (fp32 butterfly, e4m3(amax/6)).
    """
    w = bf16_to_f32(dense_bits).astype(np.float32)
    if rotate_block:
        w = rotate_rows_fp32(w, rotate_block)
    codes, sc = quantize_nvfp4_rows(w)
    return codes, np.ascontiguousarray(sc.T)


# ----------------------------------------------------------------------------
# The integer absmax quantizer of the rotation page's worked examples (section 1)
# ----------------------------------------------------------------------------

def int_absmax_quantize(x, bits: int, signed: bool = True):
    """Returns (scale, q, dequantized) with scale = max|x| / qmax, q = round(x/scale).

    qmax = 2^(bits-1) - 1 (signed, range [-2^(bits-1), qmax]) or 2^bits - 1
    (unsigned, range [0, qmax]); rounding is to nearest, ties to even.
    """
    x = np.asarray(x, dtype=np.float64)
    qmax = (1 << (bits - 1)) - 1 if signed else (1 << bits) - 1
    qmin = -(1 << (bits - 1)) if signed else 0
    scale = np.max(np.abs(x)) / qmax
    q = np.clip(np.rint(x / scale), qmin, qmax).astype(np.int64)
    return scale, q, q * scale


# ----------------------------------------------------------------------------
# MXFP4 with a grouped Hadamard: the FP-Quant forward ("Rotate in quantization
# and its vLLM implementation", section 3.3).  The page gives the configuration
# (hadamard_group_size = 32, forward_dtype "mxfp4", forward_method "abs_max"),
# the fused rotate-and-quantize step and the matmul y = alpha * (x_q w_q^T) in
# bf16.  Readings, where the page is silent:
#   * MXFP4 = E2M1 codes (the grid above) in blocks of 32 consecutive K
#     elements, each block with one shared power-of-two scale stored as an
#     E8M0 byte (value 2^(byte - 127), byte 255 = NaN), the OCP MX format;
#   * "abs_max": the block scale is the smallest power of two s with
#     amax / s <= 6 (the largest E2M1 magnitude), i.e. s = 2^ceil(log2(amax / 6)),
#     so the block's largest magnitude lands inside the grid (the absmax rule of
#     the page's section 1 under a power-of-two constraint); the exponent is
#     clamped to [-127, 127]; a zero block gets 2^-127 (byte 0) and a NaN block
#     byte 255 with zero codes;
#   * code = e2m1_rne_satfinite(x_hat / s) (exact: s is a power of two);
#   * the rotation is the fp32 butterfly of the 128-block case with block 32
#     (x_hat = fp32(butterfly_32(x) * fp32(1/sqrt(32)))), applied to the
#     activations online and to the weight rows offline (W' = W R^T, rows
#     rotated like activation rows); no smoothing and no rank-R branch;
#   * weight scales are stored like the activation scales: (N, K/32) E8M0
#     bytes, row-major; alpha is one fp32 scalar.
# ----------------------------------------------------------------------------

def e8m0_decode(bits: np.ndarray) -> np.ndarray:
    """E8M0 byte -> float64 value 2^(byte - 127); byte 255 is NaN."""
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    return np.where(b == 255, np.nan, np.exp2(b - 127.0))


def mx_abs_max_exponent(amax: np.ndarray) -> np.ndarray:
    """Smallest integer e with 2^e >= amax / 6 (amax > 0 finite), clamped to
    [-127, 127]; -127 for amax == 0.  Decided on exact values: float64 holds
    every fp32 amax and every 6 * 2^e exactly."""
    a = np.asarray(amax, dtype=np.float64)
    e = np.full(a.shape, -127, dtype=np.int64)
    pos = a > 0
    # frexp: a = f * 2^k, f in [0.5, 1); a / 6 = (f / 6) * 2^k; start from a
    # close guess and correct it with exact comparisons against 6 * 2^e.
    f, k = np.frexp(np.where(pos, a, 1.0))
    guess = k.astype(np.int64) - 2
    for _ in range(3):
        too_small = 6.0 * np.exp2(guess.astype(np.float64)) < a          # 2^guess < a / 6
        guess = np.where(too_small, guess + 1, guess)
        too_big = 6.0 * np.exp2(guess.astype(np.float64) - 1.0) >= a     # 2^(guess-1) >= a / 6
        guess = np.where(too_big, guess - 1, guess)
    e = np.where(pos, guess, e)
    return np.clip(e, -127, 127)


def quantize_mxfp4_rows(v32: np.ndarray):
    """MXFP4 quantization of fp32 rows: one E8M0 scale per 32 consecutive
    elements (the abs_max reading above).  Returns (packed codes (rows, K/2)
    uint8, scale bytes (rows, K/32) uint8)."""
    v32 = np.asarray(v32, dtype=np.float32)
    rows, K = v32.shape
    blk = v32.reshape(rows, K // 32, 32).astype(np.float64)
    amax = np.max(np.abs(blk), axis=2)
    nan_blk = np.isnan(amax)
    e = mx_abs_max_exponent(np.where(nan_blk, 0.0, np.minimum(amax, np.finfo(np.float64).max)))
    s = np.exp2(e.astype(np.float64))
    with np.errstate(over="ignore", invalid="ignore"):
        q = blk / s[:, :, None]                                       # exact: power-of-two scale
    codes = e2m1_encode_rne_satfinite(q)
    codes = np.where(nan_blk[:, :, None], np.uint8(0), codes).astype(np.uint8)
    sbytes = np.where(nan_blk, 255, e + 127).astype(np.uint8)
    return pack_e2m1(codes.reshape(rows, K)), sbytes


def dequantize_mxfp4(codes: np.ndarray, scale_bytes: np.ndarray) -> np.ndarray:
    """Packed codes (rows, K/2) + E8M0 bytes (rows, K/32) -> float64 (rows, K)."""
    c = e2m1_decode(unpack_e2m1(codes))
    return c * np.repeat(e8m0_decode(scale_bytes), 32, axis=1)


def fpquant_quantize(x_bits: np.ndarray, group: int = 32):
    """The fused rotate-and-quantize step: x (bf16 bits, (M, K)) -> x_hat =
    blockwise rotation by H_group / sqrt(group) in fp32 (group 0: none) ->
    MXFP4 (codes (M, K/2), scale bytes (M, K/32), x_hat fp32)."""
    xh = bf16_to_f32(x_bits).astype(np.float32)
    if group:
        xh = rotate_rows_fp32(xh, group)
    codes, scales = quantize_mxfp4_rows(xh)
    return codes, scales, xh


def fpquant_quantize_weight(dense_bits: np.ndarray, group: int = 32):
    """Offline weight step: dense bf16 W (N, K) -> rows rotated like activation
    rows -> MXFP4 (qweight (N, K/2), wscales (N, K/32))."""
    codes, scales, _ = fpquant_quantize(dense_bits, group)
    return codes, scales


def fpquant_forward(x_bits, qweight, wscales, alpha: float, group: int = 32, rows=None) -> np.ndarray:
    """y (M, N) float64 = alpha * (Q(x_hat) Q(W')^T), Q = MXFP4 dequantization."""
    xb = x_bits if rows is None else x_bits[rows]
    codes, scales, _ = fpquant_quantize(xb, group)
    return np.float64(alpha) * (dequantize_mxfp4(codes, scales) @ dequantize_mxfp4(qweight, wscales).T)

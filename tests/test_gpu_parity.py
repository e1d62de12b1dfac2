"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.

Bars (from the layer's definition and its NVFP4 conventions):
  * packed E2M1 codes and e4m3 scale bytes: bit-exact;
  * y (bf16): relative Frobenius error <= 5e-3 and every element within
    1e-2 * max|y_oracle|;
  * L = x_hat @ proj_down (bf16; computed as x @ bf16(diag(1/smooth) R^T proj_down)
    on tensor cores): relative Frobenius error <= 1e-2 (the bf16 rounding of
    that product matrix and of the output each contribute up to 2^-9 relative).
"""
import numpy as np
import pytest
import torch

import bit_quantized_linear_svdq_b200 as S
from bit_quantized_linear_svdq_b200 import synthetic
from oracle import svdq_oracle as O

pytestmark = pytest.mark.gpu

Y_REL_FRO = 5e-3
Y_MAX_REL = 1e-2
L_REL_FRO = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from bit_quantized_linear_svdq_b200 import build
    build.build()
    S.load_library()


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev_u8(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.uint8)).cuda()


def host_bf16_to_f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def weights_of(ck):
    if ck.qweight is None:
        qw, ws = O.quantize_weight_nvfp4(ck.dense_weight, ck.rotate_block)
        ck.qweight, ck.wscales = qw, ws
    return ck


def make_layer(ck, with_wc=True):
    ck = weights_of(ck)
    return S.SVDQLinear(dev_u8(ck.qweight), dev_u8(ck.wscales), dev_bf16(ck.proj_down), dev_bf16(ck.proj_up),
                        dev_bf16(ck.smooth_factor), dev_bf16(ck.wcscales) if with_wc else None,
                        dev_bf16(ck.wtscale) if with_wc else None, rotate_block=ck.rotate_block)


def assert_y_close(y_gpu, y_ref, what=""):
    err = y_gpu - y_ref
    rel = np.linalg.norm(err) / max(np.linalg.norm(y_ref), 1e-30)
    mx = np.max(np.abs(err)) / max(np.max(np.abs(y_ref)), 1e-30)
    assert rel <= Y_REL_FRO, f"{what} rel-Frobenius {rel:.3e}"
    assert mx <= Y_MAX_REL, f"{what} max-abs/max|y| {mx:.3e}"


def check_quantizer(layer, ck, rows=None):
    x = dev_bf16(ck.x)
    codes, scales, lowrank = layer.quantize_act(x)
    torch.cuda.synchronize()
    xb = ck.x if rows is None else ck.x[rows]
    c_ref, s_ref, xh = O.quantize_act(xb, ck.smooth_factor, ck.rotate_block)
    c_gpu = codes.cpu().numpy()
    s_gpu = scales.cpu().numpy()
    if rows is not None:
        c_gpu, s_gpu = c_gpu[rows], s_gpu[rows]
    np.testing.assert_array_equal(s_gpu, s_ref)
    bad = np.argwhere(c_gpu != c_ref)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at {bad[:5].tolist()}"
    L_ref = O.lowrank_down(xh, ck.proj_down)
    L_gpu = host_bf16_to_f64(lowrank)
    if rows is not None:
        L_gpu = L_gpu[rows]
    rel = np.linalg.norm(L_gpu - L_ref) / max(np.linalg.norm(L_ref), 1e-30)
    assert rel <= L_REL_FRO, f"L rel-Frobenius {rel:.3e}"


def check_forward(layer, ck, rows=None):
    x = dev_bf16(ck.x)
    y = layer.forward(x)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    y_gpu = host_bf16_to_f64(y)
    if rows is not None:
        y_gpu = y_gpu[rows]
    y_ref = O.linear_forward(ck, rows=rows)
    assert_y_close(y_gpu, y_ref, ck.name)
    return y


def check_forward_workspace(layer, ck):
    """White-box check of the forward path's quantizer output: the codes and
    every tensor-core scale atom in the workspace must equal the oracle's
    bytes (and the K padding must be zero)."""
    M, K = ck.M, ck.K
    x = dev_bf16(ck.x)
    ws = layer.workspace(M)
    S.svdq_linear_forward_quantize(layer.handle, x.data_ptr(), M, ws.data_ptr())
    torch.cuda.synchronize()
    w = ws.cpu().numpy()
    Kp = (K + 127) // 128 * 128
    ka_pad = 4 * ((Kp + 255) // 256)
    mtiles = (M + 127) // 128
    c_ref, s_ref, _ = O.quantize_act(ck.x, ck.smooth_factor, ck.rotate_block)
    codes = w[: M * Kp // 2].reshape(M, Kp // 2)
    np.testing.assert_array_equal(codes[:, : K // 2], c_ref)
    assert not codes[:, K // 2:].any()
    sfa = (M * Kp // 2 + 255) // 256 * 256
    # [row tile][K atom][row % 32][(row % 128) // 32][block in atom]
    atoms = w[sfa: sfa + mtiles * ka_pad * 512].reshape(mtiles, ka_pad, 32, 4, 4)
    m = np.arange(M)
    # (M, ka_pad, 4) -> (M, ka_pad * 4) scale bytes per 16-element block
    rows = atoms[m // 128, :, m % 32, (m % 128) // 32, :].reshape(M, ka_pad * 4)
    np.testing.assert_array_equal(rows[:, : K // 16], s_ref)
    assert not rows[:, K // 16:].any()


# ------------------------------------------------------------------ number-format semantics

def test_convert_semantics_ties_signed_zero_saturation():
    """Hand-made blocks exercising ties-to-even, negative values rounding to
    zero (sign kept), scale saturation and zero / tiny blocks."""
    K = 64
    rows = []
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    r0 = [6.0] + mids + [-m for m in mids] + [0.0]
    rows.append(r0 + [-6.0] + [-m for m in mids] + mids + [0.0] + [0.0] * 32)
    rows.append([6.0, -0.1, -0.2, 0.1, 0.24, -0.24, 0.26, -0.26] + [0.0] * 8 + [1e4] + [1.0] * 15 + [0.0] * 32)
    rows.append([0.0] * 16 + [1e-4] * 16 + [-3e-3] + [0.0] * 15 + [448.0 * 6] + [-1.0] * 15)
    rows.append([float(v) for v in np.linspace(-7, 7, K)])
    rows[3][5] = -0.0            # signed zeros inside blocks with a nonzero scale
    rows[3][40] = -0.0
    rows[0][15] = -0.0
    x = np.array(rows, dtype=np.float32)
    bits = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ck = synthetic.make_checkpoint(4, K, 16, 16, seed=0, n_outliers=0)
    ck.x = bits
    ck.smooth_factor = torch.ones(K).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    layer = make_layer(ck)
    check_quantizer(layer, ck)
    check_forward_workspace(layer, ck)
    check_forward(layer, ck)
    # Same blocks with some negative smooth factors (the sign-fixed division path).
    lam = np.ones(K, dtype=np.float32)
    lam[1::3] = -1.0
    lam[7] = -0.5
    ck.smooth_factor = torch.from_numpy(lam).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    layer2 = make_layer(ck)
    check_quantizer(layer2, ck)
    check_forward_workspace(layer2, ck)
    check_forward(layer2, ck)


@pytest.mark.filterwarnings("ignore:overflow encountered:RuntimeWarning")   # x / lambda overflows to inf by design
@pytest.mark.parametrize("neg_lambda", [False, True])
def test_non_finite_blocks(neg_lambda):
    """Blocks holding +-inf or NaN, or finite values that overflow once divided
    by a small smoothing factor, take the IEEE path: a NaN block gets scale byte
    0x7F and zero codes, an infinite amax saturates the scale to 448.  Codes and
    scales are compared bit-exactly in the public and the tensor-core layouts;
    every other block of the same rows must be unaffected."""
    ck = synthetic.make_checkpoint(200, 512, 256, 32, seed=14, name="non_finite_200x512")
    x = ck.x.copy()
    bf = lambda f: np.array([f], dtype=np.float32).view(np.uint32)[0] >> 16
    x[3, 5] = bf(np.inf)
    x[3, 40] = bf(-np.inf)
    x[77, 100] = bf(np.nan)
    x[130, 16 * 9 + 3] = bf(np.nan)
    x[130, 16 * 9 + 4] = bf(-np.inf)
    x[199, 511] = bf(3.0e38)            # overflows after dividing by a factor < 1
    x[150, 256:272] = bf(-3.0e38)
    ck.x = x
    sm = ck.smooth_factor.copy()
    sm[511] = bf(0.25)
    sm[256:272] = bf(0.5)
    if neg_lambda:
        sm[::7] = sm[::7] | 0x8000
    ck.smooth_factor = sm
    layer = make_layer(ck)
    xd = dev_bf16(ck.x)
    codes, scales, _ = layer.quantize_act(xd, with_lowrank=False)
    torch.cuda.synchronize()
    c_ref, s_ref, _ = O.quantize_act(ck.x, ck.smooth_factor, 0)
    np.testing.assert_array_equal(scales.cpu().numpy(), s_ref)
    np.testing.assert_array_equal(codes.cpu().numpy(), c_ref)
    assert s_ref[77, 100 // 16] == 0x7F and s_ref[3, 0] == 0x7E     # the cases above really occur
    check_forward_workspace(layer, ck)


def _bf16_of(vals):
    return torch.from_numpy(np.asarray(vals, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy() \
        .view(np.uint16)


@pytest.mark.filterwarnings("ignore:overflow encountered:RuntimeWarning")
@pytest.mark.parametrize("rot", [0, 128])
def test_subnormal_and_tiny_activations(rot):
    """Activations at and below the bottom of the fp32 range, and smoothing
    factors at the ends of the accepted magnitudes [2^-126, 2^117): subnormal
    bf16 x, x near 2^-126, tiny entries beside normal ones in the same block
    (so their codes are +-0 under a nonzero scale and the sign of zero shows),
    quotients that overflow (the IEEE path) and quotients far below 2^-19.
    Codes and scales are compared bit for bit with the oracle in both layouts."""
    M, K, N, R = 130, 512, 256, 32
    ck = synthetic.make_checkpoint(M, K, N, R, seed=31 + rot, rotate_block=rot, dense_weight=bool(rot),
                                   name=f"tiny_values_{M}x{K}_rot{rot}")
    rng = np.random.default_rng(5 + rot)
    x = O.bf16_to_f32(ck.x).astype(np.float64)
    sign = np.where(rng.random((M, K)) < 0.5, -1.0, 1.0)
    sub = (rng.integers(1, 128, (M, K)).astype(np.uint16) | np.where(sign < 0, 0x8000, 0).astype(np.uint16))
    xb = ck.x.copy()
    xb[0:32] = sub[0:32]                                            # bf16 subnormals
    xb[32:64] = _bf16_of(sign[32:64] * np.exp2(rng.uniform(-133, -100, (32, K))))   # near underflow
    mask = rng.random((32, K)) < 0.25                               # tiny values inside normal blocks
    xb[64:96] = np.where(mask, sub[64:96], xb[64:96])
    xb[96:110, 40:60] = _bf16_of(sign[96:110, 40:60] * 2.0 ** -20)  # exact tiny quotients
    ck.x = xb
    lam = O.bf16_to_f32(ck.smooth_factor).astype(np.float64)
    lam[0:16] = 2.0 ** -126 * (1 + rng.integers(0, 128, 16) / 128)  # smallest normal factors
    lam[16:32] = 2.0 ** 116 * (1 + rng.integers(0, 128, 16) / 128)  # the largest accepted
    lam[32:48] = 2.0 ** -100
    lam[48:64] = 2.0 ** 100
    lam[::9] *= -1.0
    ck.smooth_factor = _bf16_of(lam)
    assert np.array_equal(O.bf16_to_f32(ck.smooth_factor).astype(np.float64), lam)
    layer = make_layer(ck)
    codes, scales, _ = layer.quantize_act(dev_bf16(ck.x), with_lowrank=False)
    torch.cuda.synchronize()
    c_ref, s_ref, _ = O.quantize_act(ck.x, ck.smooth_factor, rot)
    np.testing.assert_array_equal(scales.cpu().numpy(), s_ref)
    bad = np.argwhere(codes.cpu().numpy() != c_ref)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at {bad[:5].tolist()}"
    # the cases really occur: signed-zero codes under a nonzero scale, saturated scales
    cr = O.unpack_e2m1(c_ref)
    sr = np.repeat(s_ref, 16, axis=1)
    assert np.any((cr == 8) & (sr != 0)) and np.any(s_ref == 0x7E)
    check_forward_workspace(layer, ck)
    assert layer.device_status() == 0


def test_negative_smooth_factors_random():
    ck = synthetic.make_checkpoint(150, 512, 256, 32, seed=12, name="negative_smooth")
    lam = O.bf16_to_f32(ck.smooth_factor).copy()
    lam[::5] *= -1.0
    ck.smooth_factor = torch.from_numpy(lam).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    layer = make_layer(ck)
    check_quantizer(layer, ck)
    check_forward(layer, ck)


# ------------------------------------------------------------------ the named workloads

SMALL = ["tiny_16x256x256_r32"]
FULL = ["attn_proj_4096x3072x3072_r32", "mlp_up_4096x3072x12288_r32", "mlp_down_rot128_4096x12288x3072_r32",
        "small_batch_m1_4096x4096_r32", "small_batch_m16_4096x4096_r32", "small_batch_m64_4096x4096_r32",
        "small_batch_m256_4096x4096_r32", "small_batch_m1024_4096x4096_r32",
        "rank_sweep_4096x3072x3072_r16", "rank_sweep_4096x3072x3072_r64", "rank_sweep_4096x3072x3072_r128"]


@pytest.mark.parametrize("name", SMALL)
def test_small_workload_full_parity(name):
    ck = synthetic.load(name)
    layer = make_layer(ck)
    check_quantizer(layer, ck)
    check_forward(layer, ck)


@pytest.mark.parametrize("name", FULL)
def test_full_workload_parity(name):
    """Full-size workloads: every code/scale byte, every element of L and
    every element of y, for all rows."""
    ck = synthetic.load(name)
    layer = make_layer(ck)
    x = dev_bf16(ck.x)
    codes, scales, _ = layer.quantize_act(x, with_lowrank=False)
    torch.cuda.synchronize()
    c_ref, s_ref, _ = O.quantize_act(ck.x, ck.smooth_factor, ck.rotate_block)
    np.testing.assert_array_equal(scales.cpu().numpy(), s_ref)
    assert np.array_equal(codes.cpu().numpy(), c_ref)
    check_forward_workspace(layer, ck)
    check_quantizer(layer, ck)
    check_forward(layer, ck)


# ------------------------------------------------------------------ ragged shapes and edge cases

def _select_gemm(kernel, monkeypatch):
    """"auto": the library's choice (1..4 rows -> the CUDA-core matrix-vector
    product; alpha folded: 9..32 rows with R <= 32 -> y^T on 128-column full-K
    tiles; above 128 rows -> 256 x 256 tiles on CTA pairs; otherwise split-K
    over a cluster for at most 32 rows, 128 x 256 tiles for R <= 32, 128 x 128
    tiles); "splitk": the same without the CUDA-core and y^T kernels, so
    split-K serves every few-row shape; "n256" / "n128": the one-CTA
    persistent kernels alone."""
    if kernel in ("splitk", "n256", "n128"):
        monkeypatch.setenv("SVDQ_GEMM_NARROW", "0")
        monkeypatch.setenv("SVDQ_GEMV", "0")
    if kernel in ("n256", "n128"):
        monkeypatch.setenv("SVDQ_SPLITK", "0")
        monkeypatch.setenv("SVDQ_GEMM_PAIR", "0")
    if kernel == "n128":
        monkeypatch.setenv("SVDQ_GEMM_TILE_N", "128")


@pytest.mark.parametrize("M,K,N,R,rot", [
    (1, 256, 256, 32, 0),
    (3, 48, 8, 16, 0),          # K < one chunk, N < one tile
    (17, 272, 136, 48, 0),      # K % 128 != 0, N % 128 != 0, odd R
    (129, 400, 200, 16, 0),     # M just over a tile, ragged everything
    (200, 1024, 384, 128, 0),
    (130, 384, 256, 32, 128),   # rotation, K = 3 rotation blocks
    (64, 2048, 640, 64, 128),
    (300, 4096, 128, 32, 0),    # split-K cluster reduction with ragged rows
    (24, 1008, 300, 128, 0),    # few rows: split-K GEMM, ragged N, R = 128
    (2048, 256, 2560, 32, 0),   # more 256 x 256 tiles than CTA pairs: two tiles per pair
    (260, 512, 300, 32, 0),     # pair tiles with N % 8 != 0: element stores instead of TMA
    (300, 768, 520, 48, 0),     # pair tiles, rank box only partly filled (R = 48 of 64)
    (40, 640, 200, 112, 0),     # R = 112: 28 groups per partial-L receive row (swizzle mask 3)
    (520, 512, 384, 96, 128),   # pair tiles with two rank boxes, three stages, rotation
    (20, 512, 300, 32, 0),      # 9..32 rows: y^T on 128-column tiles, ragged N
    (29, 768, 136, 16, 128),    # the same with rotation, R = 16
    (12, 1280, 256, 32, 0),     # y^T tiles, five K steps, two tiles
    (2, 4096, 1000, 32, 0),     # 1..4 rows: CUDA-core product, ragged N
    (4, 9216, 300, 64, 128),    # the same over three 4096-element passes, rotation, R = 64
    (3, 1040, 77, 16, 0),       # K % 32 == 16 (half-masked last piece), R = 16
])
@pytest.mark.parametrize("kernel", ["auto", "splitk", "n256", "n128"])
def test_ragged_shapes(M, K, N, R, rot, kernel, monkeypatch):
    """Every GEMM kernel on every ragged shape (see _select_gemm)."""
    _select_gemm(kernel, monkeypatch)
    ck = synthetic.make_checkpoint(M, K, N, R, seed=M + K + N + R, rotate_block=rot, dense_weight=bool(rot),
                                   wcscales="uniform", wtscale=0.75, name=f"ragged_{M}x{K}x{N}_r{R}_rot{rot}")
    layer = make_layer(ck)
    check_quantizer(layer, ck)
    check_forward_workspace(layer, ck)
    check_forward(layer, ck)


@pytest.mark.parametrize("M", [150, 2])
@pytest.mark.parametrize("kernel", ["auto", "splitk", "n256", "n128"])
def test_zero_alpha_columns(M, kernel, monkeypatch):
    """Columns with wcscales = 0 reduce to the rank-R branch alone, in every
    GEMM kernel (the folded one gives them alpha' = 1 and zero weight scales)."""
    _select_gemm(kernel, monkeypatch)
    ck = synthetic.make_checkpoint(M, 512, 520, 32, seed=12, wcscales="uniform",
                                   name=f"zero_alpha_{M}x512x520_r32")
    # Tile edges plus every seventh column: with two rows the check still
    # averages over ~170 outputs of the rank-R branch, whose bf16 L and y
    # roundings alone give ~3e-3 (20 outputs gave 5.3e-3 on a correct kernel).
    zero_cols = np.unique(np.concatenate([[0, 1, 127, 128, 255, 256, 300, 511, 512, 519], np.arange(3, 520, 7)]))
    ck.wcscales = ck.wcscales.copy()
    ck.wcscales[zero_cols] = 0
    layer = make_layer(ck)
    y = host_bf16_to_f64(check_forward(layer, ck))
    xh = O.smooth_and_rotate(ck.x, ck.smooth_factor, 0)
    lr = O.lowrank_down(xh, ck.proj_down) @ O.bf16_to_f32(ck.proj_up).astype(np.float64).T
    assert_y_close(y[:, zero_cols], lr[:, zero_cols], "zero-alpha columns")


@pytest.mark.parametrize("M,K,N,R,rot", [
    (1, 4096, 512, 32, 0),
    (2, 384, 300, 16, 0),       # three slices, ragged N
    (3, 1024, 256, 32, 128),    # rotation
    (4, 12288, 200, 16, 128),   # three 4096-element passes, rotation
    (4, 128, 64, 32, 0),        # one slice
    (1, 2176, 136, 32, 0),      # 17 slices
])
def test_few_row_path(M, K, N, R, rot):
    """1..4 rows (few-row quantizer + CUDA-core matrix-vector product) on
    shapes that cover 1..17 slices, rotation, K over three 4096-element
    passes and ragged N: y matches the oracle and repeats bit for bit."""
    ck = synthetic.make_checkpoint(M, K, N, R, seed=3 * M + K + N, rotate_block=rot, dense_weight=bool(rot),
                                   wcscales="uniform", wtscale=0.75, name=f"few_{M}x{K}x{N}_r{R}_rot{rot}")
    layer = make_layer(ck)
    y1 = check_forward(layer, ck)
    assert torch.equal(layer.forward(dev_bf16(ck.x)), y1)


def test_unfoldable_alpha_takes_plain_epilogue(monkeypatch):
    """wtscale = 2^-30 is outside the range where proj_up / alpha keeps bf16
    precision, so the layer keeps alpha in the epilogue (the 128 x 128 kernel:
    split-K, which also applies alpha in its epilogue, is switched off here);
    results still match."""
    monkeypatch.setenv("SVDQ_SPLITK", "0")
    ck = synthetic.make_checkpoint(140, 512, 384, 32, seed=13, wcscales="uniform", wtscale=2.0 ** -30,
                                   name="tiny_alpha_140x512x384_r32")
    layer = make_layer(ck)
    check_forward(layer, ck)


def test_default_wcscales_wtscale_are_ones():
    ck = synthetic.make_checkpoint(32, 256, 256, 32, seed=5)
    layer = make_layer(ck, with_wc=False)
    check_forward(layer, ck)


def test_zero_weights_give_lowrank_branch_only():
    ck = synthetic.make_checkpoint(40, 512, 256, 32, seed=6)
    ck.qweight = np.zeros_like(ck.qweight)
    layer = make_layer(ck)
    y = check_forward(layer, ck)
    xh = O.smooth_and_rotate(ck.x, ck.smooth_factor, 0)
    lr = O.lowrank_down(xh, ck.proj_down) @ O.bf16_to_f32(ck.proj_up).astype(np.float64).T
    assert_y_close(host_bf16_to_f64(y), lr, "lowrank only")


def test_deterministic_and_batch_consistent():
    ck = synthetic.make_checkpoint(300, 1024, 512, 32, seed=7)
    layer = make_layer(ck)
    x = dev_bf16(ck.x)
    y1 = layer.forward(x).clone()
    y2 = layer.forward(x).clone()
    assert torch.equal(y1, y2)
    # A sub-batch served by the same kernels (same tile kernel, same K split
    # of the quantizer) reproduces its rows bit for bit.
    y_sub = layer.forward(x[:260].contiguous())
    assert torch.equal(y_sub, y1[:260])
    # One row takes the few-row path (CUDA-core quantizer and matrix-vector
    # product), whose rank-R sums run in another order: deterministic, and
    # equal to the batched row within the layer's tolerance.
    y_one = layer.forward(x[5:6].contiguous())
    assert torch.equal(layer.forward(x[5:6].contiguous()), y_one)
    assert_y_close(host_bf16_to_f64(y_one), host_bf16_to_f64(y1[5:6]), "one row against the batch")


def test_zero_rows_is_noop():
    ck = synthetic.make_checkpoint(4, 256, 256, 32, seed=8)
    layer = make_layer(ck)
    S.svdq_linear_forward(layer.handle, 0, 0, 0, 0)
    assert S.svdq_workspace_bytes(layer.handle, 0) == 0


@pytest.mark.parametrize("M", [64, 300, 1000, 1030, 4100])
def test_forward_host_matches_device_path(M):
    """The host-buffer call pipelines its copies over row chunks: one chunk
    (the device call itself, so bit for bit the same y) for M < 1024, six from
    M = 1024 on.  A chunk's quantizer may split K over more CTAs than the whole
    call's, which changes the fp32 summation order of L = x_hat proj_down, so
    chunked results are held to the oracle's y tolerance instead."""
    ck = synthetic.make_checkpoint(M, 512, 384, 32, seed=9)
    layer = make_layer(ck)
    x = dev_bf16(ck.x)
    y_dev_ref = layer.forward(x).clone()
    xh = x.cpu().pin_memory()
    yh = torch.full((M, 384), float("nan"), dtype=torch.bfloat16).pin_memory()
    xd = torch.empty_like(x)
    yd = torch.empty((M, 384), dtype=torch.bfloat16, device="cuda")
    ws = layer.workspace(M)
    S.svdq_linear_forward_host(layer.handle, xh.data_ptr(), M, yh.data_ptr(), xd.data_ptr(), yd.data_ptr(),
                               ws.data_ptr())
    assert layer.device_status() == 0
    if M < 1024:
        assert torch.equal(yh, y_dev_ref.cpu())
    else:
        assert not torch.isnan(yh.float()).any()
        assert_y_close(host_bf16_to_f64(yh), O.linear_forward(ck), ck.name)


def test_runtime_argument_errors():
    ck = synthetic.make_checkpoint(4, 256, 256, 32, seed=10)
    layer = make_layer(ck)
    x = dev_bf16(ck.x)
    y = torch.empty((4, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(S.SvdqError) as e:
        S.svdq_linear_forward(layer.handle, x.data_ptr(), 4, y.data_ptr(), 0)
    assert e.value.status == 5
    ws = layer.workspace(4)
    with pytest.raises(S.SvdqError) as e:
        S.svdq_linear_forward(layer.handle, x.data_ptr() + 2, 4, y.data_ptr(), ws.data_ptr())
    assert e.value.status == 1
    bad = synthetic.make_checkpoint(4, 256, 256, 32, seed=11)
    bad.smooth_factor = bad.smooth_factor.copy()
    bad.smooth_factor[3] = 0
    with pytest.raises(S.SvdqError) as e:
        make_layer(bad)
    assert e.value.status == 1
    # smoothing factors outside the magnitudes [2^-126, 2^117) for which the
    # quantizer's division is exact are refused at create
    for v in (2.0 ** 117, -2.0 ** 120, 2.0 ** -127, -1e-40):
        bad.smooth_factor = synthetic.make_checkpoint(4, 256, 256, 32, seed=11).smooth_factor.copy()
        bad.smooth_factor[7] = _bf16_of([v])[0]
        with pytest.raises(S.SvdqError) as e:
            make_layer(bad)
        assert e.value.status == 1 and "magnitude" in str(e.value), v


def test_gemm_kernel_query():
    """svdq_linear_gemm_kernel names the kernel the dispatch picks (K = N =
    3072, R = 32: the attention-projection shape)."""
    ck = synthetic.make_checkpoint(8, 3072, 3072, 32, seed=21, name="query_8x3072x3072_r32")
    layer = make_layer(ck)
    for M, expect in [(1, "gemv_nvfp4"), (4, "gemv_nvfp4"), (5, "splitk"), (20, "narrow"), (100, "n256"),
                      (300, "pair")]:
        name = layer.gemm_kernel(M)
        assert expect in name, (M, name)
    assert layer.gemm_kernel(0) == ""

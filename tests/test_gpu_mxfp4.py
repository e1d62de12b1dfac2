"""GPU parity of the MXFP4 linear with a grouped Hadamard (the FP-Quant forward
of "Rotate in quantization and its vLLM implementation", section 3.3) against
the CPU oracle, through the C ABI.

Bars: packed E2M1 codes and E8M0 scale bytes bit-exact (the rotation is the
oracle's fp32 butterfly order, the scale an exact power-of-two decision);
y (bf16) within relative Frobenius 5e-3 and every element within
1e-2 * max|y_oracle| (the products are exact, so the difference is the fp32
accumulation order and the bf16 rounding of y).
"""
import numpy as np
import pytest
import torch

import bit_quantized_linear_svdq_b200 as S
from oracle import svdq_oracle as O

pytestmark = pytest.mark.gpu

Y_REL_FRO = 5e-3
Y_MAX_REL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from bit_quantized_linear_svdq_b200 import build
    build.build()
    S.load_library()


def _bf16_bits(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy() \
        .view(np.uint16)


def _dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _dev_u8(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.uint8)).cuda()


def _inputs(M, K, N, seed):
    """x ~ N(0, 1) with 1% of the channels (at least one) scaled x30, W ~ N(0, 0.02)."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((M, K), generator=g)
    ch = torch.randperm(K, generator=g)[: max(1, round(0.01 * K))]
    x[:, ch] *= 30.0
    w = torch.randn((N, K), generator=g) * 0.02
    return _bf16_bits(x.numpy()), _bf16_bits(w.numpy())


def _assert_y_close(y_gpu, y_ref, what):
    err = y_gpu - y_ref
    rel = np.linalg.norm(err) / max(np.linalg.norm(y_ref), 1e-30)
    mx = np.max(np.abs(err)) / max(np.max(np.abs(y_ref)), 1e-30)
    assert rel <= Y_REL_FRO, f"{what}: rel-Frobenius {rel:.3e}"
    assert mx <= Y_MAX_REL, f"{what}: max-abs/max|y| {mx:.3e}"


@pytest.mark.parametrize("M,K,group", [(300, 3072, 32), (7, 1056, 32), (130, 512, 0), (1, 32, 32)])
def test_quantize_bit_exact(M, K, group):
    xb, _ = _inputs(M, K, 1, seed=M + K + group)
    codes, scales = S.mxfp4_quantize(_dev_bf16(xb), group)
    torch.cuda.synchronize()
    c_ref, s_ref, _ = O.fpquant_quantize(xb, group)
    np.testing.assert_array_equal(scales.cpu().numpy(), s_ref)
    bad = np.argwhere(codes.cpu().numpy() != c_ref)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at {bad[:5].tolist()}"


@pytest.mark.filterwarnings("ignore:overflow encountered:RuntimeWarning")
@pytest.mark.parametrize("group", [0, 32])
def test_quantize_special_blocks(group):
    """Zero, NaN, infinite, subnormal and saturating blocks; ties at every E2M1
    midpoint under a power-of-two scale."""
    M, K = 8, 256
    rng = np.random.default_rng(3 + group)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[0, :32] = 0.0
    x[1, 5] = np.nan
    x[1, 70] = np.inf
    x[2, 40] = -np.inf
    x[3, :] = rng.standard_normal(K) * 1e-39          # subnormal bf16
    x[4, :] = rng.standard_normal(K) * 3e38
    s = 2.0 ** -3
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    x[5, :7] = mids * s
    x[5, 7] = 6 * s
    x[5, 8:15] = -mids * s
    x[5, 15:32] = 0.0
    xb = _bf16_bits(x)
    codes, scales = S.mxfp4_quantize(_dev_bf16(xb), group)
    torch.cuda.synchronize()
    c_ref, s_ref, _ = O.fpquant_quantize(xb, group)
    np.testing.assert_array_equal(scales.cpu().numpy(), s_ref)
    np.testing.assert_array_equal(codes.cpu().numpy(), c_ref)
    assert s_ref[1, 0] == 255 and s_ref[0, 0] == 0 if group == 0 else True


def test_weight_quantizer_matches_oracle():
    """The same kernel quantizes the weight rows offline (W' = W R^T)."""
    _, wb = _inputs(1, 1024, 384, seed=9)
    qw, ws = S.mxfp4_quantize(_dev_bf16(wb), 32)
    torch.cuda.synchronize()
    qw_ref, ws_ref = O.fpquant_quantize_weight(wb, 32)
    np.testing.assert_array_equal(qw.cpu().numpy(), qw_ref)
    np.testing.assert_array_equal(ws.cpu().numpy(), ws_ref)


@pytest.mark.parametrize("M,K,N,group,alpha", [
    (300, 3072, 512, 32, 1.0),
    (1, 1024, 256, 32, 0.5),       # one row: a 256-row pair tile with 255 rows beyond M
    (100, 1056, 300, 32, 1.25),    # K % 128 != 0, ragged N (element stores)
    (513, 512, 264, 0, 2.0),       # no rotation, ragged M and N % 8 == 0
    (4096, 3072, 3072, 32, 1.0),   # the attention-projection shape
])
def test_forward_matches_oracle(M, K, N, group, alpha):
    xb, wb = _inputs(M, K, N, seed=M + 7 * K + N)
    qw_ref, ws_ref = O.fpquant_quantize_weight(wb, group)
    layer = S.MXFP4Linear(_dev_u8(qw_ref), _dev_u8(ws_ref), alpha=alpha, hadamard_group=group)
    try:
        y = layer.forward(_dev_bf16(xb))
        torch.cuda.synchronize()
        assert layer.device_status() == 0
        y_ref = O.fpquant_forward(xb, qw_ref, ws_ref, alpha, group)
        _assert_y_close(y.float().cpu().numpy().astype(np.float64), y_ref, f"{M}x{K}x{N} g{group}")
        # a second call on new inputs: nothing stale in the workspace
        xb2, _ = _inputs(M, K, N, seed=M + 7 * K + N + 1)
        y2 = layer.forward(_dev_bf16(xb2))
        torch.cuda.synchronize()
        _assert_y_close(y2.float().cpu().numpy().astype(np.float64),
                        O.fpquant_forward(xb2, qw_ref, ws_ref, alpha, group), "second call")
    finally:
        layer.close()


def test_create_rejects_nan_scale_and_zero_rows_noop():
    _, wb = _inputs(1, 256, 256, seed=5)
    qw, ws = O.fpquant_quantize_weight(wb, 32)
    ws = ws.copy()
    ws[3, 2] = 255
    with pytest.raises(S.SvdqError) as e:
        S.MXFP4Linear(_dev_u8(qw), _dev_u8(ws))
    assert e.value.status == 1
    layer = S.MXFP4Linear(_dev_u8(qw), _dev_u8(O.fpquant_quantize_weight(wb, 32)[1]))
    try:
        y = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
        S.svdq_mxfp4_forward(layer.handle, y.data_ptr() or 256, 0, y.data_ptr() or 256, 256)
        assert S.svdq_mxfp4_workspace_bytes(layer.handle, 0) == 0
    finally:
        layer.close()

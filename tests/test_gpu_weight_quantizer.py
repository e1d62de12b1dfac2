"""GPU parity of the offline weight quantizer (svdq_quantize_weight) against
the oracle's quantize_weight_nvfp4: packed E2M1 codes and e4m3 scale bytes
bit-exact, with and without the 128-block row rotation, on ragged shapes and
special blocks (all-zero, tiny, saturating, infinite, NaN)."""
import numpy as np
import pytest
import torch

import bit_quantized_linear_svdq_b200 as S
from bit_quantized_linear_svdq_b200 import synthetic
from oracle import svdq_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from bit_quantized_linear_svdq_b200 import build
    build.build()
    S.load_library()


def _bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bits, round to nearest even (NaN kept NaN)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    nan = np.isnan(a)
    r[nan] = 0x7FC0
    return r


def _weights(N, K, seed, special=False):
    rng = np.random.default_rng(seed)
    w = rng.normal(0.0, 0.02, size=(N, K)).astype(np.float32)
    cols = rng.choice(K, size=max(1, K // 100), replace=False)
    w[:, cols] *= 30.0                                      # outlier input channels
    if special:
        w[0, 0:16] = 0.0                                    # scale 0 -> codes 0
        w[1, 16:32] = 1e-30                                 # below the smallest scale
        w[2, 32:48] = 4000.0                                # amax / 6 beyond 448: saturates
        w[3, 0:16] = np.inf
        w[3, 16] = -np.inf
        w[4, 48] = np.nan
    return _bf16_bits(w)


def _gpu_quantize(bits, rotate_block):
    w = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()
    qw, ws = S.quantize_weight(w, rotate_block)
    torch.cuda.synchronize()
    return qw.cpu().numpy(), ws.cpu().numpy()


@pytest.mark.parametrize("N,K,rot", [
    (1, 16, 0),
    (37, 48, 0),          # K < one 128-element chunk, N < one 32-row tile
    (300, 1008, 0),       # ragged chunk (K % 128 == 112) and ragged row tile
    (64, 4096, 0),
    (8, 128, 128),
    (100, 384, 128),
    (257, 512, 128),      # one row past a row tile
])
def test_matches_oracle_bit_exact(N, K, rot):
    bits = _weights(N, K, seed=N * 7 + K + rot)
    qw, ws = _gpu_quantize(bits, rot)
    qw_ref, ws_ref = O.quantize_weight_nvfp4(bits, rot)
    assert qw.shape == qw_ref.shape and ws.shape == ws_ref.shape
    assert np.array_equal(ws, ws_ref), f"scales differ at {np.argwhere(ws != ws_ref)[:5]}"
    assert np.array_equal(qw, qw_ref), f"codes differ at {np.argwhere(qw != qw_ref)[:5]}"


@pytest.mark.filterwarnings("ignore::RuntimeWarning")
@pytest.mark.parametrize("rot", [0, 128])
def test_special_blocks(rot):
    bits = _weights(40, 256, seed=5 + rot, special=True)
    qw, ws = _gpu_quantize(bits, rot)
    qw_ref, ws_ref = O.quantize_weight_nvfp4(bits, rot)
    assert np.array_equal(ws, ws_ref), f"scales differ at {np.argwhere(ws != ws_ref)[:5]}"
    assert np.array_equal(qw, qw_ref), f"codes differ at {np.argwhere(qw != qw_ref)[:5]}"
    if not rot:
        assert ws[0, 0] == 0 and not qw[0, :8].any()        # all-zero block
        assert ws[2, 2] == 0x7E                            # 448, saturated


def test_rotated_checkpoint_weights():
    """The rotated MLP-down checkpoint's dense weight: the GPU gives the bytes
    the oracle gives, so a layer built from either is the same layer."""
    ck = synthetic.make_checkpoint(16, 1024, 384, 32, seed=3, rotate_block=128, dense_weight=True,
                                   name="dense_rot_16x1024x384_r32")
    qw, ws = _gpu_quantize(ck.dense_weight, 128)
    qw_ref, ws_ref = O.quantize_weight_nvfp4(ck.dense_weight, 128)
    assert np.array_equal(qw, qw_ref) and np.array_equal(ws, ws_ref)

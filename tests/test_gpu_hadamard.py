"""GPU parity of the standalone Walsh-Hadamard transform
(svdq_hadamard_transform) against the oracle's hadamard_transform: bit-exact
rows for every size 2^k up to 32768, bf16 and fp16, and the transform applied
twice gives back the input up to the two roundings to the storage type."""
import numpy as np
import pytest
import torch

import bit_quantized_linear_svdq_b200 as S
from oracle import svdq_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from bit_quantized_linear_svdq_b200 import build
    build.build()
    S.load_library()


def _bits(rows, n, dtype, seed):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((rows, n)) * np.exp(rng.uniform(-3, 3, (rows, 1)))).astype(np.float32)
    if dtype == "bf16":
        return O.f32_to_bf16_bits(x)
    return x.astype(np.float16).view(np.uint16)


def _gpu(bits, dtype):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()
    t = t.view(torch.bfloat16 if dtype == "bf16" else torch.float16)
    S.hadamard_transform(t)                      # in place
    torch.cuda.synchronize()
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("rows,n", [(5, 1), (3, 2), (7, 16), (9, 32), (300, 64), (33, 128), (11, 1024),
                                    (3, 4096), (2, 8192), (3, 32768), (8193, 8)])
def test_matches_oracle_bit_exact(rows, n, dtype):
    bits = _bits(rows, n, dtype, seed=rows * 31 + n)
    got = _gpu(bits, dtype)
    ref = O.hadamard_transform(bits, n, dtype)
    assert np.array_equal(got, ref), f"differs at {np.argwhere(got != ref)[:5]}"


@pytest.mark.parametrize("n", [128, 32768])
def test_twice_is_identity_up_to_rounding(n):
    bits = _bits(4, n, "bf16", seed=n)
    once = _gpu(bits, "bf16")
    twice = _gpu(once, "bf16")
    np.testing.assert_array_equal(twice, O.hadamard_transform(O.hadamard_transform(bits, n), n))
    x0 = O.bf16_to_f32(bits).astype(np.float64)
    x2 = O.bf16_to_f32(twice).astype(np.float64)
    assert np.max(np.abs(x2 - x0)) <= 2 ** -6 * np.abs(x0).max()


def test_zero_rows_is_noop():
    S.svdq_hadamard_transform(0, 0, 64, 0)

"""The few-row CUDA-core product (csrc/gemv_nvfp4.cu) sums each 16-element
scale block as two fp16 lanes of eight E2M1 x E2M1 products, then adds the
block sum times s_a * s_w into fp32.  Its claim: the fp16 lane sums and the
fp32 block sum are exact, and so is the e4m3 x e4m3 scale product, so the
only roundings are the fp32 accumulation per block and the final bf16 store.
This test checks that numerical argument exhaustively on the CPU; it checks
the method, not the kernel (the GPU parity tests check the kernel)."""
import itertools

import numpy as np

# E2M1 magnitudes (OCP MX FP4: 1 sign, 2 exponent, 1 mantissa bit).
E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
E2M1_ALL = np.concatenate([E2M1, -E2M1])


def e4m3_values():
    """Every finite E4M3 (fn) value: bias 7, subnormals at exponent field 0,
    0x7F / 0xFF are NaN (the largest finite magnitude is 448)."""
    vals = []
    for b in range(256):
        s, e, m = b >> 7, (b >> 3) & 0xF, b & 7
        if e == 0xF and m == 7:
            continue
        v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
        vals.append(-v if s else v)
    return np.array(vals)


def test_e2m1_products_are_quarter_multiples_up_to_36():
    p = np.multiply.outer(E2M1_ALL, E2M1_ALL).ravel()
    assert np.all(p * 4 == np.round(p * 4))
    assert np.max(np.abs(p)) == 36.0


def test_every_eight_product_lane_sum_is_exact_in_fp16():
    # A lane holds eight products: any multiple of 1/4 with |s| <= 8 * 36.
    # fp16 must represent each such value, so that every fused multiply-add
    # of the lane (exact product + exact partial sum) is itself exact.
    k = np.arange(-8 * 36 * 4, 8 * 36 * 4 + 1)
    s = k / 4.0
    assert np.array_equal(s.astype(np.float16).astype(np.float64), s)


def test_lane_sums_reach_their_bound():
    # The bound is attained (eight 6 x 6 products), so it cannot be tightened,
    # and the lane sum 288 sits in the fp16 binade [256, 512) of spacing 1/4.
    assert np.float16(8 * 36.0) == 288.0
    assert np.spacing(np.float16(288.0)) == 0.25


def test_block_sum_of_two_lanes_is_exact_in_fp32():
    k = np.arange(-2 * 8 * 36 * 4, 2 * 8 * 36 * 4 + 1)
    s = k / 4.0
    assert np.array_equal(s.astype(np.float32).astype(np.float64), s)


def test_random_blocks_match_exact_sums():
    # fp16 fused multiply-add emulated in fp64 (exact operands, one rounding
    # to fp16 per step), on random and on extreme blocks.
    rng = np.random.default_rng(0)
    blocks = [rng.choice(E2M1_ALL, size=(2, 16)) for _ in range(2000)]
    blocks.append(np.stack([np.full(16, 6.0), np.full(16, 6.0)]))
    blocks.append(np.stack([np.full(16, -6.0), np.full(16, 6.0)]))
    for a, w in blocks:
        lanes = [0.0, 0.0]
        for i in range(16):
            h = i % 2                   # the two halves of one f16x2: even and odd elements
            lanes[h] = float(np.float16(a[i] * w[i] + lanes[h]))
        assert float(np.float32(lanes[0]) + np.float32(lanes[1])) == float(np.dot(a, w))


def test_e4m3_scale_products_are_exact_in_fp32():
    v = e4m3_values()
    pos = np.unique(np.abs(v))
    prod = np.multiply.outer(pos, pos).ravel()
    assert np.array_equal(prod.astype(np.float32).astype(np.float64), prod)
    # and the smallest nonzero product is a normal fp32 number
    nz = prod[prod > 0]
    assert nz.min() >= np.finfo(np.float32).tiny


def test_e4m3_values_are_exact_in_fp16():
    # The kernel converts scale bytes with cvt.rn.f16x2.e4m3x2; every finite
    # e4m3 value (448 max, 2^-9 min subnormal) is an fp16 value.
    v = e4m3_values()
    assert np.array_equal(v.astype(np.float16).astype(np.float64), v)


def test_e2m1_values_are_exact_in_fp16():
    assert np.array_equal(E2M1_ALL.astype(np.float16).astype(np.float64), E2M1_ALL)


def test_lane_split_covers_each_block_once():
    # Within a 16-byte piece (32 elements, two blocks) the kernel's f16x2
    # accumulator h0 takes bytes 0-7 (elements 0-15, block 0) and h1 bytes
    # 8-15 (block 1); each byte's two elements go to the two halves.
    elems = {0: set(), 1: set()}
    for q, b in itertools.product(range(4), range(4)):
        byte = 4 * q + b
        lane = 0 if q < 2 else 1
        elems[lane].update({2 * byte, 2 * byte + 1})
    assert elems[0] == set(range(16)) and elems[1] == set(range(16, 32))

"""Pins for the CPU oracle: page examples, closed forms, library routines,
brute force and invariants.  None of these re-types the oracle's own formula:
each checks it against something fixed outside it.

Sources cited per test:
  [rot]  vllm_quantization_rotate.md ("Rotate in quantization and its vLLM
         implementation"): section 1 worked INT4 examples and Q&A, section 2.1
         rotation identity, section 2.2 Sylvester Hadamard, section 3.1 Hadacore
         test pattern (fast transform vs dense matmul; applying it twice is the
         identity).
  [svdq] "SVDQuant W4A4" (vLLM-Omni svdquant.md): "Checkpoint contract" and
         "Runtime support".
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import svdq_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _bf16_bits(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------- [rot] section 1

def test_int4_unsigned_example():
    g = _golden("rotate_page_int4_examples.json")["unsigned_int4"]
    scale, q, deq = O.int_absmax_quantize(g["x"], 4, signed=False)
    assert abs(scale - g["scale"]) < 5e-3
    assert list(q) == g["q"]
    np.testing.assert_allclose(deq, g["dequant"], atol=1e-9)


def test_int4_extreme_outlier_example_and_slips():
    g = _golden("rotate_page_int4_examples.json")["extreme_outlier"]
    x = np.array(g["x"])
    scale, q, deq = O.int_absmax_quantize(x, 4, signed=True)
    assert abs(scale - g["scale"]) < 5e-3
    assert list(q) == g["q"]
    np.testing.assert_allclose(x - deq, g["error"], atol=1e-9)
    assert abs(np.mean((x - deq) ** 2) - g["mse"]) < 5e-4
    H4 = np.array(_golden("rotate_page_hadamard.json")["H4_normalized"])
    xr = x @ H4.T
    printed = np.array(g["rotated_printed"])
    ok = [i for i in range(4) if i not in g["rotated_slip_indices"]]
    np.testing.assert_allclose(xr[ok], printed[ok], atol=5e-3)
    # The two slips: the exact values are -40.00 and 39.80.
    np.testing.assert_allclose(xr[g["rotated_slip_indices"]], [-40.0, 39.8], atol=1e-12)
    s2, q2, d2 = O.int_absmax_quantize(xr, 4, signed=True)
    assert abs(s2 - g["rotated_scale"]) < 5e-4
    assert list(q2) == g["rotated_q"]
    np.testing.assert_allclose(d2, g["rotated_dequant"], atol=5e-3)
    # Inverse rotation with the same (symmetric) matrix.
    np.testing.assert_allclose(d2 @ H4, g["recovered"], atol=5e-3)


def test_int4_realistic_example_mse_drop():
    g = _golden("rotate_page_int4_examples.json")["realistic"]
    x = np.array(g["x"])
    scale, q, deq = O.int_absmax_quantize(x, 4, signed=True)
    assert abs(scale - g["scale"]) < 5e-4
    assert list(q) == g["q"]
    np.testing.assert_allclose(deq, g["dequant"], atol=5e-4)
    np.testing.assert_allclose(deq - x, g["error"], atol=5e-4)  # printed as dequant - x
    mse_plain = np.mean((x - deq) ** 2)
    # the page squares its rounded intermediates (0.514, 0.214), hence 1e-3
    assert abs(mse_plain - g["mse"]) < 1e-3
    # Rotation by the oracle's own block transform (block 4), fp64.
    xr = O.rotate_rows_f64(x[None, :], 4)[0]
    np.testing.assert_allclose(xr, g["rotated"], atol=5e-4)
    s2, q2, d2 = O.int_absmax_quantize(xr, 4, signed=True)
    assert abs(s2 - g["rotated_scale"]) < 5e-4
    assert list(q2) == g["rotated_q"]
    np.testing.assert_allclose(d2, g["rotated_dequant"], atol=5e-4)
    rec = O.rotate_rows_f64(d2[None, :], 4)[0]        # the inverse is the same transform
    np.testing.assert_allclose(rec, g["recovered"], atol=5e-4)
    np.testing.assert_allclose(rec - x, g["recovered_error"], atol=5e-4)
    mse_rot = np.mean((x - rec) ** 2)
    assert abs(mse_rot - g["rotated_mse"]) < 1e-3
    # the page's 69% is 1 - 0.073/0.237 on its printed MSEs; exact values give 69.6%
    assert int(100 * (1 - g["rotated_mse"] / g["mse"])) == g["mse_reduction_percent"]
    assert abs(100 * (1 - mse_rot / mse_plain) - g["mse_reduction_percent"]) < 1.0
    assert abs(np.max(np.abs(x - deq)) - g["max_abs_error_plain"]) < 1e-9
    assert abs(np.max(np.abs(x - rec)) - g["max_abs_error_rotated"]) < 5e-4
    qa = _golden("rotate_page_int4_examples.json")["qa_observations"]
    assert abs((x.max() - x.min()) - qa["range_plain"]) < 1e-9
    assert abs((xr.max() - xr.min()) - qa["range_rotated"]) < 1e-9
    assert abs(np.abs(xr).max() - qa["max_rotated"]) < 1e-12
    assert round(100 * (1 - qa["max_rotated"] / qa["max_plain"])) == qa["max_reduction_percent"]
    for name, bits, signed in (("int4", 4, True), ("uint4", 4, False), ("int8", 8, True)):
        s, _, _ = O.int_absmax_quantize([1.0], bits, signed)
        assert abs(1.0 / s - qa["signed_int_divisors"][name]) < 1e-12


# ---------------------------------------------------------------- [rot] sections 2.2, 3.1

def test_sylvester_matches_printed_matrices():
    g = _golden("rotate_page_hadamard.json")
    for n, key in ((1, "H1"), (2, "H2"), (4, "H4")):
        np.testing.assert_array_equal(O.sylvester_hadamard(n), np.array(g[key]))
    np.testing.assert_array_equal(O.sylvester_hadamard(4) / 2, np.array(g["H4_normalized"]))


@pytest.mark.parametrize("n", [2, 4, 8, 16, 32, 64, 128, 256])
def test_hadamard_closed_forms(n):
    H = O.sylvester_hadamard(n)
    np.testing.assert_array_equal(H, H.T)                      # symmetric
    np.testing.assert_array_equal(H @ H.T, n * np.eye(n))      # H H^T = n I
    assert set(np.unique(H)) == {-1.0, 1.0}


@pytest.mark.parametrize("n", [2, 4, 8, 16, 32, 64, 128])
def test_butterfly_equals_dense_and_is_involution(n):
    # Hadacore test pattern: fast transform == x @ H^T, twice == identity.
    rng = np.random.default_rng(n)
    x = rng.standard_normal((5, 3 * n))
    H = O.sylvester_hadamard(n)
    dense = (x.reshape(5, 3, n) @ H.T).reshape(5, 3 * n)
    fast = O.hadamard_butterfly(x, n, np.float64)
    np.testing.assert_allclose(fast, dense, rtol=0, atol=1e-12 * n)
    twice = O.rotate_rows_f64(O.rotate_rows_f64(x, n), n)
    np.testing.assert_allclose(twice, x, rtol=0, atol=1e-12)
    # fp32 butterfly stays within fp32 rounding of the exact transform.
    x32 = x.astype(np.float32)
    r32 = O.rotate_rows_fp32(x32, n).astype(np.float64)
    r64 = O.rotate_rows_f64(x32.astype(np.float64), n)
    assert np.max(np.abs(r32 - r64)) <= 1e-5 * max(1.0, np.abs(r64).max())


def test_rotation_identity_before_quantization():
    # [rot] 2.1: y = x W = (x R^T)(R W); checkpoint W is (N, K), so both sides
    # rotate rows.  Exact up to fp64 rounding.
    rng = np.random.default_rng(7)
    x = rng.standard_normal((6, 512))
    W = rng.standard_normal((9, 512))
    y = x @ W.T
    yr = O.rotate_rows_f64(x, 128) @ O.rotate_rows_f64(W, 128).T
    np.testing.assert_allclose(yr, y, rtol=0, atol=1e-12 * np.abs(y).max())


def test_rotation_preserves_norm_and_spreads_outlier():
    x = np.zeros((1, 128))
    x[0, 5] = 80.0
    xr = O.rotate_rows_f64(x, 128)
    np.testing.assert_allclose(np.abs(xr), 80.0 / np.sqrt(128), rtol=1e-15)
    assert abs(np.linalg.norm(xr) - 80.0) < 1e-12


# ---------------------------------------------------------------- number formats

def test_bf16_decode_matches_torch():
    bits = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16)
    ours = O.bf16_to_f32(bits)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).float().numpy()
    fin = np.isfinite(ref)
    np.testing.assert_array_equal(ours[fin], ref[fin])
    assert np.array_equal(np.isnan(ours), np.isnan(ref))


def test_e4m3_decode_matches_torch_all_bytes():
    b = np.arange(256, dtype=np.uint8)
    ours = O.e4m3_decode(b)
    ref = torch.from_numpy(b.copy()).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    fin = ~np.isnan(ref)
    np.testing.assert_array_equal(ours[fin], ref[fin])
    assert np.nanmax(ours) == 448.0 and O.e4m3_decode(np.uint8(1)) == 2.0 ** -9


def test_e4m3_encode_matches_torch_rne_in_range():
    rng = np.random.default_rng(3)
    v = np.concatenate([
        rng.uniform(0, 448, 20000), rng.uniform(0, 0.02, 20000),
        np.exp2(rng.uniform(-12, 8.8, 20000))]).astype(np.float32)
    # Exact midpoints between all consecutive finite codes.
    tab = O.e4m3_decode(np.arange(127, dtype=np.uint8))
    mids = ((tab[:-1] + tab[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (tab[:-1] + tab[1:]) / 2)  # exact in fp32
    v = np.concatenate([v, mids, -v[:1000]])
    ours = O.e4m3_encode_rne_satfinite(v)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ours, ref)


def test_e4m3_encode_saturates_and_roundtrips():
    assert O.e4m3_encode_rne_satfinite(np.float32(1e6)) == 0x7E
    assert O.e4m3_encode_rne_satfinite(np.float32(449.0)) == 0x7E
    assert O.e4m3_encode_rne_satfinite(np.float32(2.0 ** -10)) == 0       # tie -> even (0)
    assert O.e4m3_encode_rne_satfinite(np.float32(2.0 ** -10 * 1.0001)) == 1
    b = np.arange(127, dtype=np.uint8)
    np.testing.assert_array_equal(O.e4m3_encode_rne_satfinite(O.e4m3_decode(b)), b)
    np.testing.assert_array_equal(O.e4m3_encode_rne_satfinite(-O.e4m3_decode(b[1:])), b[1:] | 0x80)


def _e4m3_exact_nearest(fr: Fraction) -> int:
    """Independent brute force: nearest finite e4m3 code by exact rational distance."""
    best = None
    for c in range(127):
        val = Fraction(O.e4m3_decode(np.uint8(c)).item())
        d = abs(val - fr)
        key = (d, c & 1)          # ties: even mantissa first
        if best is None or key < best[0]:
            best = (key, c)
    return best[1]


def test_scale_rule_fp32_quotient_equals_exact_quotient():
    # s = e4m3(fp32(amax/6)) must equal e4m3 of the exact amax/6: the fp32
    # quotient can never cross an e4m3 rounding midpoint.  Brute force over
    # every midpoint of the finite e4m3 grid with amax a few fp32 ulps around 6*mid.
    tab = O.e4m3_decode(np.arange(127, dtype=np.uint8))
    mids = (tab[:-1] + tab[1:]) / 2
    checked = 0
    for mid in mids[::3]:
        centre = np.float32(6 * mid)
        cands = [centre]
        for _ in range(3):
            cands.append(np.nextafter(cands[-1], np.float32(np.inf)))
        c2 = [centre]
        for _ in range(3):
            c2.append(np.nextafter(c2[-1], np.float32(-np.inf)))
        for a in cands + c2[1:]:
            q32 = np.float32(a) / np.float32(6)
            got = int(O.e4m3_encode_rne_satfinite(q32))
            want = _e4m3_exact_nearest(Fraction(float(a)) / 6)
            assert got == want, (a, got, want)
            checked += 1
    assert checked > 100


def test_e2m1_table_and_ties():
    np.testing.assert_array_equal(O.e2m1_decode(np.arange(8)), [0, .5, 1, 1.5, 2, 3, 4, 6])
    np.testing.assert_array_equal(O.e2m1_decode(np.arange(8, 16)), [-0.0, -.5, -1, -1.5, -2, -3, -4, -6])
    ties = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for v, c in ties.items():
        assert O.e2m1_encode_rne_satfinite(np.float32(v)) == c
        assert O.e2m1_encode_rne_satfinite(np.float32(-v)) == c | 8
    assert O.e2m1_encode_rne_satfinite(np.float32(7.0)) == 7
    assert O.e2m1_encode_rne_satfinite(np.float32(1e30)) == 7
    assert O.e2m1_encode_rne_satfinite(np.float32(-0.1)) == 8      # sign kept at zero
    assert O.e2m1_encode_rne_satfinite(np.float32(0.26)) == 1


def test_e2m1_encode_against_exact_brute_force():
    rng = np.random.default_rng(11)
    v = np.concatenate([rng.uniform(-7, 7, 3000), rng.uniform(-0.3, 0.3, 500)]).astype(np.float32)
    grid = [Fraction(g) for g in (0, 0.5, 1, 1.5, 2, 3, 4, 6)]
    ours = O.e2m1_encode_rne_satfinite(v)
    for val, c in zip(v, ours):
        fr = abs(Fraction(float(val)))
        best = min(range(8), key=lambda i: (abs(grid[i] - fr), i & 1))
        want = best | (8 if val < 0 else 0)
        assert int(c) == want, (val, c, want)


def test_pack_nibble_order():
    codes = np.array([[1, 2, 3, 4]], dtype=np.uint8)
    packed = O.pack_e2m1(codes)
    np.testing.assert_array_equal(packed, [[0x21, 0x43]])
    np.testing.assert_array_equal(O.unpack_e2m1(packed), codes)


# ---------------------------------------------------------------- NVFP4 quantizer

def test_nvfp4_bruteforce_all_codes_all_scales():
    # Every positive finite e4m3 scale s and all 16 E2M1 codes: a block holding
    # code*s for each code (one entry is +6s so amax = 6s) must quantize back to
    # exactly those codes with scale byte s.
    codes = np.arange(16, dtype=np.uint8)
    vals = O.e2m1_decode(codes)
    blocks, want_s = [], []
    for sb in range(1, 127):
        s = O.e4m3_decode(np.uint8(sb)).item()
        blocks.append((vals * s).astype(np.float32))
        want_s.append(sb)
    v = np.stack(blocks)
    assert np.array_equal(v.astype(np.float64), np.stack([vals * O.e4m3_decode(np.uint8(b)).item() for b in want_s]))
    packed, sbytes = O.quantize_nvfp4_rows(v)
    np.testing.assert_array_equal(sbytes[:, 0], want_s)
    np.testing.assert_array_equal(O.unpack_e2m1(packed), np.tile(codes, (len(want_s), 1)))


def test_nvfp4_midpoints_go_to_even_code():
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    even = [0, 2, 2, 4, 4, 6, 6]
    for sb in (0x08, 0x30, 0x3B, 0x55, 0x01):
        s = O.e4m3_decode(np.uint8(sb)).item()
        row = np.zeros(16)
        row[:7] = mids * s
        row[7] = 6 * s
        row[8:15] = -mids * s
        packed, sbytes = O.quantize_nvfp4_rows(row[None, :].astype(np.float32))
        assert sbytes[0, 0] == sb
        c = O.unpack_e2m1(packed)[0]
        np.testing.assert_array_equal(c[:7], even)
        np.testing.assert_array_equal(c[8:15], np.array(even) | 8)


def test_nvfp4_zero_and_tiny_blocks():
    row = np.zeros((1, 32), np.float32)
    row[0, 16:] = -1e-4          # amax/6 below half the smallest subnormal scale
    packed, sb = O.quantize_nvfp4_rows(row)
    np.testing.assert_array_equal(sb, [[0, 0]])
    np.testing.assert_array_equal(packed, np.zeros((1, 16), np.uint8))


def test_nvfp4_saturation():
    row = np.zeros((1, 16), np.float32)
    row[0, 0] = 1e5              # amax/6 > 448 -> scale saturates at 448, code at 6
    row[0, 1] = 448.0 * 6
    row[0, 2] = -448.0
    packed, sb = O.quantize_nvfp4_rows(row)
    assert sb[0, 0] == 0x7E
    c = O.unpack_e2m1(packed)[0]
    assert c[0] == 7 and c[1] == 7 and c[2] == 0xA    # -448/448 = -1 -> code 2 with sign


def test_smoothing_power_of_two_shifts_scales():
    # x / smooth with smooth = 2 halves every x_hat exactly: codes unchanged,
    # every (normal-range) scale byte drops by one exponent step (8 codes).
    rng = np.random.default_rng(5)
    x = _bf16_bits(rng.standard_normal((4, 64)) * 3)
    c1, s1, _ = O.quantize_act(x, _bf16_bits(np.ones(64)), 0)
    c2, s2, _ = O.quantize_act(x, _bf16_bits(np.full(64, 2.0)), 0)
    np.testing.assert_array_equal(c1, c2)
    normal = (s1 >> 3) > 1
    np.testing.assert_array_equal(s2[normal].astype(int), s1[normal].astype(int) - 8)


# ---------------------------------------------------------------- full layer

def _hand_case():
    g = _golden("hand_case_k32.json")

    class C:
        pass

    ck = C()
    M, K, N, R = (g["shape"][k] for k in ("M", "K", "N", "R"))
    x = np.zeros((M, K))
    x[0, g["x_nonzero"]["k"]] = g["x_nonzero"]["value"]
    ck.x = _bf16_bits(x)
    ck.smooth_factor = _bf16_bits(np.ones(K))
    ck.qweight = np.zeros((N, K // 2), np.uint8)
    for e in g["qweight_nonzero_bytes"]:
        ck.qweight[e["n"], e["byte_index"]] = e["value"]
    ck.wscales = np.full((K // 16, N), O.e4m3_encode_rne_satfinite(np.float32(g["wscales_all"])), np.uint8)
    pd = np.zeros((K, R))
    pd[g["proj_down_nonzero"]["k"], g["proj_down_nonzero"]["r"]] = g["proj_down_nonzero"]["value"]
    ck.proj_down = _bf16_bits(pd)
    ck.proj_up = _bf16_bits(g["proj_up"])
    ck.wcscales = _bf16_bits(g["wcscales"])
    ck.wtscale = _bf16_bits([g["wtscale"]])
    ck.rotate_block = 0
    return g, ck


def test_hand_case_k32():
    g, ck = _hand_case()
    codes, scales, _ = O.quantize_act(ck.x, ck.smooth_factor, 0)
    np.testing.assert_array_equal(scales[0], g["act_scale_bytes"])
    assert codes[0, 8] == g["act_codes_byte8"]
    y = O.linear_forward(ck)
    np.testing.assert_array_equal(y[0], g["y"])


def _hand_case_smooth():
    g = _golden("hand_case_smooth_k32.json")

    class C:
        pass

    ck = C()
    M, K, N, R = (g["shape"][k] for k in ("M", "K", "N", "R"))
    x = np.zeros((M, K))
    for e in g["x_nonzero"]:
        x[0, e["k"]] = e["value"]
    ck.x = _bf16_bits(x)
    lam = np.ones(K)
    for e in g["smooth_factor_non_unit"]:
        lam[e["k"]] = e["value"]
    ck.smooth_factor = _bf16_bits(lam)
    ck.qweight = np.zeros((N, K // 2), np.uint8)
    for e in g["qweight_nonzero_bytes"]:
        ck.qweight[e["n"], e["byte_index"]] = e["value"]
    ck.wscales = np.full((K // 16, N), O.e4m3_encode_rne_satfinite(np.float32(g["wscales_all"])), np.uint8)
    pd = np.zeros((K, R))
    for e in g["proj_down_nonzero"]:
        pd[e["k"], e["r"]] = e["value"]
    ck.proj_down = _bf16_bits(pd)
    ck.proj_up = _bf16_bits(g["proj_up"])
    ck.wcscales = _bf16_bits(g["wcscales"])
    ck.wtscale = _bf16_bits([g["wtscale"]])
    ck.rotate_block = 0
    return g, ck


def test_hand_case_smooth_factor():
    # [svdq] Checkpoint contract (smooth_factor): x_hat = x / smooth_factor
    # feeds both the quantizer and the rank-R branch.  Every number in the
    # fixture is derived by hand; unsmoothed or multiplied inputs, or a rank-R
    # branch fed with x instead of x_hat, all change y.
    g, ck = _hand_case_smooth()
    codes, scales, xh = O.quantize_act(ck.x, ck.smooth_factor, 0)
    np.testing.assert_array_equal(scales[0], g["act_scale_bytes"])
    np.testing.assert_array_equal(codes[0], g["act_code_bytes"])
    np.testing.assert_array_equal(O.lowrank_down(xh, ck.proj_down)[0], g["lowrank"])
    y = O.linear_forward(ck)
    np.testing.assert_array_equal(y[0], g["y"])


def _grid_checkpoint(seed, M=3, K=64, N=5, R=4):
    """Activations whose every 16-block already lies on the NVFP4 grid (with a
    +-6s entry), smooth = 1, no rotation."""
    rng = np.random.default_rng(seed)
    x = np.zeros((M, K))
    for m in range(M):
        for b in range(K // 16):
            sb = rng.integers(0x20, 0x50)
            s = O.e4m3_decode(np.uint8(sb)).item()
            c = rng.integers(0, 16, 16)
            c[rng.integers(0, 16)] = 7 if rng.random() < 0.5 else 15
            x[m, b * 16:(b + 1) * 16] = O.e2m1_decode(c) * s

    class C:
        pass

    ck = C()
    ck.x = _bf16_bits(x)
    assert np.array_equal(O.bf16_to_f32(ck.x).astype(np.float64), x)      # representable
    ck.smooth_factor = _bf16_bits(np.ones(K))
    ck.qweight = rng.integers(0, 256, (N, K // 2)).astype(np.uint8)
    ck.wscales = O.e4m3_encode_rne_satfinite(rng.uniform(0.01, 0.1, (K // 16, N)).astype(np.float32))
    ck.proj_down = _bf16_bits(rng.standard_normal((K, R)) * 0.02)
    ck.proj_up = _bf16_bits(rng.standard_normal((N, R)) * 0.02)
    ck.wcscales = _bf16_bits(rng.uniform(0.8, 1.2, N))
    ck.wtscale = _bf16_bits([0.5])
    ck.rotate_block = 0
    return ck, x


def test_exact_recovery_on_grid():
    ck, x = _grid_checkpoint(1)
    codes, scales, xh = O.quantize_act(ck.x, ck.smooth_factor, 0)
    np.testing.assert_array_equal(O.dequantize_nvfp4(codes, scales), x)
    W = O.dequantize_weight(ck.qweight, ck.wscales)
    alpha = O.bf16_to_f32(ck.wcscales).astype(np.float64) * 0.5
    lr = (x @ O.bf16_to_f32(ck.proj_down).astype(np.float64)) @ O.bf16_to_f32(ck.proj_up).astype(np.float64).T
    y_exact = alpha * (x @ W.T) + lr
    np.testing.assert_allclose(O.linear_forward(ck), y_exact, rtol=1e-13, atol=1e-13)


def test_gemm_bruteforce_tiny():
    # Pure-Python loops over the contract (qweight nibbles, wscales[k//16, n]).
    ck, x = _grid_checkpoint(2, M=2, K=32, N=3, R=2)
    y = O.linear_forward(ck)
    pd = O.bf16_to_f32(ck.proj_down)
    pu = O.bf16_to_f32(ck.proj_up)
    wc = O.bf16_to_f32(ck.wcscales)
    for m in range(2):
        for n in range(3):
            acc = 0.0
            for k in range(32):
                byte = int(ck.qweight[n, k // 2])
                nib = (byte >> 4) if (k % 2) else (byte & 0xF)
                mag = [0, .5, 1, 1.5, 2, 3, 4, 6][nib & 7] * (-1 if nib & 8 else 1)
                acc += x[m, k] * mag * O.e4m3_decode(np.uint8(ck.wscales[k // 16, n])).item()
            lr = sum(sum(x[m, k] * float(pd[k, r]) for k in range(32)) * float(pu[n, r]) for r in range(2))
            want = float(wc[n]) * 0.5 * acc + lr
            assert abs(y[m, n] - want) <= 1e-12 * max(1.0, abs(want))


def test_special_cases():
    ck, x = _grid_checkpoint(3, M=4, K=64, N=6, R=3)
    y = O.linear_forward(ck)
    # qweight all zero -> y is the rank-R branch alone
    zero_q = np.zeros_like(ck.qweight)
    lr_only = O.linear_forward(ck, qweight=zero_q)
    lr = (x @ O.bf16_to_f32(ck.proj_down).astype(np.float64)) @ O.bf16_to_f32(ck.proj_up).astype(np.float64).T
    np.testing.assert_allclose(lr_only, lr, rtol=1e-14, atol=1e-14)
    # wtscale x2 doubles the main term only
    ck.wtscale = _bf16_bits([1.0])
    y2 = O.linear_forward(ck)
    np.testing.assert_allclose(y2 - lr, 2 * (y - lr), rtol=1e-13, atol=1e-13)
    # a single row equals that row of the batch
    np.testing.assert_allclose(O.linear_forward(ck, rows=[2])[0], y2[2], rtol=0, atol=0)


def test_rotated_weight_quantizer_roundtrip():
    # Offline W' = R W quantization: dequantized W' rotated back approximates W,
    # and an all-grid row survives unrotated quantization exactly.
    rng = np.random.default_rng(9)
    W = rng.standard_normal((4, 256)) * 0.02
    qw, ws = O.quantize_weight_nvfp4(_bf16_bits(W), 128)
    assert qw.shape == (4, 128) and ws.shape == (16, 4)
    Wq = O.dequantize_weight(qw, ws)
    back = O.rotate_rows_f64(Wq, 128)
    rel = np.linalg.norm(back - O.bf16_to_f32(_bf16_bits(W))) / np.linalg.norm(W)
    assert rel < 0.2          # 4-bit with coarse (subnormal) e4m3 scales


# ---------------------------------------------------------------- composition: smooth, then rotate, one x_hat for both branches

def _rotation_matrix(K, block):
    """Dense blockdiag(H_block / sqrt(block)) (K, K) from the Sylvester recursion."""
    H = O.sylvester_hadamard(block) / np.sqrt(block)
    R = np.zeros((K, K))
    for b in range(K // block):
        R[b * block:(b + 1) * block, b * block:(b + 1) * block] = H
    return R


@pytest.mark.parametrize("block", [4, 16])
def test_exact_recovery_with_smoothing_and_rotation(block):
    # [rot] 2.1 with [svdq] smooth_factor: pick the quantized target x_hat on
    # the NVFP4 grid (power-of-two scales, a +-6s entry per block), then build
    # the layer input that smoothing followed by rotation maps onto it:
    # x_hat = (x / lam) R^T  <=>  x = (x_hat R) * lam  (R symmetric, R R = I).
    # Blocks 4 and 16 normalise by 1/2 and 1/4, and lam holds powers of two,
    # so every step is exact and y must equal the closed form exactly.  Rotating
    # before smoothing, or feeding x (not x_hat) to the rank-R branch, breaks it.
    rng = np.random.default_rng(20 + block)
    M, K, N, R = 3, 64, 5, 4
    xh = np.zeros((M, K))
    for m in range(M):
        for b in range(K // 16):
            s = 2.0 ** int(rng.integers(-3, 3))
            c = rng.integers(0, 16, 16)
            c[rng.integers(0, 16)] = 7 if rng.random() < 0.5 else 15
            xh[m, b * 16:(b + 1) * 16] = O.e2m1_decode(c) * s
    lam = 2.0 ** rng.integers(-1, 3, K).astype(np.float64)
    Rm = _rotation_matrix(K, block)
    x = (xh @ Rm) * lam[None, :]

    class C:
        pass

    ck = C()
    ck.x = _bf16_bits(x)
    assert np.array_equal(O.bf16_to_f32(ck.x).astype(np.float64), x)        # representable
    ck.smooth_factor = _bf16_bits(lam)
    ck.qweight = rng.integers(0, 256, (N, K // 2)).astype(np.uint8)
    ck.wscales = O.e4m3_encode_rne_satfinite(rng.uniform(0.01, 0.1, (K // 16, N)).astype(np.float32))
    ck.proj_down = _bf16_bits(rng.standard_normal((K, R)) * 0.02)
    ck.proj_up = _bf16_bits(rng.standard_normal((N, R)) * 0.02)
    ck.wcscales = _bf16_bits(rng.uniform(0.8, 1.2, N))
    ck.wtscale = _bf16_bits([0.5])
    ck.rotate_block = block
    codes, scales, xh_o = O.quantize_act(ck.x, ck.smooth_factor, block)
    np.testing.assert_array_equal(xh_o.astype(np.float64), xh)
    np.testing.assert_array_equal(O.dequantize_nvfp4(codes, scales), xh)
    W = O.dequantize_weight(ck.qweight, ck.wscales)
    alpha = O.bf16_to_f32(ck.wcscales).astype(np.float64) * 0.5
    pd = O.bf16_to_f32(ck.proj_down).astype(np.float64)
    pu = O.bf16_to_f32(ck.proj_up).astype(np.float64)
    y_exact = alpha * (xh @ W.T) + (xh @ pd) @ pu.T
    np.testing.assert_allclose(O.linear_forward(ck), y_exact, rtol=1e-13, atol=1e-13)


def _random_layer_input(rng, M, K):
    x = rng.standard_normal((M, K)) * 2.0
    x[:, rng.choice(K, 3, replace=False)] *= 30.0
    lam = rng.uniform(0.5, 2.0, K)
    return _bf16_bits(x), _bf16_bits(lam)


def test_rotation_identity_through_rank_r_branch():
    # [rot] 2.1: (x R^T)(R P) = x P.  With every weight code zero, y is the
    # rank-R branch alone, so the 128-block rotated layer with proj_down' =
    # bf16(R proj_down) must give the unrotated layer's y.  The two differ only
    # by the bf16 rounding of proj_down' (2^-9 relative per entry) and the fp32
    # rounding of x_hat (at most a few 2^-24 relative per butterfly stage);
    # the bound below is that, entry by entry.  Rotating before smoothing, or
    # a rank-R branch fed with x, misses it by orders of magnitude.
    rng = np.random.default_rng(41)
    M, K, N, R = 4, 256, 6, 3
    x_bits, lam_bits = _random_layer_input(rng, M, K)
    pd = O.bf16_to_f32(_bf16_bits(rng.standard_normal((K, R)) * 0.02)).astype(np.float64)
    Rm = _rotation_matrix(K, 128)
    pd_rot_bits = _bf16_bits(Rm @ pd)

    class C:
        pass

    def layer(block, pd_bits):
        ck = C()
        ck.x, ck.smooth_factor = x_bits, lam_bits
        ck.qweight = np.zeros((N, K // 2), np.uint8)
        ck.wscales = O.e4m3_encode_rne_satfinite(np.full((K // 16, N), 0.05, np.float32))
        ck.proj_down = pd_bits
        ck.proj_up = _bf16_bits(rng_pu)
        ck.wcscales = _bf16_bits(np.ones(N))
        ck.wtscale = _bf16_bits([1.0])
        ck.rotate_block = block
        return O.linear_forward(ck)

    rng_pu = rng.standard_normal((N, R)) * 0.02
    y_plain = layer(0, _bf16_bits(pd))
    y_rot = layer(128, pd_rot_bits)
    xs = np.abs(O.bf16_to_f32(x_bits).astype(np.float64) / O.bf16_to_f32(lam_bits).astype(np.float64))
    rpd = Rm @ pd
    pu = np.abs(O.bf16_to_f32(_bf16_bits(rng_pu)).astype(np.float64))
    xh_rot = np.abs(O.smooth_and_rotate(x_bits, lam_bits, 128).astype(np.float64))
    xr = xs @ np.abs(Rm)                             # l1 bound on a rotated entry's partial sums
    bound_L = xh_rot @ (2.0 ** -9 * np.abs(rpd)) + 16 * 2.0 ** -24 * (xr @ np.abs(rpd) + xs @ np.abs(pd))
    bound = bound_L @ pu.T
    assert np.all(np.abs(y_rot - y_plain) <= bound), np.max(np.abs(y_rot - y_plain) / bound)
    assert np.max(np.abs(y_plain)) > 10 * np.max(bound)      # the check is not vacuous


def test_rotation_identity_through_main_product_dense():
    # [rot] 2.1 on the main product before quantization: with W' = W R^T (the
    # checkpoint's (N, K) rows rotated), x_hat_rot W'^T = x_hat W^T, where
    # x_hat_rot is the oracle's smoothed-then-rotated activation.  Exact up to
    # the fp32 rounding of x_hat; smoothing after rotating misses it.
    rng = np.random.default_rng(43)
    M, K, N = 5, 384, 7
    x_bits, lam_bits = _random_layer_input(rng, M, K)
    W = rng.standard_normal((N, K))
    xh0 = O.smooth_and_rotate(x_bits, lam_bits, 0).astype(np.float64)
    xh1 = O.smooth_and_rotate(x_bits, lam_bits, 128).astype(np.float64)
    Wr = O.rotate_rows_f64(W, 128)
    y0 = xh0 @ W.T
    y1 = xh1 @ Wr.T
    scale = np.abs(xh0) @ np.abs(W).T
    assert np.all(np.abs(y1 - y0) <= 2.0 ** -19 * scale + 1e-12)
    # the exact real x_hat R^T agrees with the fp32 one to fp32 rounding
    np.testing.assert_allclose(xh1, O.rotate_rows_f64(xh0, 128), rtol=0, atol=2.0 ** -20 * np.abs(xh0).max())


# ---------------------------------------------------------------- [rot] section 3.1: the standalone transform

def test_f32_to_bf16_matches_torch():
    # The library conversion (round to nearest even) on random values, ties,
    # subnormals, the largest finite values and infinities.
    rng = np.random.default_rng(11)
    v = rng.standard_normal(20000).astype(np.float32) * np.float32(3.0) ** rng.integers(-40, 40, 20000)
    ties = (np.arange(1, 2000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    special = np.array([0.0, -0.0, 1e-40, -1e-40, 3.4e38, -3.4e38, np.inf, -np.inf], dtype=np.float32)
    allv = np.concatenate([v, ties, -ties, special]).astype(np.float32)
    ref = torch.from_numpy(allv).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(O.f32_to_bf16_bits(allv), ref)
    nanbits = O.f32_to_bf16_bits(np.array([np.nan], dtype=np.float32))
    assert (nanbits[0] & 0x7F80) == 0x7F80 and (nanbits[0] & 0x7F) != 0


@pytest.mark.parametrize("n", [1, 2, 8, 64, 512, 2048])
def test_hadamard_transform_equals_dense(n):
    # Hadacore's check (section 3.1): the transform equals x @ H^T (normalised),
    # here within fp32 accumulation error plus one bf16 rounding.
    rng = np.random.default_rng(n + 1)
    x = rng.standard_normal((3, n)).astype(np.float32)
    xb = O.f32_to_bf16_bits(x)
    y = O.bf16_to_f32(O.hadamard_transform(xb, n)).astype(np.float64)
    H = O.sylvester_hadamard(n) / np.sqrt(n)
    dense = O.bf16_to_f32(xb).astype(np.float64) @ H.T
    tol = 2.0 ** -8 * np.abs(dense) + 1e-6 * np.sqrt(n) * np.abs(dense).max()
    assert np.all(np.abs(y - dense) <= tol)


@pytest.mark.parametrize("n,dtype", [(16, "bf16"), (4096, "bf16"), (32768, "bf16"), (1024, "fp16")])
def test_hadamard_transform_involution_and_norm(n, dtype):
    # Applying the transform twice returns x up to the two roundings to the
    # storage type; one application preserves the row norm (H / sqrt(n) is
    # orthogonal); large n agrees with the exact fp64 butterfly.
    rng = np.random.default_rng(n)
    x = rng.standard_normal((2, n)).astype(np.float32)
    xb = O.f32_to_bf16_bits(x) if dtype == "bf16" else x.astype(np.float16).view(np.uint16)
    dec = (lambda b: O.bf16_to_f32(b)) if dtype == "bf16" else (lambda b: b.view(np.float16).astype(np.float32))
    x0 = dec(xb).astype(np.float64)
    y = O.hadamard_transform(xb, n, dtype)
    yy = dec(y).astype(np.float64)
    exact = O.rotate_rows_f64(x0, n)
    eps = 2.0 ** -8 if dtype == "bf16" else 2.0 ** -11
    assert np.max(np.abs(yy - exact)) <= eps * np.abs(exact).max() + 1e-5 * np.abs(exact).max()
    np.testing.assert_allclose(np.linalg.norm(yy, axis=1), np.linalg.norm(x0, axis=1), rtol=4 * eps)
    back = dec(O.hadamard_transform(y, n, dtype)).astype(np.float64)
    assert np.max(np.abs(back - x0)) <= 4 * eps * np.abs(x0).max()


# ---------------------------------------------------------------- [rot] section 3.3: MXFP4 with a grouped Hadamard (FP-Quant)

def test_e8m0_decode_matches_torch_all_bytes():
    b = np.arange(256, dtype=np.uint8)
    ours = O.e8m0_decode(b)
    ref = torch.from_numpy(b.copy()).view(torch.float8_e8m0fnu).float().numpy().astype(np.float64)
    assert np.isnan(ours[255]) and np.isnan(ref[255])
    np.testing.assert_array_equal(ours[:255][ref[:255] > 0], ref[:255][ref[:255] > 0])
    assert ours[127] == 1.0 and ours[0] == 2.0 ** -127 and ours[254] == 2.0 ** 127


def test_mx_abs_max_exponent_exact_boundaries():
    # The smallest power of two s with amax / s <= 6, checked by exact rational
    # arithmetic at every boundary amax = 6 * 2^e and one fp32 ulp either side.
    def brute(a: Fraction) -> int:
        e = -200
        while Fraction(6) * Fraction(2) ** e < a:
            e += 1
        return max(-127, min(127, e))
    checked = 0
    for e in range(-126, 126):
        c = np.float32(6.0 * 2.0 ** e)
        for a in (c, np.nextafter(c, np.float32(np.inf)), np.nextafter(c, np.float32(0))):
            got = int(O.mx_abs_max_exponent(np.array([float(a)]))[0])
            assert got == brute(Fraction(float(a))), (e, a, got)
            checked += 1
    rng = np.random.default_rng(17)
    for a in np.exp2(rng.uniform(-140, 128, 300)).astype(np.float32):
        if not np.isfinite(a) or a == 0:
            continue
        assert int(O.mx_abs_max_exponent(np.array([float(a)]))[0]) == brute(Fraction(float(a)))
        checked += 1
    assert checked > 900
    assert O.mx_abs_max_exponent(np.array([0.0]))[0] == -127


def test_mxfp4_bruteforce_all_codes_all_scales():
    # Every E8M0 scale whose 6 * s is a finite fp32 value, all 16 E2M1 codes:
    # a block holding code * s (with +6s, so amax = 6s) quantizes back to those
    # codes with scale byte log2(s) + 127.
    codes = np.arange(16, dtype=np.uint8)
    vals = O.e2m1_decode(np.concatenate([codes, codes]))            # 32 elements per block
    blocks, want = [], []
    for e in range(-127, 126):
        blocks.append((vals * 2.0 ** e).astype(np.float32))
        want.append(e + 127)
    v = np.stack(blocks)
    assert np.array_equal(v.astype(np.float64), np.stack([vals * 2.0 ** (b - 127) for b in want]))
    packed, sb = O.quantize_mxfp4_rows(v)
    np.testing.assert_array_equal(sb[:, 0], want)
    np.testing.assert_array_equal(O.unpack_e2m1(packed), np.tile(np.concatenate([codes, codes]), (len(want), 1)))
    np.testing.assert_array_equal(O.dequantize_mxfp4(packed, sb), v.astype(np.float64))


def test_mxfp4_ties_zero_nan_inf_blocks():
    s = 2.0 ** -3
    row = np.zeros((4, 32), np.float32)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    row[0, :7] = mids * s
    row[0, 7] = 6 * s
    row[0, 8:15] = -mids * s
    row[1, 3] = np.nan
    row[2, 5] = np.inf
    row[2, 6] = 1.0
    # row 3 stays zero
    packed, sb = O.quantize_mxfp4_rows(row)
    c = O.unpack_e2m1(packed)
    np.testing.assert_array_equal(c[0, :7], [0, 2, 2, 4, 4, 6, 6])
    np.testing.assert_array_equal(c[0, 8:15], np.array([0, 2, 2, 4, 4, 6, 6]) | 8)
    assert sb[0, 0] == 127 - 3
    assert sb[1, 0] == 255 and not c[1].any()                       # NaN block: NaN scale, zero codes
    assert sb[2, 0] == 254 and c[2, 5] == 7 and c[2, 6] == 0         # inf saturates, the rest underflows
    assert sb[3, 0] == 0 and not c[3].any()                         # zero block: smallest scale


@pytest.mark.parametrize("group", [0, 32])
def test_fpquant_exact_recovery_and_rotation_identity(group):
    # group 0: activations and weights already on the MXFP4 grid quantize
    # exactly, so y equals alpha * x W^T in fp64.  group 32: before
    # quantization the grouped rotation leaves the product unchanged,
    # (x R^T)(W R^T)^T = x W^T ([rot] 2.1), here through the oracle's fp32
    # rotation of both operands.
    rng = np.random.default_rng(61 + group)
    M, K, N = 3, 128, 5

    def grid(rows):
        out = np.zeros((rows, K))
        for r in range(rows):
            for b in range(K // 32):
                c = rng.integers(0, 16, 32)
                c[rng.integers(0, 32)] = 7
                out[r, 32 * b:32 * (b + 1)] = O.e2m1_decode(c) * 2.0 ** int(rng.integers(-4, 4))
        return out
    if group == 0:
        x, W = grid(M), grid(N)
        qw, ws = O.fpquant_quantize_weight(_bf16_bits(W), 0)
        y = O.fpquant_forward(_bf16_bits(x), qw, ws, 0.75, 0)
        np.testing.assert_array_equal(y, 0.75 * (x @ W.T))
    else:
        x = rng.standard_normal((M, K))
        W = rng.standard_normal((N, K))
        xb, Wb = _bf16_bits(x), _bf16_bits(W)
        _, _, xh = O.fpquant_quantize(xb, 32)
        _, _, wh = O.fpquant_quantize(Wb, 32)
        ref = O.bf16_to_f32(xb).astype(np.float64) @ O.bf16_to_f32(Wb).astype(np.float64).T
        got = xh.astype(np.float64) @ wh.astype(np.float64).T
        assert np.all(np.abs(got - ref) <= 2.0 ** -18 * np.abs(x).sum(1)[:, None] * np.abs(W).max())
        # the fp32 grouped rotation is the dense H_32 / sqrt(32) up to fp32 rounding
        H = O.sylvester_hadamard(32) / np.sqrt(32)
        dense = (O.bf16_to_f32(xb).astype(np.float64).reshape(M, K // 32, 32) @ H.T).reshape(M, K)
        np.testing.assert_allclose(xh, dense, rtol=0, atol=1e-6 * np.abs(dense).max())

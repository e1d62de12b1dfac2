"""The quantizer divides without the divide unit: with y = RN(1/b) it computes
q0 = RN(a*y), r = RN(a - b*q0) (fused), q1 = RN(q0 + r*y) (fused).  This test
compiles a small C program and checks, exhaustively over every significand
pair that occurs in the kernel (bf16 / bf16 for x / smooth_factor, fp32 /
e4m3-significand for x_hat / scale and amax / 6), that q1 equals the IEEE
correctly rounded quotient.  It checks the numerical method, not the kernel."""
import os
import shutil
import subprocess

import pytest

SRC = os.path.join(os.path.dirname(__file__), "native", "division_check.c")


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    out = str(tmp_path_factory.mktemp("div") / "division_check")
    flags = ["-O2", "-ffp-contract=off"]
    # Hardware FMA where available (glibc's fmaf is correctly rounded either
    # way) and OpenMP threads for the exhaustive all-operand mode.
    for extra in (["-mfma", "-fopenmp"], ["-mfma"], ["-fopenmp"], []):
        try:
            subprocess.run([cc, *flags, *extra, SRC, "-o", out, "-lm"], check=True, capture_output=True)
            return out
        except subprocess.CalledProcessError:
            continue
    pytest.fail("could not compile " + SRC)


@pytest.mark.parametrize("mode,count", [("bf16", 32768), ("e4m3", 67108864)])
def test_markstein_division_exact(exe, mode, count):
    r = subprocess.run([exe, mode], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip() == f"checked {count} mismatches 0"


def test_smoothing_division_all_bf16_operands(exe):
    # Every finite bf16 x (zeros and subnormals too) over every smoothing factor
    # 2^-100 <= |s| < 2^128, both sign layouts: the quotient equals RN(x / s)
    # except where |RN(x / s)| < 2^-19, where it may be one ulp off with the
    # same sign -- a value that quantizes to code +-0 (and, as a block's
    # largest magnitude, to scale 0) whatever the scale, so codes and scales
    # stay exact.
    r = subprocess.run([exe, "bf16all"], capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("checked 3810263040 mismatches 0 "), r.stdout


def test_two_op_division_all_bf16_operands(exe):
    # The activation quantizer's division RN(x*yh + RN(x*yl)) (yh = RZ(1/s),
    # yl = RN(1/s - yh) with yh's sign) over every finite bf16 x and every
    # normal bf16 smoothing factor of magnitude in [2^-126, 2^117), both signs
    # (the magnitudes create accepts): equal to the IEEE quotient except one ulp
    # below 2^-19 with the same sign, which leaves codes and scales unchanged.
    r = subprocess.run([exe, "rr_bf16all"], capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout + r.stderr
    assert " mismatches 0 " in r.stdout, r.stdout


def test_two_op_division_fp32_over_e4m3_significands(exe):
    # x_hat / scale and amax / 6 with the same two-op division: every fp32
    # significand (both signs) over the eight e4m3 significands, exact.
    r = subprocess.run([exe, "rr_e4m3"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip() == "checked 134217728 mismatches 0"

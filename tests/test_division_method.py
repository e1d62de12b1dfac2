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
    # Hardware FMA where available; glibc's fmaf is correctly rounded either way.
    try:
        subprocess.run([cc, *flags, "-mfma", SRC, "-o", out, "-lm"], check=True, capture_output=True)
    except subprocess.CalledProcessError:
        subprocess.run([cc, *flags, SRC, "-o", out, "-lm"], check=True)
    return out


@pytest.mark.parametrize("mode,count", [("bf16", 32768), ("e4m3", 67108864)])
def test_markstein_division_exact(exe, mode, count):
    r = subprocess.run([exe, mode], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip() == f"checked {count} mismatches 0"

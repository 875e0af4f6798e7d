"""The quantizer kernels' division method, checked exhaustively on the CPU.

Every E4M3 code is the saturating round-to-nearest-even conversion of the IEEE
binary32 quotient fl32(x / scale), scale = fl32(amax / 448) (page
"ProCreations/Nanbeige4.3-33B-FP8", introduction: dynamic per-token/group-128
activation scales; the same rule for the 128x128 weight blocks).  The kernels
form both quotients from a correctly rounded reciprocal and one fused
multiply-add correction instead of a division.  `c/quotient_method.c` restates
that method in plain C and compares it with the C library's IEEE division over
its whole input domain: every positive finite BF16 amax, and every BF16 x with
|x| <= amax, both signs (about 1.03e9 pairs).  The GPU test
test_gpu_quotient.py runs the kernels themselves over the same domain.
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_corrected_quotient_equals_ieee_division(tmp_path):
    exe = tmp_path / "quotient_method"
    subprocess.run(["gcc", "-O2", "-std=c99", "-ffp-contract=off", "-fopenmp",
                    os.path.join(HERE, "c", "quotient_method.c"), "-o", str(exe), "-lm"],
                   check=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "0 differ" in res.stdout and "0 bit differences" in res.stdout

"""The NVFP4 encoder computes amax / 6 as a reciprocal product with one fused correction step
instead of a division (see div6_rn in the CUDA sources). Block scales must match the oracle
bit for bit, so the identity is checked here for every finite fp32 input the fast path takes."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_div6_fast_path_is_correctly_rounded(tmp_path):
    exe = str(tmp_path / "div6_check")
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-o", exe, os.path.join(HERE, "div6_check.c"), "-lm"])
    out = subprocess.run([exe], capture_output=True, text=True, check=True, timeout=600).stdout.split()
    checked, bad = int(out[0]), int(out[1])
    assert checked == 0x7F7FFFFF - 0x01000000 + 1   # all finite floats from 2^-125 up
    assert bad == 0

"""The quantizers replace x / s by a reciprocal and one Markstein correction
step (see blockwise_scaled_fp8_fp8bw_b200/csrc/quant.cu).  This CPU test
proves, exhaustively over all bf16 inputs a block can hold, that the scheme
yields the same E4M3 (and E5M2) code as IEEE division (host restatement in
C; IEEE binary32 with fused multiply-add behaves identically on the GPU
without flush-to-zero)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


import pytest


@pytest.mark.parametrize("qmax", ["448", "57344"])   # E4M3, E5M2
def test_markstein_step_matches_ieee_division(tmp_path, qmax):
    exe = str(tmp_path / "division_scheme_check")
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-march=x86-64-v3",
                           os.path.join(HERE, "c", "division_scheme_check.c"), "-o", exe, "-lm"])
    out = subprocess.run([exe, qmax], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "bad 0 badsign 0" in out.stdout
    n = int(out.stdout.split()[1])
    assert n > 10 ** 9

"""The two fp32 identities the CUDA quantisers use instead of a division
subroutine and a rounding instruction (kv4_append.cu: div_by_const and
biased_code2), checked on the host with IEEE fmaf: the corrected division by
7 and 127 against IEEE division, and the snapped nearest-even rounding of
x/s against rint for bf16 x, fp16 s and reciprocals up to 4 ulps off.
Every bf16 numerator and every 7th fp16 scale here; stride 1 of the same
program is the exhaustive run."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_quantiser_arithmetic_identities(tmp_path):
    exe = str(tmp_path / "quantiser_arithmetic")
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-o", exe,
                           os.path.join(HERE, "c", "quantiser_arithmetic.c"), "-lm"])
    r = subprocess.run([exe, "7"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "0 mismatches\nrounding" in r.stdout and r.stdout.rstrip().endswith("0 mismatches"), r.stdout

"""The group-quantisation kernel divides by an E4M3 scale (and the scale's
span by 3) with one multiply by the correctly rounded reciprocal and one
fused-multiply-add correction (Markstein's method) instead of an IEEE
divide.  tests/fast_division_check.c proves on the host, in IEEE fp32 with
fused multiply-add, that this gives the IEEE quotient for every E4M3
significand and every a with a normal quotient (one binade of quotients by
default; every fp32 bit pattern with the argument "all")."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def test_markstein_quotient_equals_ieee_divide(tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    exe = tmp_path / "fdc"
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-fopenmp", os.path.join(HERE, "fast_division_check.c"),
                    "-o", str(exe), "-lm"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.startswith("ok"), out.stdout

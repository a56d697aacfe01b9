"""The row quantisers form the scale fl(m / 127) from RN(1/127) and two fused
multiply-adds (Markstein's correction) instead of a division instruction.
That is exact only if it equals IEEE division for every input the kernels
can see: m is a row maximum clamped at 1e-8, so every fp32 value from 1e-8 up
to the largest finite one.  tests/c/div_by_127.c checks all of them (about
1.3e9 values, seconds in C)."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_markstein_division_by_127_is_exact_for_every_fp32(tmp_path):
    exe = tmp_path / "div_by_127"
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-o", str(exe), os.path.join(HERE, "c", "div_by_127.c"),
                    "-lm"], check=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "0 differences" in res.stdout

"""The exact division the kernels use for a group's scale: a / 7 (int4) and
a / 127 (int8) as a multiply by the rounded reciprocal plus one fma residual
correction.  The kernels rely on it being equal to the IEEE quotient; this
checks that identity on the host for every non-negative finite float (the
reciprocal constants are the ones the kernels use)."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_const_division_exhaustive(tmp_path):
    exe = tmp_path / "const_division"
    subprocess.run(["gcc", "-O2", "-march=native", "-ffp-contract=off", "-fopenmp", "-o", str(exe),
                    os.path.join(HERE, "const_division.c"), "-lm"], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True,
                         timeout=600).stdout.split()
    got = dict(zip(out[0::2], map(int, out[1::2])))
    assert got == {"7": 0, "127": 0}

"""The pack kernel derives the fp32 quotients of its fp16 path without a
division (Markstein's correction on a faithful first quotient).  This checks
that arithmetic, restated in plain C, against the host's IEEE division:
exhaustively for the group scale RN((max - min) / (2^b - 1)) over every fp32
difference of fp16 values, and over every fp16 value of sampled ranges
(including ranges that put t / s exactly on half-integers) for the codes'
quotient RN((x - min) / s).  The GPU parity tests then compare the kernel's
codes with the oracle byte for byte."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_division_free_quotients_match_ieee_division(tmp_path):
    exe = tmp_path / "quotient_check"
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-o", str(exe),
                    os.path.join(HERE, "quotient", "quotient_check.c"), "-lm"], check=True)
    r = subprocess.run([str(exe), "1500"], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "mismatches 0" in r.stdout and "exact half-integer quotients 0," not in r.stdout, r.stdout

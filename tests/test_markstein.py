"""The quantizer's division shortcut equals IEEE division for every 16-bit
input significand and every binary32 divisor significand (exhaustive, CPU)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def test_markstein_exhaustive(tmp_path):
    exe = str(tmp_path / "markstein_check")
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-o", exe,
                           os.path.join(HERE, "markstein_check.c"), "-lm"])
    out = subprocess.run([exe], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout
    assert "checked 8589934592 pairs, 0 mismatches" in out.stdout

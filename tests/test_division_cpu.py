"""The codec's shared-divisor division (Markstein's correction after a
correctly rounded reciprocal) must reproduce IEEE division bit for bit; the
4-bit codes depend on it.  Checked on the host CPU with a C program that
performs the same sequence of fp32 operations with a hardware FMA."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("cc") is None and shutil.which("gcc") is None, reason="no C compiler")
def test_shared_divisor_division_equals_ieee(tmp_path):
    cc = shutil.which("cc") or shutil.which("gcc")
    exe = tmp_path / "div"
    src = os.path.join(HERE, "native", "shared_divisor_check.c")
    flags = ["-O2", "-ffp-contract=off"]
    probe = subprocess.run([cc, "-mfma", "-x", "c", "-", "-o", os.devnull, "-c"], input="int x;",
                           capture_output=True, text=True)
    if probe.returncode == 0:
        flags.append("-mfma")
    subprocess.run([cc, *flags, src, "-o", str(exe), "-lm"], check=True)
    r = subprocess.run([str(exe), "20000000"], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "mismatches 0" in r.stdout

"""The kernels' division-free block scale s = a / 448 (one multiply by
RN(1/448) and an FMA correction) equals IEEE division for every float a from
the eps floor to FLT_MAX: tests/c/div448_check.c, compiled without
floating-point contraction and run over all 1.35e9 dividends (about 10 s)."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_division_by_448_is_correctly_rounded_for_every_block_absmax(tmp_path):
    exe = tmp_path / "div448_check"
    subprocess.run(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                    os.path.join(HERE, "c", "div448_check.c"), "-o", str(exe), "-lm"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "1352931585 dividends, all correctly rounded" in r.stdout, r.stdout

"""Host logic of the CTA-pair GEMM's tile order: the dense enumeration of the tiles that touch the
upper triangle (csrc/tile_upper.h), checked exhaustively on CPU for up to 100 x 100 tiles and group
heights 8 and 16 (compiled with the host C++ compiler)."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "post_weight_quantization_17_b200", "csrc")


@pytest.mark.skipif(shutil.which("g++") is None, reason="no host C++ compiler")
def test_upper_tile_enumeration(tmp_path):
    exe = tmp_path / "tile_upper_check"
    subprocess.run(["g++", "-O2", "-std=c++17", "-I", CSRC, "-o", str(exe),
                    os.path.join(HERE, "tile_upper_check.cpp")], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "bad=0" in out.stdout

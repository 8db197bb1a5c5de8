"""bench.py's CPU legs: the reference arm (the oracle on a bounded sample) prints the contract's
JSON line, for static and dynamic groups; the W4A16 line's CPU sample extrapolates by rows."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("grid", ["static", "dynamic"])
def test_reference_arm_line(grid):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--scale", "0.0625", "--grid", grid],
                       capture_output=True, text=True, timeout=600, cwd=ROOT,
                       env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "weights/s"
    assert line["higher_is_better"] is True and line["steps"] == 1
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["config"]["grid"] == grid


def test_w4a16_cpu_sample_extrapolates_by_rows():
    sys.path.insert(0, ROOT)
    import bench
    s, full, desc = bench.oracle_w4a16_sample(1024, 512, 4, 64)
    assert 0 < s and full == pytest.approx(s * 1024 / 64)
    assert "64 of 1024 rows" in desc

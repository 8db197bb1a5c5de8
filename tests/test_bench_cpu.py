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


def test_gpus_n_without_launcher_starts_its_own_ranks(monkeypatch):
    """--gpus N > 1 outside torchrun re-launches bench.py under torch.distributed.run with N
    processes on this node (rendezvous on 127.0.0.1) and the same arguments."""
    sys.path.insert(0, ROOT)
    import bench
    seen = {}

    def fake_call(cmd, cwd=None):
        seen["cmd"], seen["cwd"] = cmd, cwd
        return 0

    monkeypatch.setattr(bench.subprocess, "call", fake_call)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--gpus", "4", "--steps", "2", "--warmup", "3"])
    with pytest.raises(SystemExit) as e:
        bench.main()
    assert e.value.code == 0
    cmd = seen["cmd"]
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--master-addr=127.0.0.1" in cmd
    assert cmd[-6:] == ["--gpus", "4", "--steps", "2", "--warmup", "3"]
    assert cmd[-7].endswith("bench.py")


def test_workload_configs():
    sys.path.insert(0, ROOT)
    import bench
    g5 = bench.workload(5)
    assert len(g5) == 1 and g5[0].mats[0].m == 12288 and g5[0].x_spec.chunk == 8192
    assert bench.weights_per_step(g5) == 12288 * 49152
    assert bench.workload(5, bits=2)[0].mats[0].bits == 2
    g4 = bench.workload(4)
    assert [len(g.mats) for g in g4] == [3, 1, 2, 1]
    assert bench.weights_per_step(g4) == 4 * 4096 * 4096 + 2 * 11008 * 4096 + 4096 * 11008
    assert all(g.x_spec.chunk == g.x_spec.n_tokens for g in g4)   # one call over all tokens
    assert bench.baseline_cols(49152, 65536) == 2048 and bench.baseline_cols(100, 512) == 100


def test_peak_regime_and_stage_peaks():
    """The roofline peaks follow the regime of the timed steps: sustained when the power cap held
    the median SM clock below 90 % of its maximum, burst otherwise (or without clock samples)."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench.peak_regime({"sm_mhz": 1425.0, "sm_max_mhz": 1965.0}) == "sustained"
    assert bench.peak_regime({"sm_mhz": 1965.0, "sm_max_mhz": 1965.0}) == "burst"
    assert bench.peak_regime({"sm_mhz": 1800.0, "sm_max_mhz": 1965.0}) == "burst"
    assert bench.peak_regime(None) == "burst"
    peaks = {"bf16": 1672.7, "bf16_sustained": 1410.6, "hbm": 6544.3, "source": "measured"}
    g5 = bench.workload(5)
    st = {"hessian": 140.0, "prepare": 470.0}
    sus = bench.stage_rooflines(g5, st, None, peaks, 600.0, "sustained")
    bur = bench.stage_rooflines(g5, st, None, peaks, 750.0, "burst")
    assert sus["a1_hessian"]["peak"] == 1410.6 and bur["a1_hessian"]["peak"] == 1672.7
    assert sus["a3_factor"]["peak"] == pytest.approx(200.0)      # TF32 / 3
    assert bur["a3_factor"]["peak"] == pytest.approx(250.0)
    f = 158332895625216.0    # N d (d + 1) for the fc2 layer: 65536 x 49152 x 49153
    assert sus["a1_hessian"]["work"] == f
    assert sus["a1_hessian"]["achieved"] == pytest.approx(f / 0.140 / 1e12)

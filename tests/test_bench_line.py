"""The benchmark's JSON line: the reference arm (the oracle, on CPU) and the
library arm (on a GPU) each print one line with the keys the harness reads."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BASE_KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
             "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"}


def _run(*args, timeout):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                       capture_output=True, text=True, timeout=timeout)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    return json.loads(lines[0])


def test_reference_arm_line():
    line = _run("--impl", "reference", "--steps", "1", "--warmup", "3", timeout=600)
    assert BASE_KEYS <= set(line)
    assert line["impl"] == "reference"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["value"] > 0


@pytest.mark.gpu
def test_library_arm_line():
    line = _run("--steps", "3", "--warmup", "3", "--cpu-seconds", "1", timeout=900)
    assert BASE_KEYS <= set(line)
    for k in ("roofline", "cpu_baseline", "e2e", "clocks", "gpu_launches", "kernels"):
        assert k in line, k
    rf = line["roofline"]
    assert rf["bound"] in ("hbm", "tensor") and rf["peak"] > 0 and 0 < rf["frac"] < 2
    assert line["gpu_launches"] > 0 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] > 0 and line["e2e"]["d2h_bytes_per_step"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["atomic_variation"]["tree"]["distinct_outputs"] == 1

"""The benchmark's reference arm (the oracle timed on the host cores) on the
CPU: one JSON line with the native arm's metric, unit and direction, a
``cpu_baseline`` that describes the run, and an ``e2e`` object with no copies;
ranks other than 0 exit 0 without work or output."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(rank: int):
    env = dict(os.environ, RANK=str(rank))
    return subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
         "--warmup", "3"],
        cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


@pytest.mark.timeout(600)
def test_reference_arm_json_line():
    sys.path.insert(0, ROOT)
    import bench

    r = _run(0)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC
    assert d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["data"] == "synthetic" and d["vs_baseline"] is None
    assert d["config"]["workload"].startswith("blasst_prefill")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert "query tiles" in cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["decode"]["unit"] == "GB/s" and d["decode"]["value"] > 0


def test_reference_arm_other_ranks_silent():
    r = _run(1)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""

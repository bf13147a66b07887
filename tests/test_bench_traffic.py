"""The DRAM traffic that bench.py reports beside each roofline comes from a
committed ncu capture (profiles/traffic.json), keyed by a hash of the kernel's
sources: a capture of an older kernel must read as unmeasured, never as the
current kernel's traffic."""
import json
import os
import shutil

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _captures():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("kernel", sorted(_captures()))
def test_committed_capture_matches_committed_sources(kernel):
    """Each committed capture was taken of the kernel as committed."""
    t = bench.profiled_traffic(kernel)
    assert t is not None, f"{kernel}: sources changed since the capture; recapture it"
    assert t == _captures()[kernel]["traffic_bytes_per_launch"]
    assert t > 0


def test_any_source_edit_voids_the_capture(tmp_path, monkeypatch):
    """Changing one byte of any hashed source (a comment included) makes the
    lookup return None; restoring it brings the figure back."""
    caps = _captures()
    kernel = sorted(caps)[0]
    srcs = caps[kernel]["sources"]
    (tmp_path / "profiles").mkdir()
    shutil.copy(os.path.join(ROOT, "profiles", "traffic.json"), tmp_path / "profiles")
    for s in srcs:
        dst = tmp_path / s
        dst.parent.mkdir(parents=True, exist_ok=True)
        shutil.copy(os.path.join(ROOT, s), dst)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic(kernel) == caps[kernel]["traffic_bytes_per_launch"]
    for s in srcs:
        p = tmp_path / s
        original = p.read_bytes()
        p.write_bytes(original + b"\n// edited\n")
        assert bench.profiled_traffic(kernel) is None, s
        p.write_bytes(original)
    assert bench.profiled_traffic(kernel) == caps[kernel]["traffic_bytes_per_launch"]
    assert bench.profiled_traffic("no_such_kernel") is None

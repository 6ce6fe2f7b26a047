"""bench.py's roofline object and its DRAM-traffic markers, on CPU.

The roofline fraction is algorithmic bytes per launch over the kernel's
measured time against the measured copy peak; the traffic figure beside it
comes from a marker in a committed ncu summary, and counts only while the
kernel's sources hash to the value the marker was captured under."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_roofline_entry_arithmetic():
    # 2,113,929,216 credited bytes in 390 us against a 6453.7 GB/s copy
    ms = 0.390
    achieved = 2113929216 / (ms * 1e-3) / 1e9
    r = bench.roofline_entry("dispatch", achieved, 6453.7, "measured", ms, 2538052500)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["kernel"] == "dispatch"
    assert r["achieved"] == pytest.approx(5420.33, abs=0.01)
    assert r["frac"] == pytest.approx(5420.33 / 6453.7, abs=1e-4)
    # the measured traffic over the same time: 2538 MB in 390 us
    assert r["traffic"] == 2538052500
    assert r["traffic_gbs"] == pytest.approx(6507.83, abs=0.01)
    assert r["traffic_frac"] == pytest.approx(6507.83 / 6453.7, abs=1e-4)
    assert r["peak_kind"] == "measured copy bandwidth"


def test_roofline_entry_without_traffic():
    r = bench.roofline_entry("combine", 5000.0, 6453.7, "fallback", 0.1, None)
    assert r["traffic"] is None
    assert "traffic_gbs" not in r and "traffic_frac" not in r
    assert r["frac"] == pytest.approx(5000.0 / 6453.7, abs=1e-4)
    assert r["peak_kind"] == "fallback copy bandwidth"


@pytest.fixture
def scratch_tree(tmp_path, monkeypatch):
    """A copy of the layout bench.py reads: csrc sources and profiles/."""
    csrc = tmp_path / "combine_moe_layout_06_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in ("combine.cu", "moe_common.cuh", "bulk.cu", "dispatch.cu"):
        (csrc / name).write_text(f"// {name}\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return tmp_path


def _marker(stage, workload, nbytes, sha):
    return f"<!-- roofline-traffic kernel={stage} workload={workload} bytes={nbytes} sources={sha} -->\n"


def test_traffic_marker_follows_the_kernel_sources(scratch_tree):
    sha_c = bench.kernel_source_sha("combine")
    sha_d = bench.kernel_source_sha("dispatch")
    assert sha_c != sha_d and len(sha_c) == 16
    (scratch_tree / "profiles" / "t.md").write_text(
        "# summary\n" + _marker("combine", "dsv3", 123, sha_c) + _marker("dispatch", "dsv3", 456, sha_d)
        + _marker("combine", "olmoe", 789, "0" * 16))
    assert bench.profiled_traffic("combine", "dsv3") == 123
    assert bench.profiled_traffic("dispatch", "dsv3") == 456
    assert bench.profiled_traffic("combine", "olmoe") is None      # captured on other sources
    assert bench.profiled_traffic("combine", "qwen3") is None      # never captured
    # a change to a shared header invalidates both kernels' markers
    (scratch_tree / "combine_moe_layout_06_b200" / "csrc" / "moe_common.cuh").write_text("// changed\n")
    assert bench.kernel_source_sha("combine") != sha_c
    assert bench.profiled_traffic("combine", "dsv3") is None
    assert bench.profiled_traffic("dispatch", "dsv3") is None


def test_traffic_marker_ignores_other_sources_files(scratch_tree):
    sha_c = bench.kernel_source_sha("combine")
    (scratch_tree / "profiles" / "a.md").write_text(_marker("combine", "dsv3", 1, sha_c))
    # a change to a file the combine does not hash leaves its marker valid
    (scratch_tree / "combine_moe_layout_06_b200" / "csrc" / "bulk.cu").write_text("// changed\n")
    assert bench.profiled_traffic("combine", "dsv3") == 1

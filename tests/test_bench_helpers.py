"""Host-side helpers of bench.py (no GPU): the L2 rotation count, the timing-
hygiene note, the DRAM-traffic lookup that must go null when the kernel sources
change, and the peaks file with its fallback."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from w4a4_mixed_precision_b200 import inputs  # noqa: E402


def test_rotation_keeps_each_cycle_above_twice_l2():
    for per_set in (1e6, 9.8e6, 42.7e6, 139.8e6, 632e6):
        n = bench._copies_for(per_set)
        assert 2 <= n <= 16
        assert n * per_set > 2 * bench.L2_BYTES or n == 16


def test_l2_note_names_the_regime():
    assert bench._l2_note(inputs.workload(4)).startswith("larger than L2")
    assert bench._l2_note(inputs.workload(0)).startswith("small case")


def _write_table(path, h):
    with open(path, "w") as f:
        f.write("| kernel | source hash | dram read (B) | dram write (B) | traffic (B) |"
                " algorithmic (B) | ncu time (us) |\n|---|---|---|---|---|---|---|\n")
        f.write(f"| w4a4_gemm_kernel | {h} | 1 | 2 | 3 | 4 | 5.0 |\n")


def test_traffic_only_for_the_profiled_sources(tmp_path, monkeypatch):
    h = bench._kernel_source_hash()
    os.makedirs(tmp_path / "profiles")
    table = tmp_path / "profiles" / "traffic.md"
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "_kernel_source_hash", lambda: h)
    _write_table(table, h)
    assert bench._profiled_traffic("w4a4_gemm_kernel") == 3
    assert bench._profiled_traffic("reorder_quant_kernel") is None
    _write_table(table, "0" * 16)                  # another version of the sources
    assert bench._profiled_traffic("w4a4_gemm_kernel") is None


def test_peaks_fall_back_without_the_measured_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, kind = bench._peaks()
    assert kind == "fallback" and peaks["hbm_gbs"] == pytest.approx(6650.0)

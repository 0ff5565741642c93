"""Host logic of bench.py that needs no GPU: the DRAM-traffic record is used only while the
kernel sources it was measured on are unchanged (comment edits aside), and the record
holds a positive byte count for every benchmark workload."""
import json
import os
import shutil

import pytest

import bench


def test_traffic_record_matches_sources_and_covers_workloads():
    with open(bench.TRAFFIC_FILE) as f:
        t = json.load(f)
    assert t["kernel_sources_sha256"] == bench.kernel_sources_sha256()
    for w in [bench.DEFAULT_WORKLOAD] + bench.SECONDARY_WORKLOADS:
        v = bench.measured_traffic(w)
        assert v is not None and v > 0, w


def test_source_hash_ignores_comments_not_code(tmp_path, monkeypatch):
    csrc = tmp_path / "mixture_experts_grouped_top_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in bench.KERNEL_SOURCES:
        shutil.copy(os.path.join(bench.ROOT, "mixture_experts_grouped_top_b200", "csrc", name), csrc / name)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_sources_sha256()
    target = csrc / bench.KERNEL_SOURCES[0]
    target.write_text("// a new comment line\n\n" + target.read_text())
    assert bench.kernel_sources_sha256() == h0
    target.write_text(target.read_text() + "\nstatic int moe_extra_symbol = 1;\n")
    assert bench.kernel_sources_sha256() != h0
    # a changed source makes the record unusable rather than wrong
    assert bench.measured_traffic(bench.DEFAULT_WORKLOAD) is None

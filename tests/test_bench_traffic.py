"""The DRAM traffic records behind the bench's roofline.traffic: they belong to the kernel
sources they were captured from, and a record for other sources reads as null."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

RECORDS = os.path.join(ROOT, "profiles", "dram_traffic.json")


def test_every_record_is_for_the_current_kernel_sources():
    with open(RECORDS) as f:
        recs = json.load(f)
    assert recs
    h = bench.kernel_source_hash()
    for wl, rec in recs.items():
        assert rec["kernel_source_hash"] == h, f"{wl}: captured from other kernel sources"
        assert rec["dram_bytes_per_launch"] == rec["dram_bytes_read"] + rec["dram_bytes_write"] > 0
        assert "--clock-control none" in rec["command"], wl
        assert bench.load_traffic(wl) == rec["dram_bytes_per_launch"]


def test_a_record_for_other_sources_reads_as_null(monkeypatch):
    with open(RECORDS) as f:
        wl = next(iter(json.load(f)))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.load_traffic(wl) is None
    assert bench.load_traffic("no_such_workload") is None


def test_the_hash_ignores_comments_and_blank_lines():
    src = "int a;  // note\n/* block\n   comment */ int b;\n\n\n"
    assert bench.strip_comments(src) == "int a;\n int b;"
    assert bench.strip_comments(src) == bench.strip_comments(src.replace("note", "other note"))
    assert bench.strip_comments(src) != bench.strip_comments(src.replace("int b", "int c"))

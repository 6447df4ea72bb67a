"""CPU checks of how bench.py reports the measured DRAM traffic of the decode call: it reads the
`traffic-record` lines of the ncu summaries and uses one only for the stock workload and the kernel
sources the capture was taken on (the hash leaves comments out)."""
import dataclasses
import re

import bench
from mla_latent_kv_27_b200 import workloads as wl


def test_records_parse_and_name_stock_workloads():
    recs = bench.traffic_records()
    assert recs, "no traffic records under profiles/"
    for name, entries in recs.items():
        assert name in wl.WORKLOADS, name
        for nbytes, h in entries:
            assert nbytes > 0 and re.fullmatch(r"[0-9a-f]{16}", h)


def test_record_is_used_only_for_its_sources_and_the_stock_workload(monkeypatch):
    recs = bench.traffic_records()
    name, [(nbytes, h)] = next(iter(sorted(recs.items())))
    w = wl.WORKLOADS[name]
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: h)
    assert bench.measured_traffic(w) == nbytes
    # a resized workload is not the captured one
    assert bench.measured_traffic(dataclasses.replace(w, batch=w.batch + 1)) is None
    # other kernel sources: the record no longer describes the kernel
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.measured_traffic(w) is None


def test_source_hash_ignores_comments_and_blank_lines(tmp_path, monkeypatch):
    csrc = tmp_path / "mla_latent_kv_27_b200" / "csrc"
    csrc.mkdir(parents=True)
    for n in bench.TRAFFIC_SOURCES:
        (csrc / n).write_text("int a = 1;  // one\n\nint b = 2;\n")
    monkeypatch.setattr(bench, "__file__", str(tmp_path / "bench.py"))
    h0 = bench.kernel_source_hash()
    (csrc / bench.TRAFFIC_SOURCES[0]).write_text("// header\nint a = 1;  // first\nint b = 2;\n\n")
    assert bench.kernel_source_hash() == h0
    (csrc / bench.TRAFFIC_SOURCES[0]).write_text("int a = 3;\nint b = 2;\n")
    assert bench.kernel_source_hash() != h0

"""Host logic of bench.py that needs no GPU: the ncu traffic summary is used
only while the kernel sources it was captured from are unchanged."""
import os

import bench


def write_summary(root, gemm_digest, act_digest):
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    with open(os.path.join(root, "profiles", "toy_dram.txt"), "w") as f:
        f.write("# DRAM bytes per launch\n")
        f.write(f"gemm_source_digest: {gemm_digest}\n")
        f.write(f"act_source_digest: {act_digest}\n")
        f.write("gemm a 100 20\ngemm b 300 40\nact a 7 3\n")


def test_traffic_used_while_sources_match(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    write_summary(str(tmp_path), bench.source_digest(bench.GEMM_SOURCES), bench.source_digest(bench.ACT_SOURCES))
    t = bench.load_traffic("toy")
    assert t["gemm"] == {"a": 120, "b": 340}
    assert t["act"] == {"a": 10}


def test_traffic_dropped_when_a_kernel_changed(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    write_summary(str(tmp_path), "0" * 16, bench.source_digest(bench.ACT_SOURCES))
    t = bench.load_traffic("toy")
    assert t["gemm"] is None
    assert t["act"] == {"a": 10}


def test_no_summary_no_traffic(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_traffic("missing") == {"gemm": None, "act": None}


def test_digest_covers_every_source():
    a = bench.source_digest(bench.GEMM_SOURCES)
    assert len(a) == 16 and a != bench.source_digest(bench.ACT_SOURCES)

"""Host logic of bench.py that needs no GPU: the ncu traffic summary is used
only while the kernel sources it was captured from are unchanged, and the
clock record keeps the samples taken inside the timed region."""
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


def poller_lines(times, sm=1965, reasons="0,0,0,0"):
    return ["ready\n"] + [f"{t:.6f},{sm},1965,612.5,{reasons}\n" for t in times]


def test_clock_record_keeps_the_samples_inside_the_timed_region():
    lines = poller_lines([0.990, 0.995]) + ["1.001000,1800,1965,700.0,0,0,0,1\n", "1.002000,1900,1965,710.0,0,0,0,0\n",
                                            "1.003000,1950,1965,705.0,0,0,0,0\n"] + poller_lines([1.010])[1:]
    c = bench.summarize_clock_samples(lines, 1.0005, 1.0045)
    assert c["samples"] == 3 and c["window"] == "inside the timed region"
    assert c["sm_mhz"] == 1900 and c["sm_max_mhz"] == 1965
    assert c["reasons"] == ["sw_power_cap"] and c["power_w_max"] == 710.0
    assert abs(c["window_ms"] - 4.0) < 1e-6


def test_clock_record_flags_every_throttle_reason():
    lines = ["1.0,1200,1965,500.0,1,0,0,0\n", "1.001,1200,1965,500.0,0,1,1,0\n"]
    c = bench.summarize_clock_samples(lines, 0.5, 2.0)
    assert c["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_clock_record_falls_back_to_the_nearest_samples():
    c = bench.summarize_clock_samples(poller_lines([0.90, 0.95, 1.20, 1.30, 2.0]), 1.0, 1.001)
    assert c["samples"] == 3 and c["window"] == "nearest to the timed region"
    assert bench.summarize_clock_samples(["ready\n", "garbage\n"], 0.0, 1.0) is None


def test_clock_sampler_without_a_gpu_returns_no_record():
    with bench.ClockSampler("0") as clk:
        clk.mark_start()
        clk.mark_end()
    assert clk.summary() is None

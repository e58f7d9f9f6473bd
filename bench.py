"""Benchmark of the ConvRot linear on B200.

One step = one pass of the whole online path (rotate + per-token quantize +
integer GEMM + dequant) over every linear of the workload, for one batch of M
synthetic tokens.  Default workload: the W8A8 ViT-L encoder linears (qkv
1024->3072, proj 1024->1024, fc1 1024->4096, fc2 4096->1024) at M = 5184 tokens
(72 x 72 patches), Hadamard block 128.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

Multi-GPU runs (torchrun, one process per GPU) are independent replicas: each
rank processes its own batch of tokens (M-split, no collective on the data
path); the timed region is bracketed by barriers and the max over ranks counts.
Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from rotated_bit_quantized_block_b200 import binding as cr  # noqa: E402
from rotated_bit_quantized_block_b200 import workloads as wl  # noqa: E402

METRIC = "ConvRot W8A8/W4A4 linear TOPS and tokens/s (rotate+quant+GEMM+dequant), % roofline"
L2_BYTES = 126 * 1024 * 1024


def replica_ids(rank: int, n_sets: int = 2) -> list:
    """Independent input draws of one rank: weak scaling, no two ranks share a batch."""
    return [rank * n_sets + r for r in range(n_sets)]


def max_over_ranks(value: float, world: int, device) -> float:
    """The slowest rank's time counts (all ranks take part in the same reduction)."""
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(M: int, world: int, steps: int, elapsed_ms: float) -> float:
    """Tokens processed by all ranks divided by the max-over-ranks elapsed time."""
    return M * world * steps / (elapsed_ms / 1000.0)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------------------------------------ traffic

CSRC = os.path.join(ROOT, "rotated_bit_quantized_block_b200", "csrc")
GEMM_SOURCES = ("gemm_tcgen05.cuh", "device_utils.cuh")
ACT_SOURCES = ("rotate_quant.cuh", "device_utils.cuh")


def source_digest(names) -> str:
    """sha256 (first 16 hex digits) of the kernel sources, in order."""
    import hashlib
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(CSRC, n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_traffic(workload: str):
    """DRAM bytes per launch from the committed ncu summary of this workload
    (profiles/<workload>_dram.txt), per kernel and linear; a kernel whose
    sources changed since the capture gets None."""
    path = os.path.join(ROOT, "profiles", f"{workload}_dram.txt")
    out = {"gemm": None, "act": None}
    if not os.path.exists(path):
        return out
    digests, rows = {}, {"gemm": {}, "act": {}}
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.endswith(":") or ": " in line:
                k, v = line.split(":", 1)
                digests[k.strip()] = v.strip()
                continue
            kind, linear, rd, wr = line.split()
            rows[kind][linear] = int(rd) + int(wr)
    for kind, names in (("gemm", GEMM_SOURCES), ("act", ACT_SOURCES)):
        if rows[kind] and digests.get(f"{kind}_source_digest") == source_digest(names):
            out[kind] = rows[kind]
    return out


# ------------------------------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while the timed region runs."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (FileNotFoundError, OSError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None:
            return None
        self.out.flush()
        rows = []
        with open(self.out.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) == 9:
                    rows.append(parts)
        os.unlink(self.out.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        loaded = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max((float(r[3]) for r in rows if r[3].replace(".", "").isdigit()), default=None)}


# ------------------------------------------------------------------------------------------ workload

class Replica:
    """Device buffers of one independent batch: per linear X, Y, codes, workspace."""

    def __init__(self, w: wl.Workload, replica: int, device):
        self.items = []
        for i, lin in enumerate(w.linears):
            X, W, _ = wl.linear_inputs(w, i, replica=replica)
            Xd = torch.from_numpy(X).to(device)
            Wd = torch.from_numpy(W).to(device)
            Wq, sw = cr.convrot_quantize_weight(Wd, w.block, w.bits_of(lin), cr.CLIP_MSE)
            need = cr.convrot_linear_workspace_bytes(w.M, lin.K, lin.N, w.bits_of(lin))
            self.items.append({
                "lin": lin, "X": Xd, "Xhost": torch.from_numpy(X).pin_memory(), "Wq": Wq, "sw": sw,
                "Y": torch.empty((w.M, lin.N), dtype=torch.float16, device=device),
                "Yhost": torch.empty((w.M, lin.N), dtype=torch.float16).pin_memory(),
                "ws": torch.empty(need, dtype=torch.uint8, device=device),
                "W": Wd,
            })

    def nbytes(self):
        return sum(it["X"].nbytes + it["Y"].nbytes + it["Wq"].nbytes + it["ws"].nbytes for it in self.items)


def run_step(w, rep, stream, events=None):
    """One pass over every linear: rotate+quant kernel, then GEMM+dequant kernel.

    The two kernels are launched through convrot_linear_quant_act and
    convrot_linear_gemm, the two halves of convrot_linear_*.  With ``events`` (per linear: act start,
    act end = GEMM start, GEMM end) every kernel is bracketed for per-kernel
    timing; event nodes between kernels also stop the next kernel from starting
    early, so the throughput pass runs without them.
    """
    for i, it in enumerate(rep.items):
        lin = it["lin"]
        ws = it["ws"]
        if events is not None:
            events[i][0].record(stream)
        cr.convrot_linear_quant_act(it["X"], w.block, w.bits_of(lin), ws, stream=stream)
        if events is not None:
            events[i][1].record(stream)
        cr.convrot_linear_gemm(ws, w.M, lin.K, w.bits_of(lin), it["Wq"], it["sw"], None, it["Y"], stream=stream)
        if events is not None:
            events[i][2].record(stream)


def run_e2e(w, reps, stream, steps):
    """``steps`` steps through the public linear entry point with every step's X
    copied in from pinned host memory and Y copied back.  Uploads run on their
    own stream and downloads on another (PCIe is full duplex), each linear
    waiting only for its own input, so one linear's upload overlaps the previous
    linear's compute and download.  A device buffer is rewritten only after its
    previous contents were consumed (X by the linear, Y by the download).
    Forks from and joins back into ``stream`` (capturable in a CUDA graph)."""
    device = stream.device
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    consumed, downloaded = {}, {}
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    for s in range(steps):
        r = s % 2
        for i, it in enumerate(reps[r].items):
            key = (r, i)
            if key in consumed:
                s_in.wait_event(consumed[key])
            with torch.cuda.stream(s_in):
                it["X"].copy_(it["Xhost"], non_blocking=True)
                uploaded = torch.cuda.Event()
                uploaded.record(s_in)
            stream.wait_event(uploaded)
            if key in downloaded:
                stream.wait_event(downloaded[key])
            fn = cr.convrot_linear_w8a8 if w.bits_of(it["lin"]) == 8 else cr.convrot_linear_w4a4
            fn(it["X"], it["Wq"], it["sw"], w.block, None, it["Y"], it["ws"], stream)
            done = torch.cuda.Event()
            done.record(stream)
            consumed[key] = done
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                it["Yhost"].copy_(it["Y"], non_blocking=True)
                out = torch.cuda.Event()
                out.record(s_out)
            downloaded[key] = out
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)


# ------------------------------------------------------------------------------------------ CPU oracle

_ORACLE_WEIGHTS = {}


def oracle_weights(w: wl.Workload):
    """Inputs and oracle-converted weights of every linear (converted once, untimed,
    as the GPU's offline conversion is)."""
    import oracle  # the oracle is only used by the CPU baseline legs

    if w.name not in _ORACLE_WEIGHTS:
        weights = []
        for i in range(len(w.linears)):
            X, W, _ = wl.linear_inputs(w, i)
            qw, sw, _ = oracle.quantize_weight(W, w.block, w.bits_of(w.linears[i]), oracle.CLIP_MSE)
            weights.append((X, qw, sw))
        _ORACLE_WEIGHTS[w.name] = weights
    return _ORACLE_WEIGHTS[w.name]


def time_oracle(w: wl.Workload, budget_s: float, max_rows: int | None = None):
    """Times the CPU oracle (rotate+quant, integer GEMM, dequant) on a bounded
    sample of rows of every linear of the workload."""
    import oracle  # the oracle is only used by the CPU baseline legs

    threads = oracle.set_threads(os.cpu_count() or 1)
    weights = oracle_weights(w)

    def run(rows):
        t0 = time.perf_counter()
        for lin, (X, qw, sw) in zip(w.linears, weights):
            oracle.linear(X[:rows], qw, sw, w.block, w.bits_of(lin))
        return time.perf_counter() - t0

    rows = max(1, min(w.M, 2 * threads))
    t = run(rows)
    target = int(rows * budget_s / max(t, 1e-6))
    rows = max(1, min(w.M if max_rows is None else max_rows, target))
    t = run(rows)
    return {"rows": rows, "seconds": t, "tokens_per_s": rows / t, "threads": threads,
            "ops": sum(2 * rows * l.K * l.N for l in w.linears)}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# ------------------------------------------------------------------------------------------ arms

def reference_arm(args, w, rank, world):
    """The oracle, as it stands, on the host cores: the CPU reference arm."""
    if rank != 0:
        return
    budget = max(2.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        time_oracle(w, budget / 4)
    runs = [time_oracle(w, budget) for _ in range(args.steps)]
    tps = [r["tokens_per_s"] for r in runs]
    value = statistics.median(tps)
    rows = runs[0]["rows"]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * w.M / value,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": dtype_of(w, mma=False),
        "data": "synthetic", "config": config_of(w),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": runs[0]["threads"], "kind": "oracle",
                         "sample": f"{rows} of {w.M} tokens through every linear per step "
                                   f"(rotate+quant, int GEMM, dequant); weights converted untimed; "
                                   f"CPU {cpu_model()}"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "tops": value * sum(2 * l.K * l.N for l in w.linears) / 1e12,
    }
    print(json.dumps(line), flush=True)


def weight_streaming(M: int, bits: int) -> bool:
    """Whether the library runs this linear's GEMM as the weight-streaming kernel
    (its plan: up to 4 tokens with int8 weights, 8 with int4)."""
    return M <= (8 if bits == 4 else 4)


def widths(w: wl.Workload):
    return sorted({w.bits_of(l) for l in w.linears}, reverse=True)


def dtype_of(w: wl.Workload, mma: bool = True) -> str:
    names = {8: "int8", 4: "int4 (int8 MMA)" if mma else "int4"}
    return " / ".join(names[b] for b in widths(w))


def config_of(w: wl.Workload):
    if len(widths(w)) == 1:
        width = f"W{w.bits}A{w.bits}"
    else:
        width = "per-layer " + ", ".join(f"{l.name} W{w.bits_of(l)}A{w.bits_of(l)}" for l in w.linears)
    return {
        "workload": f"{w.name}: " + ", ".join(f"{l.name} {l.K}->{l.N}" for l in w.linears)
                    + f"; M={w.M} tokens; Hadamard block {w.block}; {width}; "
                      f"acts N(0,1) with {w.outlier_frac:.1%} outlier channels x{w.outlier_factor:g}; "
                      f"W N(0,{w.w_sigma})",
        "M": w.M, "block": w.block, "bits": w.bits if len(widths(w)) == 1 else [w.bits_of(l) for l in w.linears],
        "linears": [[l.name, l.K, l.N] for l in w.linears],
        "parallelism": "replicas (M-split, no collective)",
    }


def ours_arm(args, w, rank, world, local_rank):
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    cr.load_library()
    peaks = load_peaks()
    stream = torch.cuda.Stream(device)

    # offline conversion (timed once, reported separately; not part of a step)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    reps = [Replica(w, replica=r, device=device) for r in replica_ids(rank)]
    torch.cuda.synchronize()
    setup_s = time.perf_counter() - t0
    per_set = reps[0].nbytes()
    # offline weight conversion time, measured by itself
    wq_ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    with torch.cuda.stream(stream):
        wq_ev[0].record(stream)
        for it in reps[0].items:
            cr.convrot_quantize_weight(it["W"], w.block, w.bits_of(it["lin"]), cr.CLIP_MSE, stream=stream)
        wq_ev[1].record(stream)
    torch.cuda.synchronize()
    weight_quant_ms = wq_ev[0].elapsed_time(wq_ev[1])
    for rep in reps:
        for it in rep.items:
            del it["W"]

    # warm-up (eager), also initializes per-device kernel attributes before capture
    with torch.cuda.stream(stream):
        for s in range(args.warmup):
            run_step(w, reps[s % 2], stream)
    torch.cuda.synchronize()
    cr.convrot_device_status(stream)

    # capture the K timed steps twice: as they run (throughput), and with events
    # around every kernel (per-kernel durations for the rooflines)
    n_lin = len(w.linears)
    events = [[[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)] for _ in range(n_lin)]
              for _ in range(args.steps)]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for s in range(args.steps):
            run_step(w, reps[s % 2], stream)
    graph_ev = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_ev, stream=stream):
        for s in range(args.steps):
            run_step(w, reps[s % 2], stream, events=events[s])
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        graph.replay()  # untimed replays of the captured steps
        graph_ev.replay()
    torch.cuda.synchronize()

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(device.index) as clk, torch.cuda.stream(stream):
        start.record(stream)
        graph.replay()
        end.record(stream)
        torch.cuda.synchronize()
        graph_ev.replay()
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    elapsed_ms = start.elapsed_time(end)
    act_ms = [[events[s][i][0].elapsed_time(events[s][i][1]) for i in range(n_lin)] for s in range(args.steps)]
    gemm_ms = [[events[s][i][1].elapsed_time(events[s][i][2]) for i in range(n_lin)] for s in range(args.steps)]
    cr.convrot_device_status(stream)
    clocks = clk.summary()

    elapsed_ms = max_over_ranks(elapsed_ms, world, device)
    ms_per_step = elapsed_ms / args.steps
    tokens = w.M * world * args.steps
    value = whole_job_tokens_per_s(w.M, world, args.steps, elapsed_ms)

    # end to end through the public entry point, host buffers in pinned memory
    h2d = sum(it["X"].nbytes for it in reps[0].items)
    d2h = sum(it["Y"].nbytes for it in reps[0].items)
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    # the K steps (copies included) captured once, so that host-side launch
    # cost does not stand in for the device's copy and compute time
    graph_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_e2e, stream=stream):
        run_e2e(w, reps, stream, args.steps)
    with torch.cuda.stream(stream):
        graph_e2e.replay()  # untimed
        torch.cuda.synchronize()
        e_start.record(stream)
        graph_e2e.replay()
        e_end.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end), world, device)
    if world > 1:
        torch.distributed.barrier()
    e2e_value = whole_job_tokens_per_s(w.M, world, args.steps, e2e_ms)
    cr.convrot_device_status(stream)

    if rank != 0:
        return
    ops_step = w.ops()
    gemm_total_ms = sum(sum(r) for r in gemm_ms)
    gemm_ops_total = ops_step * args.steps
    achieved_tops = gemm_ops_total / (gemm_total_ms / 1000.0) / 1e12
    int8_peak = 2.0 * peaks["bf16_tflops"]  # dense int8 = 2 x dense bf16 (4.5 vs 2.25 POPS nominal)
    per_linear_ms = [statistics.mean(gemm_ms[s][i] for s in range(args.steps)) for i in range(n_lin)]
    per_linear_act_ms = [statistics.mean(act_ms[s][i] for s in range(args.steps)) for i in range(n_lin)]
    traffic = load_traffic(w.name)
    gemm_traffic = traffic["gemm"]
    gemm_bytes = {l.name: w.M * l.K + l.N * l.K * w.bits_of(l) // 8 + 2 * w.M * l.N + 4 * w.M + 4 * l.N
                  for l in w.linears}
    if all(weight_streaming(w.M, w.bits_of(l)) for l in w.linears):
        # the fewest tokens run the weight-streaming GEMM: bound by reading the weights
        achieved = sum(gemm_bytes.values()) * args.steps / (gemm_total_ms / 1000.0) / 1e9
        bound = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                 "frac": achieved / peaks["hbm_gbs"], "kernel": "gemv_i8 (weight-streaming, dp4a)",
                 "peak_note": f"{peaks['source']} HBM copy bandwidth"}
    else:
        bound = {"bound": "tensor", "achieved": achieved_tops, "peak": int8_peak, "unit": "TOPS",
                 "frac": achieved_tops / int8_peak,
                 "kernel": "gemm_i8_tcgen05 (int8 x int8 -> int32, fused dequant epilogue)",
                 "peak_note": f"dense int8 = 2 x {peaks['source']} bf16 burst {peaks['bf16_tflops']} TFLOP/s"}
    roofline = {
        **bound,
        # mean DRAM bytes per GEMM launch of one step, from the committed ncu capture
        "traffic": (statistics.mean(gemm_traffic.values()) if gemm_traffic else None),
        "traffic_per_linear": gemm_traffic,
        "algorithmic_bytes_per_linear": gemm_bytes,
        "timing": "second timed pass of the same steps with CUDA events around every kernel launch",
        "per_linear_ms": {l.name: round(t, 5) for l, t in zip(w.linears, per_linear_ms)},
        "per_linear_tops": {l.name: round(2 * w.M * l.K * l.N / (t / 1000) / 1e12, 1)
                            for l, t in zip(w.linears, per_linear_ms)},
    }
    act_bytes = [w.M * l.K * 2 + w.M * l.K + 4 * w.M for l in w.linears]  # codes one byte each in the linear
    act_total_ms = sum(per_linear_act_ms)
    act_gbs = sum(act_bytes) / (act_total_ms / 1000.0) / 1e9
    act_traffic = traffic["act"]
    rotate_quant = {
        "bound": "hbm", "achieved": act_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
        "frac": act_gbs / peaks["hbm_gbs"], "kernel": "act_rotate_quant",
        "traffic": (statistics.mean(act_traffic.values()) if act_traffic else None),
        "traffic_per_linear": act_traffic,
        "algorithmic_bytes_per_linear": {l.name: b for l, b in zip(w.linears, act_bytes)},
        "per_linear_ms": {l.name: round(t, 5) for l, t in zip(w.linears, per_linear_act_ms)},
        "per_linear_gbs": {l.name: round(b / (t / 1000) / 1e9, 1)
                           for l, b, t in zip(w.linears, act_bytes, per_linear_act_ms)},
    }
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": dtype_of(w), "data": "synthetic",
        "config": dict(config_of(w), l2=f"inputs larger than L2: 2 rotating buffer sets of "
                                        f"{per_set / 2**20:.0f} MiB each (L2 {L2_BYTES >> 20} MiB)"),
        "tops": ops_step * world * args.steps / (elapsed_ms / 1000.0) / 1e12,
        "roofline": roofline,
        "rotate_quant": rotate_quant,
        "offline_weight_quant_ms": weight_quant_ms,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "path": "convrot_linear_* with pinned-host X copied in and Y copied out every step "
                        "(uploads and downloads on their own streams, overlapping the linears; the K steps "
                        "replayed from one CUDA graph)"},
        "gpu_launches": 2 * n_lin * args.steps,
        "clocks": clocks,
        "setup_s": setup_s,
    }
    if world == 1 and not args.no_cpu_baseline:
        cb = time_oracle(w, budget_s=args.cpu_budget)
        line["cpu_baseline"] = {
            "value": cb["tokens_per_s"], "unit": "tokens/s", "cores": cb["threads"], "kind": "oracle",
            "sample": f"{cb['rows']} of {w.M} tokens through every linear (rotate+quant, int GEMM, dequant) "
                      f"in {cb['seconds']:.1f} s; weights converted untimed; CPU {cpu_model()}",
        }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="vit_l_w8a8")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.workload.startswith("msweep"):
        w = wl.msweep(int(args.workload.rsplit("M", 1)[1]))
    else:
        w = wl.WORKLOADS[args.workload]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        reference_arm(args, w, rank, world)
        return
    if world > 1:
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        ours_arm(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

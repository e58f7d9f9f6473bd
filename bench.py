"""Benchmark of the ConvRot linear on B200.

One step = one pass of the whole online path (rotate + per-token quantize +
integer GEMM + dequant) over every linear of the workload, for one batch of M
synthetic tokens, through the public linear entry points (one fused launch per
linear where the plan allows).  Default workload: the W8A8 DiT linears (qkv
1536->4608, fc1 1536->6144, fc2 6144->1536) at M = 8192 tokens (batch 2 x 4096),
Hadamard block 128 -- the largest configuration.  The same JSON line carries
sub-results for the ViT-L W8A8 / W4A4 / mixed-width linears and the M sweep,
and context rows (cuBLAS fp16 linear, torch._int_mm ceiling).

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
# (the GEMM kernels with activation warps, and the fused small-M kernel, run the rotation code too)
GEMM_SOURCES = ("gemm_tcgen05.cuh", "gemv.cuh", "rotate_quant.cuh", "device_utils.cuh")
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

# A separate process polls NVML (the library nvidia-smi reads; nothing is set)
# every millisecond, so that samples fall inside a timed region of a few
# milliseconds.  Each line: monotonic time, SM MHz, max SM MHz, power W, and the
# flags hw_slowdown, hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap.
_NVML_POLLER = r"""
import sys, time, pynvml
dev, out, period = sys.argv[1], sys.argv[2], float(sys.argv[3])
pynvml.nvmlInit()
h = pynvml.nvmlDeviceGetHandleByUUID(dev) if dev.startswith("GPU-") else pynvml.nvmlDeviceGetHandleByIndex(int(dev))
mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
bits = (pynvml.nvmlClocksEventReasonHwSlowdown, pynvml.nvmlClocksEventReasonHwThermalSlowdown,
        pynvml.nvmlClocksEventReasonSwThermalSlowdown, pynvml.nvmlClocksEventReasonSwPowerCap)
with open(out, "w", buffering=1) as f:
    f.write("ready\n")
    while True:
        t = time.monotonic()
        sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
        rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
        pw = pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0
        f.write("%.6f,%d,%d,%.1f,%s\n" % (t, sm, mx, pw, ",".join("1" if rs & b else "0" for b in bits)))
        time.sleep(period)
"""
_REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]


def summarize_clock_samples(lines, t0, t1):
    """Clock record of the timed region [t0, t1] (host monotonic seconds) from
    the poller's lines: the samples inside it, else the three nearest to it."""
    rows = []
    for line in lines:
        parts = line.strip().split(",")
        if len(parts) != 8:
            continue
        try:
            rows.append((float(parts[0]), float(parts[1]), float(parts[2]), float(parts[3]),
                         [p == "1" for p in parts[4:8]]))
        except ValueError:
            continue
    if not rows:
        return None
    inside = [r for r in rows if t0 <= r[0] <= t1]
    window = "inside the timed region"
    if not inside:
        mid = 0.5 * (t0 + t1)
        inside = sorted(rows, key=lambda r: abs(r[0] - mid))[:3]
        window = "nearest to the timed region"
    return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
            "reasons": sorted({n for r in inside for n, on in zip(_REASONS, r[4]) if on}),
            "samples": len(inside), "window": window, "window_ms": round(1e3 * (t1 - t0), 3),
            "power_w_max": max(r[3] for r in inside), "source": "NVML, polled every 1 ms"}


def nvml_device_id(device) -> str:
    """The device's NVML id: its UUID ("GPU-" and 8-4-4-4-12 hex digits, which
    does not depend on CUDA_VISIBLE_DEVICES), else its CUDA index."""
    try:
        h = bytes(int(x) & 0xFF for x in torch.cuda.get_device_properties(device).uuid.bytes).hex()
        if len(h) == 32:
            return f"GPU-{h[:8]}-{h[8:12]}-{h[12:16]}-{h[16:20]}-{h[20:]}"
    except Exception:  # noqa: BLE001 -- properties without a UUID
        pass
    return str(device.index)


class ClockSampler:
    """Samples the SM clock and throttle reasons during the timed region: a
    separate process polls NVML every millisecond (nvidia-smi at 100 ms where
    the Python NVML bindings are missing); ``mark_start`` / ``mark_end`` bracket
    the region on the host's monotonic clock."""
    SMI_QUERY = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
                 "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                 "clocks_event_reasons.sw_power_cap")

    def __init__(self, dev_id: str):
        self.dev_id = dev_id
        self.proc = None
        self.smi = False
        self.smi_out = None
        self.t0 = self.t1 = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.out.close()

    def __enter__(self):
        try:
            self.proc = subprocess.Popen([sys.executable, "-c", _NVML_POLLER, self.dev_id, self.out.name, "0.001"],
                                         stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            ready, deadline = False, time.monotonic() + 20.0
            while not ready and time.monotonic() < deadline and self.proc.poll() is None:
                with open(self.out.name) as f:
                    ready = f.read(6) == "ready\n"
                if not ready:
                    time.sleep(0.01)
            if not ready:
                raise OSError("the NVML poller did not start")
        except (FileNotFoundError, OSError):
            self.stop()
            self.smi = True
            try:
                self.smi_out = open(self.out.name, "w")
                self.proc = subprocess.Popen(["nvidia-smi", "-i", self.dev_id, f"--query-gpu={self.SMI_QUERY}",
                                              "--format=csv,noheader,nounits", "-lms", "100"],
                                             stdout=self.smi_out, stderr=subprocess.DEVNULL)
                time.sleep(0.3)
            except (FileNotFoundError, OSError):
                self.proc = None
        time.sleep(0.02)  # a few samples before the region
        return self

    def mark_start(self):
        self.t0 = time.monotonic()

    def mark_end(self):
        self.t1 = time.monotonic()

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.proc = None
        if self.smi_out is not None:
            self.smi_out.close()
            self.smi_out = None

    def __exit__(self, *exc):
        time.sleep(0.02)  # samples after the region
        self.stop()

    def summary(self):
        try:
            with open(self.out.name) as f:
                lines = f.readlines()
            os.unlink(self.out.name)
        except OSError:
            return None
        if self.t0 is None or self.t1 is None:
            return None
        if not self.smi:
            return summarize_clock_samples(lines, self.t0, self.t1)
        # nvidia-smi fallback: no timestamps, the samples around the region
        rows = [[p.strip() for p in line.split(",")] for line in lines]
        rows = [r for r in rows if len(r) == 7]
        num = lambda v: float(v) if v.replace(".", "").isdigit() else None  # noqa: E731
        sm = [num(r[0]) for r in rows if num(r[0]) is not None]
        mx = [num(r[1]) for r in rows if num(r[1]) is not None]
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted({n for r in rows for n, v in zip(_REASONS, r[3:7]) if v.lower() == "active"}),
                "samples": len(rows), "window": "around the timed region", "window_ms": round(1e3 * (self.t1 - self.t0), 3),
                "power_w_max": max((num(r[2]) for r in rows if num(r[2]) is not None), default=None),
                "source": "nvidia-smi, every 100 ms"}


# ------------------------------------------------------------------------------------------ workload

def set_count(w: wl.Workload) -> int:
    """Rotating buffer sets so that one pass over all of them moves more than
    4 x L2 (weights, X, Y and workspaces): no timed step finds its inputs in L2."""
    per_set = 0
    for lin in w.linears:
        b = w.bits_of(lin)
        per_set += lin.N * lin.K * b // 8 + 2 * w.M * lin.K + 2 * w.M * lin.N + w.M * lin.K
    return max(2, min(32, -(-int(4 * L2_BYTES) // max(per_set, 1))))


class Replica:
    """Device buffers of one independent batch: per linear X, Y, weights and workspace."""

    def __init__(self, w: wl.Workload, replica: int, device, host_copies: bool = False):
        self.items = []
        for i, lin in enumerate(w.linears):
            X, W, _ = wl.linear_inputs(w, i, replica=replica)
            Xd = torch.from_numpy(X).to(device)
            Wd = torch.from_numpy(W).to(device)
            Wq, sw = cr.convrot_quantize_weight(Wd, w.block, w.bits_of(lin), cr.CLIP_MSE)
            need = cr.convrot_linear_workspace_bytes(w.M, lin.K, lin.N, w.bits_of(lin))
            item = {"lin": lin, "X": Xd, "Wq": Wq, "sw": sw, "W": Wd,
                    "Y": torch.empty((w.M, lin.N), dtype=torch.float16, device=device),
                    "ws": torch.empty(need, dtype=torch.uint8, device=device)}
            if host_copies:
                item["Xhost"] = torch.from_numpy(X).pin_memory()
                item["Yhost"] = torch.empty((w.M, lin.N), dtype=torch.float16).pin_memory()
            self.items.append(item)

    def nbytes(self):
        return sum(it["X"].nbytes + it["Y"].nbytes + it["Wq"].nbytes + it["ws"].nbytes for it in self.items)


def linear_call(w, it, stream):
    """One linear through the public entry point (one fused launch where the plan allows)."""
    fn = cr.convrot_linear_w8a8 if w.bits_of(it["lin"]) == 8 else cr.convrot_linear_w4a4
    fn(it["X"], it["Wq"], it["sw"], w.block, None, it["Y"], it["ws"], stream)


def run_step(w, rep, stream):
    """One pass over every linear of the workload for one batch of tokens."""
    for it in rep.items:
        linear_call(w, it, stream)


def graph_ms(calls, stream, reps: int = 3) -> float:
    """Average device time of one call of ``calls`` (a list of callables taking a
    stream), captured back to back in one CUDA graph and replayed: events on the
    launching stream around the replay; best of ``reps`` replays."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for c in calls:
            c(stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        g.replay()  # untimed
        torch.cuda.synchronize()
        best = None
        for _ in range(reps):
            e0.record(stream)
            g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            t = e0.elapsed_time(e1) / len(calls)
            best = t if best is None else min(best, t)
    del g
    return best


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
        r = s % len(reps)
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
            linear_call(w, it, stream)
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


def time_oracle(w: wl.Workload, budget_s: float, max_rows: int | None = None, threads: int | None = None):
    """Times the CPU oracle (rotate+quant, integer GEMM, dequant) on a bounded
    sample of rows of every linear of the workload (all host cores unless
    ``threads`` is given)."""
    import oracle  # the oracle is only used by the CPU baseline legs

    threads = oracle.set_threads(threads or os.cpu_count() or 1)
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


def linear_bytes(w, lin, M=None) -> int:
    """Algorithmic bytes of one linear with the rotate+quant fused in: X read,
    codes in and out of L2 are not counted, weights, Y and scales."""
    M = w.M if M is None else M
    return 2 * M * lin.K + lin.N * lin.K * w.bits_of(lin) // 8 + 2 * M * lin.N + 4 * M + 4 * lin.N


def act_bytes(w, lin) -> int:
    """Algorithmic bytes of the activation pass: X read, one code byte per element and the scales written."""
    return 3 * w.M * lin.K + 4 * w.M


def measure_workload(w, reps, stream, steps, peaks, clock_index=None, warmup=3):
    """Times one workload: ``warmup`` eager steps, then the step graph (``steps``
    steps over rotating buffer sets, the value), then every linear by itself
    (the public linear, and its two halves apart) in graphs of back-to-back
    launches over the same sets."""
    n_sets = len(reps)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for s in range(warmup):
            run_step(w, reps[s % n_sets], stream)
    torch.cuda.synchronize()
    cr.convrot_device_status(stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for s in range(steps):
            run_step(w, reps[s % n_sets], stream)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = None
    with torch.cuda.stream(stream):
        g.replay()  # untimed
        torch.cuda.synchronize()
        if clock_index is not None:
            with ClockSampler(clock_index) as clk:
                clk.mark_start()
                start.record(stream)
                g.replay()
                end.record(stream)
                torch.cuda.synchronize()
                clk.mark_end()
            clocks = clk.summary()
        else:
            start.record(stream)
            g.replay()
            end.record(stream)
            torch.cuda.synchronize()
    del g
    elapsed_ms = start.elapsed_time(end)
    cr.convrot_device_status(stream)

    per = {}
    for i, lin in enumerate(w.linears):
        bits = w.bits_of(lin)
        items = [rep.items[i] for rep in reps]
        plan = cr.convrot_linear_plan(w.M, lin.K, lin.N, bits, w.block, items[0]["ws"].numel())
        calls = [(lambda st, it=it: linear_call(w, it, st)) for it in items] * 2
        act = [(lambda st, it=it: cr.convrot_linear_quant_act(it["X"], w.block, bits, it["ws"], stream=st))
               for it in items] * 2
        if plan["weights_widened"]:
            # the W4A4 linear's GEMM multiplies the weights its activation launch widened
            # to int8 codes; they follow the int8-weight plan's part of the workspace
            off = cr.convrot_linear_workspace_bytes(w.M, lin.K, lin.N, 8)
            for it in items:
                cr.convrot_linear_w4a4(it["X"], it["Wq"], it["sw"], w.block, None, it["Y"], it["ws"], stream)
            gw = [it["ws"][off: off + lin.N * lin.K].view(torch.int8).view(lin.N, lin.K) for it in items]
            gemm = [(lambda st, it=it, g=g: cr.convrot_linear_gemm(it["ws"], w.M, lin.K, 8, g, it["sw"], None,
                                                                   it["Y"], stream=st))
                    for it, g in zip(items, gw)] * 2
        else:
            gemm = [(lambda st, it=it: cr.convrot_linear_gemm(it["ws"], w.M, lin.K, bits, it["Wq"], it["sw"], None,
                                                              it["Y"], stream=st)) for it in items] * 2
        t_lin, t_act, t_gemm = graph_ms(calls, stream), graph_ms(act, stream), graph_ms(gemm, stream)
        per[lin.name] = {"plan": plan, "linear_ms": t_lin, "act_ms": t_act, "gemm_ms": t_gemm}
        if plan["fused_available"]:
            # the rotation fused into the GEMM kernel (convrot_linear_w8a8_fused), for comparison
            fused = [(lambda st, it=it: cr.convrot_linear_w8a8_fused(it["X"], it["Wq"], it["sw"], w.block, None,
                                                                     it["Y"], it["ws"], st)) for it in items] * 2
            per[lin.name]["fused_ms"] = graph_ms(fused, stream)
    cr.convrot_device_status(stream)

    ops = w.ops()
    lin_ms = sum(v["linear_ms"] for v in per.values())
    # the dominant kernel: the GEMM (the activation launch is reported under rotate_quant)
    dom_ms = sum(v["gemm_ms"] for v in per.values())
    int8_peak = 2.0 * peaks["bf16_tflops"]  # dense int8 = 2 x dense bf16 (4.5 vs 2.25 POPS nominal)
    # the GEMM's algorithmic bytes: activation codes (one byte each), weight codes, Y and the scales
    gemm_bytes = {l.name: linear_bytes(w, l) - w.M * l.K for l in w.linears}
    ridge = int8_peak * 1e12 / (peaks["hbm_gbs"] * 1e9)  # int8 ops per byte where the two roofs meet
    if ops / sum(gemm_bytes.values()) < ridge:
        # few tokens: bound by streaming the weights (and the activation codes)
        achieved = sum(gemm_bytes.values()) / (dom_ms / 1e3) / 1e9
        kinds = {v["plan"]["gemm_kind"] for v in per.values()}
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"],
                "kernel": ("gemv_i8 (weight-streaming, dp4a)" if kinds == {2} else
                           "gemm_i8_tcgen05 feature-major (all tokens in one tile, K split over clusters)"),
                "peak_note": f"{peaks['source']} HBM copy bandwidth; the GEMM's {ops / sum(gemm_bytes.values()):.0f} "
                             f"int8 ops per byte lie below the ridge of {ridge:.0f}",
                "per_linear_frac": {l.name: round(gemm_bytes[l.name] / (per[l.name]["gemm_ms"] / 1e3) / 1e9
                                                  / peaks["hbm_gbs"], 3) for l in w.linears}}
    else:
        achieved = ops / (dom_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": int8_peak, "unit": "TOPS",
                "frac": achieved / int8_peak,
                "kernel": "gemm_i8_tcgen05 (int8 x int8 -> int32 in TMEM, dequant epilogue)",
                "peak_note": f"dense int8 = 2 x {peaks['source']} bf16 burst {peaks['bf16_tflops']} TFLOP/s",
                "per_linear_frac": {l.name: round(2 * w.M * l.K * l.N / (per[l.name]["gemm_ms"] / 1e3) / 1e12
                                                  / int8_peak, 3) for l in w.linears}}
    roof.update({
        "timing": "each linear alone: CUDA graph of back-to-back launches over the rotating buffer sets, "
                  "CUDA events on the launching stream around the replay",
        "per_linear_us": {n: round(1e3 * v["gemm_ms"], 2) for n, v in per.items()},
    })
    act_total_ms = sum(v["act_ms"] for v in per.values())
    act_gbs = sum(act_bytes(w, l) for l in w.linears) / (act_total_ms / 1e3) / 1e9
    rq = {"bound": "hbm", "achieved": act_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
          "frac": act_gbs / peaks["hbm_gbs"],
          "kernel": "act_rotate_quant_tma (the activation launch of the two-launch linear; fused into the GEMM "
                    "otherwise)",
          "algorithmic_bytes_per_linear": {l.name: act_bytes(w, l) for l in w.linears},
          "per_linear_us": {n: round(1e3 * v["act_ms"], 2) for n, v in per.items()},
          "per_linear_gbs": {l.name: round(act_bytes(w, l) / (per[l.name]["act_ms"] / 1e3) / 1e9, 1)
                             for l in w.linears}}
    fused_cmp = {n: {"fused_us": round(1e3 * v["fused_ms"], 2), "two_launch_us": round(1e3 * v["linear_ms"], 2)}
                 for n, v in per.items() if "fused_ms" in v}
    return {
        "fused_linear": fused_cmp,
        "elapsed_ms": elapsed_ms, "ms_per_step": elapsed_ms / steps, "clocks": clocks,
        "tokens_per_s": w.M * steps / (elapsed_ms / 1e3), "tops": ops * steps / (elapsed_ms / 1e3) / 1e12,
        "roofline": roof, "rotate_quant": rq,
        "kernel_us_per_step": round(1e3 * lin_ms, 2),
        "act_plus_gemm_us_per_step": round(1e3 * sum(v["act_ms"] + v["gemm_ms"] for v in per.values()), 2),
        "launches_per_step": sum(v["plan"]["launches"] for v in per.values()),
        "plans": {n: v["plan"] for n, v in per.items()},
    }


def eager_ms(fn, stream, reps: int = 20) -> float:
    """Average device time of ``fn()`` launched ``reps`` times back to back on
    ``stream`` (library calls that are not captured into graphs here)."""
    with torch.cuda.stream(stream):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def context_rows(w, reps, stream, peaks):
    """Context only: cuBLAS fp16 F.linear on the same shapes (over the same
    rotating buffer sets), and a torch._int_mm 8192^3 int8 ceiling."""
    out = {}
    try:
        per = {}
        for i, lin in enumerate(w.linears):
            pairs = [(rep.items[i]["X"], rep.items[i]["W16"]) for rep in reps]
            k = [0]

            def call(pairs=pairs, k=k):
                X, W = pairs[k[0] % len(pairs)]
                k[0] += 1
                torch.nn.functional.linear(X, W)
            per[lin.name] = round(1e3 * eager_ms(call, stream), 2)
        out["f_linear_fp16_us"] = per
        out["f_linear_fp16_us_per_step"] = round(sum(per.values()), 2)
    except Exception as e:  # context only
        out["f_linear_fp16_error"] = repr(e)[:200]
    try:
        n = 8192
        a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=stream.device)
        b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=stream.device)
        ms = eager_ms(lambda: torch._int_mm(a, b), stream, reps=10)
        out["int_mm_8192_tops"] = round(2 * n ** 3 / (ms / 1e3) / 1e12, 1)
        out["int_mm_8192_frac_of_int8_peak"] = round(2 * n ** 3 / (ms / 1e3) / 1e12 / (2 * peaks["bf16_tflops"]), 3)
        del a, b
    except Exception as e:
        out["int_mm_error"] = repr(e)[:200]
    return out


def ours_arm(args, w, rank, world, local_rank):
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    cr.load_library()
    peaks = load_peaks()
    stream = torch.cuda.Stream(device)

    torch.cuda.synchronize()
    t0 = time.perf_counter()
    n_sets = args.sets if args.sets > 0 else set_count(w)
    reps = [Replica(w, replica=r, device=device, host_copies=True) for r in replica_ids(rank, n_sets)]
    torch.cuda.synchronize()
    setup_s = time.perf_counter() - t0
    per_set = reps[0].nbytes()
    # offline weight conversion, measured by itself (not part of a step)
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
            it["W16"] = it.pop("W")

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    m = measure_workload(w, reps, stream, args.steps, peaks, clock_index=nvml_device_id(device),
                         warmup=args.warmup)
    if world > 1:
        torch.distributed.barrier()
    elapsed_ms = max_over_ranks(m["elapsed_ms"], world, device)
    value = whole_job_tokens_per_s(w.M, world, args.steps, elapsed_ms)

    # end to end through the public entry point, host buffers in pinned memory
    h2d = sum(it["X"].nbytes for it in reps[0].items)
    d2h = sum(it["Y"].nbytes for it in reps[0].items)
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
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
    del graph_e2e
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end), world, device)
    if world > 1:
        torch.distributed.barrier()
    e2e_value = whole_job_tokens_per_s(w.M, world, args.steps, e2e_ms)
    cr.convrot_device_status(stream)

    if rank != 0:
        return
    traffic = load_traffic(w.name)
    roofline = dict(m["roofline"])
    roofline["traffic"] = statistics.mean(traffic["gemm"].values()) if traffic["gemm"] else None
    roofline["traffic_per_linear"] = traffic["gemm"]
    # the GEMM's own: activation codes in, weight codes, Y and the scales
    roofline["algorithmic_bytes_per_linear"] = {l.name: linear_bytes(w, l) - w.M * l.K for l in w.linears}
    rotate_quant = dict(m["rotate_quant"])
    rotate_quant["traffic"] = statistics.mean(traffic["act"].values()) if traffic["act"] else None
    rotate_quant["traffic_per_linear"] = traffic["act"]
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": dtype_of(w), "data": "synthetic",
        "config": dict(config_of(w), l2=(f"inputs larger than L2: {n_sets} rotating buffer sets of "
                                         f"{per_set / 2**20:.0f} MiB each, {n_sets * per_set / L2_BYTES:.1f} x "
                                         f"L2 per pass (L2 {L2_BYTES >> 20} MiB)"
                                         if n_sets * per_set > 1.5 * L2_BYTES else
                                         f"{n_sets} buffer set(s) of {per_set / 2**20:.0f} MiB: "
                                         f"NOT larger than 1.5 x L2 (profiling run)")),
        "tops": m["tops"] * world,
        "roofline": roofline,
        "rotate_quant": rotate_quant,
        "kernel_us_per_step": m["kernel_us_per_step"],
        "act_plus_gemm_us_per_step": m["act_plus_gemm_us_per_step"],
        "fused_linear": m["fused_linear"],
        "plans": m["plans"],
        "offline_weight_quant_ms": weight_quant_ms,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "path": "convrot_linear_* with pinned-host X copied in and Y copied out every step "
                        "(uploads and downloads on their own streams, overlapping the linears; the K steps "
                        "replayed from one CUDA graph)"},
        "gpu_launches": m["launches_per_step"] * args.steps,
        "clocks": m["clocks"],
        "setup_s": setup_s,
    }
    if world == 1 and not args.no_sub_results:
        subs = {}
        for name in SUB_WORKLOADS:
            if name == w.name:
                continue
            sw_ = workload_by_name(name)
            sreps = [Replica(sw_, replica=r, device=device) for r in range(set_count(sw_))]
            sm = measure_workload(sw_, sreps, stream, args.sub_steps, peaks)
            subs[name] = {
                "tokens_per_s": sm["tokens_per_s"], "tops": sm["tops"], "us_per_step": 1e3 * sm["ms_per_step"],
                "kernel_us_per_step": sm["kernel_us_per_step"],
                "act_plus_gemm_us_per_step": sm["act_plus_gemm_us_per_step"], "fused_linear": sm["fused_linear"],
                "roofline_bound": sm["roofline"]["bound"], "roofline_frac": sm["roofline"]["frac"],
                "roofline_achieved": sm["roofline"]["achieved"], "roofline_unit": sm["roofline"]["unit"],
                "per_linear_frac": sm["roofline"]["per_linear_frac"],
                "rotate_quant_frac": sm["rotate_quant"]["frac"], "rotate_quant_gbs": sm["rotate_quant"]["achieved"],
                "plans": {n: f"{'widened int4 weights, ' if p['weights_widened'] else ''}"
                             f"{['token-major', 'feature-major', 'gemv'][p['gemm_kind']]}"
                             f"{' bn' + str(p['tile_n']) if p['tile_n'] else ''}{' pair' if p['cta_pair'] else ''}"
                             f"{' stream-K' if p['stream_k'] else ''}{' split' + str(p['k_splits']) if p['k_splits'] > 1 else ''}"
                          for n, p in sm["plans"].items()},
                "sets": len(sreps),
            }
            del sreps
            torch.cuda.empty_cache()
        line["sub_results"] = subs
        line["context"] = context_rows(w, reps, stream, peaks)
    if world == 1 and not args.no_cpu_baseline:
        cb = time_oracle(w, budget_s=args.cpu_budget)
        line["cpu_baseline"] = {
            "value": cb["tokens_per_s"], "unit": "tokens/s", "cores": cb["threads"], "kind": "oracle",
            "sample": f"{cb['rows']} of {w.M} tokens through every linear (rotate+quant, int GEMM, dequant) "
                      f"in {cb['seconds']:.1f} s; weights converted untimed; CPU {cpu_model()}",
        }
        single = {}
        for name in ("tiny_w8a8", "vit_l_w8a8"):
            c = time_oracle(workload_by_name(name), budget_s=args.cpu_budget / 4, threads=1)
            single[name] = {"tokens_per_s": c["tokens_per_s"], "rows": c["rows"], "seconds": round(c["seconds"], 2)}
        line["cpu_baseline"]["single_thread"] = single
    print(json.dumps(line), flush=True)


SUB_WORKLOADS = ("vit_l_w8a8", "vit_l_w4a4", "vit_l_mixed", "msweep_w8a8_M1", "msweep_w8a8_M16",
                 "msweep_w8a8_M128", "msweep_w8a8_M1024", "msweep_w8a8_M4096", "msweep_w8a8_M16384")


def workload_by_name(name: str) -> wl.Workload:
    if name.startswith("msweep"):
        return wl.msweep(int(name.rsplit("M", 1)[1]))
    return wl.WORKLOADS[name]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="dit_w8a8")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sub-results", action="store_true")
    ap.add_argument("--sub-steps", type=int, default=10)
    # rotating buffer sets (default: enough to move 4 x L2 per pass); fewer
    # only to keep a profiler capture small -- its timings then see warm L2
    ap.add_argument("--sets", type=int, default=0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    w = workload_by_name(args.workload)

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

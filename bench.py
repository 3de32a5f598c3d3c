"""Benchmark of the packed ternary matmul library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tq|reference]
                    [--workload NAME]

Metric: effective weight GB/s (packed bytes the fused matmul must read: codes,
scales, code book) and % of measured HBM peak. One step is one pass of the hot
path over one batch of synthetic input for the chosen workload (default
`fmt_b_4096`: Format B 4096 x 4096 layers, ladder 3^-(k-1), alpha 0.02, no
rho, x at batch 1 and at batch 4). Distinct layer copies rotate so that no
timed launch re-reads codes from L2. Every step runs as CUDA-graph replays of
the library's C-ABI calls, timed with CUDA events on the launching stream.

`--impl reference` times the CPU oracle (single thread) on a bounded sample of
the same workload and prints the same JSON line with "impl": "reference".
Multi-GPU (torchrun): independent replicas, one per GPU, no data-path
collective; timing is the max over ranks.
"""
import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from packed_weight_matmul_b200 import inputs as I  # noqa: E402

METRIC = ("fused packed-ternary GEMV/GEMM effective weight GB/s and % HBM "
          "peak, batch 1–64")
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 2 ** 20


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "src": "measured",
                "bf16_tflops": float(p.get("bf16_tflops", 1590.0)),
                "bf16_tflops_sustained": float(
                    p.get("bf16_tflops_sustained", 1400.0))}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "src": "fallback",
                "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---- distributed plumbing (replicas only) -------------------------------------

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.distributed.init_process_group(
            "nccl", timeout=datetime.timedelta(seconds=120),
            device_id=torch.device("cuda", local))
    return world, rank, local


def dist_max(v: float, world: int) -> float:
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device="cuda")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


# ---- clocks -----------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}",
                 f"--query-gpu=timestamp,{self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = [r.split(", ") for r in out.strip().splitlines() if r.strip()]
        sm, smax, reasons, powers = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        for r in rows:
            if len(r) < 10:
                continue
            try:
                sm.append(float(r[2]))
                smax.append(float(r[3]))
                powers.append(float(r[4]))
            except ValueError:
                continue
            for name, val in zip(names, r[6:10]):
                if val.strip() == "Active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(smax),
                "power_w_max": max(powers), "samples": len(sm),
                "reasons": sorted(reasons)}


# ---- kernel-source hash (ncu traffic is only reported for the same kernel) --------

def kernel_hash(files):
    h = hashlib.sha256()
    for f in files:
        path = os.path.join(ROOT, "packed_weight_matmul_b200", "csrc", f)
        if os.path.exists(path):
            with open(path, "rb") as fh:
                h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_label, files, units):
    """dram bytes per launch from the committed ncu summary, or None when the
    kernel source changed since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            table = json.load(f)
    except (OSError, ValueError):
        return None
    e = table.get(kernel_label)
    if not e or e.get("source_hash") != kernel_hash(files):
        return None
    return e["dram_bytes_per_unit"] * units


# ---- workloads ----------------------------------------------------------------------

class Step:
    """One graph replay inside a step: `launches` library launches that move
    `bytes` algorithmic bytes, attributed to one kernel."""

    def __init__(self, name, graph, bytes_, launches, kernel, flops=0.0):
        self.name, self.graph, self.bytes = name, graph, bytes_
        self.launches, self.kernel, self.flops = launches, kernel, flops


class FmtB4096:
    """Format B 4096 x 4096 layers, ladder 3^-(k-1), alpha 0.02, no rho, x at
    batch 1 and 4. `layers` distinct code copies rotate (> 3x L2)."""
    name = "fmt_b_4096"
    N = K = 4096
    BATCHES = (1, 4)
    SOURCES = ("tq_linear.cu", "tq_linear_simple.cu", "tq_gemv_b.cu")

    def __init__(self, layers=24):
        self.layers = layers

    def describe(self):
        return {"workload": f"{self.name}: Format B {self.N}x{self.K} uint8 "
                f"codes uniform 0..242, ladder a_k=3^-(k-1), alpha=0.02, no "
                f"rho; x bf16 N(0,1) at batch 1 and 4",
                "layers_rotated": self.layers,
                "bytes_resident": self.layers * self.N * self.K,
                "l2": "rotating distinct layers, resident bytes > 3x L2: no "
                      "timed launch re-reads codes from L2",
                "batches": list(self.BATCHES), "parallelism": "replicas"}

    def weight_bytes(self):
        return self.N * self.K + 972

    def setup(self, tq, dev):
        lut = tq.tq_build_lut(I.ALPHA, I.ladder_pow3().numpy())
        self.lut_d = torch.from_numpy(lut).to(dev)
        self.codes = [I.codes_uniform(self.N, self.K, 1 + 7919 * i, device=dev)
                      for i in range(self.layers)]
        self.w = [tq.weights_b(c, self.lut_d) for c in self.codes]
        self.x_host = {b: I.x_normal(b, self.K, 20 + b).pin_memory()
                       for b in self.BATCHES}
        self.x = {b: self.x_host[b].to(dev) for b in self.BATCHES}
        self.y = {b: torch.zeros(self.layers, b, self.N, device=dev)
                  for b in self.BATCHES}
        self.y_host = {b: torch.empty_like(self.y[b], device="cpu").pin_memory()
                       for b in self.BATCHES}

    def capture(self, tq):
        steps = []
        for b in self.BATCHES:
            for i in range(self.layers):  # warm the path once before capture
                tq.tq_linear(self.w[i], self.x[b], self.y[b][i])
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for i in range(self.layers):
                    tq.tq_linear(self.w[i], self.x[b], self.y[b][i])
            steps.append(Step(f"batch{b}", g, self.layers * self.weight_bytes(),
                              self.layers, f"linear_b_batch{b}",
                              2.0 * b * self.N * self.K * self.layers))
        return steps

    def h2d(self):
        for b in self.BATCHES:
            self.x[b].copy_(self.x_host[b], non_blocking=True)
        return sum(self.x_host[b].numel() * 2 for b in self.BATCHES)

    def d2h(self):
        for b in self.BATCHES:
            self.y_host[b].copy_(self.y[b], non_blocking=True)
        return sum(self.y[b].numel() * 4 for b in self.BATCHES)

    # -- oracle legs --
    def oracle_setup(self):
        from oracle import oref
        self.oref = oref
        self.codes_h = I.codes_uniform(self.N, self.K, 1).numpy()
        self.lut_h = oref.build_lut(I.ALPHA, I.ladder_pow3().numpy())
        self.xb_h = {b: I.bits(I.x_normal(b, self.K, 20 + b))
                     for b in self.BATCHES}

    def oracle_pass(self, rows):
        """One oracle pass over `rows` rows at every batch; returns bytes."""
        for b in self.BATCHES:
            self.oref.linear_B(self.codes_h[:rows], self.lut_h, self.xb_h[b])
        return len(self.BATCHES) * rows * self.K


WORKLOADS = {"fmt_b_4096": FmtB4096}


# ---- the two arms ------------------------------------------------------------------------

def time_oracle(wl, seconds):
    """Time the single-threaded oracle for about `seconds` on whole passes."""
    wl.oracle_setup()
    rows = 64
    t0 = time.perf_counter()
    wl.oracle_pass(rows)
    dt = time.perf_counter() - t0
    rows = int(max(1, min(wl.N, rows * seconds / max(dt, 1e-6) / 4)))
    total_bytes, t_total, passes = 0, 0.0, 0
    while t_total < seconds:
        t0 = time.perf_counter()
        total_bytes += wl.oracle_pass(rows)
        t_total += time.perf_counter() - t0
        passes += 1
    return total_bytes, t_total, rows, passes


def run_reference(args, world, rank):
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]()
    wl.oracle_setup()
    # size each step so the whole run ends within about two minutes
    t0 = time.perf_counter()
    wl.oracle_pass(16)
    per_row = (time.perf_counter() - t0) / 16
    budget = 90.0 / max(1, args.steps + args.warmup)
    rows = int(max(1, min(wl.N, budget / max(per_row, 1e-9))))
    for _ in range(args.warmup):
        wl.oracle_pass(rows)
    t0 = time.perf_counter()
    nbytes = 0
    for _ in range(args.steps):
        nbytes += wl.oracle_pass(rows)
    dt = time.perf_counter() - t0
    value = nbytes / dt / 1e9
    sample = (f"{rows} of {wl.N} rows of one {wl.N}x{wl.K} layer per step, "
              f"at batch {' and '.join(map(str, wl.BATCHES))}")
    line = {"impl": "reference", "metric": METRIC, "value": value,
            "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "config": wl.describe(),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_tq(args, world, rank, local):
    from packed_weight_matmul_b200 import tq
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = WORKLOADS[args.workload]()
    wl.setup(tq, dev)
    steps = wl.capture(tq)
    stream = torch.cuda.current_stream()

    def one_step(marks=None):
        if marks is not None:
            marks[0].record(stream)
        for i, s in enumerate(steps):
            s.graph.replay()
            if marks is not None:
                marks[i + 1].record(stream)

    for _ in range(max(3, args.warmup)):
        one_step()
    torch.cuda.synchronize()
    # one event per graph boundary per step: per-graph (per-kernel) durations
    # come from the same timed region as the step time
    marks = [[torch.cuda.Event(enable_timing=True)
              for _ in range(len(steps) + 1)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    for k in range(args.steps):
        one_step(marks[k])
    torch.cuda.synchronize()
    barrier(world)
    elapsed_ms = marks[0][0].elapsed_time(marks[-1][-1])
    per = np.zeros(len(steps))
    for m in marks:
        for i in range(len(steps)):
            per[i] += m[i].elapsed_time(m[i + 1])
    per /= args.steps
    time.sleep(0.2)
    clk = clocks.stop()
    elapsed_ms = dist_max(elapsed_ms, world)
    step_bytes = sum(s.bytes for s in steps)
    value = world * step_bytes * args.steps / (elapsed_ms / 1e3) / 1e9

    # e2e: pinned H2D of the step's inputs, the graphs, D2H of the results
    e_start, e_end = torch.cuda.Event(enable_timing=True), \
        torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e_start.record(stream)
    h2d = d2h = 0
    for _ in range(args.steps):
        h2d = wl.h2d()
        one_step()
        d2h = wl.d2h()
    e_end.record(stream)
    torch.cuda.synchronize()
    e2e_ms = dist_max(e_start.elapsed_time(e_end), world)
    e2e_value = world * step_bytes * args.steps / (e2e_ms / 1e3) / 1e9

    if rank != 0:
        return
    pk = peaks()
    # dominant kernel: the graph with the largest share of the step
    dom = int(np.argmax(per))
    s = steps[dom]
    per_launch_s = per[dom] / 1e3 / s.launches
    bytes_per_launch = s.bytes / s.launches
    achieved = bytes_per_launch / per_launch_s / 1e9
    traffic = ncu_traffic(s.kernel, wl.SOURCES, 1)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": wl.describe(),
        "pct_hbm_peak": 100.0 * value / world / pk["hbm_gbs"],
        "roofline": {"bound": "hbm", "achieved": achieved,
                     "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / pk["hbm_gbs"],
                     "traffic": traffic, "kernel": s.kernel,
                     "peak_src": pk["src"],
                     "algorithmic_bytes_per_launch": bytes_per_launch},
        "per_graph_ms": {st.name: float(p) for st, p in zip(steps, per)},
        "per_graph_gbs": {st.name: st.bytes / (p / 1e3) / 1e9
                          for st, p in zip(steps, per)},
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "clocks": clk,
        "gpu_launches": int(sum(st.launches for st in steps) * args.steps),
    }
    if world == 1 and not args.no_cpu_baseline:
        nbytes, secs, rows, passes = time_oracle(wl, args.cpu_seconds)
        line["cpu_baseline"] = {
            "value": nbytes / secs / 1e9, "unit": "GB/s", "cores": 1,
            "kind": "oracle",
            "sample": f"{passes} passes over {rows} rows of one "
                      f"{wl.N}x{wl.K} layer at batch "
                      f"{' and '.join(map(str, wl.BATCHES))} "
                      f"({secs:.1f} s, single thread)"}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["tq", "reference"], default="tq")
    ap.add_argument("--workload", choices=sorted(WORKLOADS),
                    default="fmt_b_4096")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_tq(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

"""Benchmark of the packed ternary matmul library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tq|reference]
                    [--workload NAME] [--batch B ...]

Metric: effective weight GB/s (packed bytes the fused matmul must read: codes,
scales, code book) and % of measured HBM peak, batch 1-64. One step is one
pass of the hot path over one batch of synthetic input for the chosen
workload. The default, `decode_step`, is the 60-block decode step of
Gemma-4-31B-shaped Format B linear layers (q, k, v 8192 x 5376; o 5376 x
8192; gate, up 21504 x 5376; down 5376 x 21504; 31.4 GB of codes resident) at
batch 1, 4, 16 and 64: one CUDA graph of the 420 ordered tq_linear calls per
batch, all four graphs in every step. Every step runs as CUDA-graph replays of
the library's C-ABI calls, timed with CUDA events on the launching stream.

`--impl reference` times the CPU oracle (all host cores) on a bounded sample
of the same workload and prints the same JSON line with "impl": "reference".
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
    """One process per GPU (torchrun env). NCCL when there is a GPU; gloo on a
    host without one (the reference arm and the CPU tests of this path)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        timeout = datetime.timedelta(seconds=120)
        if torch.cuda.is_available():
            torch.distributed.init_process_group(
                "nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            torch.distributed.init_process_group("gloo", timeout=timeout)
    return world, rank, local


def dist_max(v: float, world: int) -> float:
    """Max of v over the ranks (the slowest rank's time)."""
    if world == 1:
        return v
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
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
    sources the captured kernel is built from (the entry's "files", else the
    workload's) changed since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            table = json.load(f)
    except (OSError, ValueError):
        return None
    e = table.get(kernel_label)
    if not e or e.get("source_hash") != kernel_hash(e.get("files", files)):
        return None
    return e["dram_bytes_per_unit"] * units


# ---- workloads ----------------------------------------------------------------------

class Step:
    """One graph replay inside a step: `launches` library launches that move
    `bytes` algorithmic bytes, attributed to one kernel."""

    def __init__(self, name, graph, bytes_, launches, kernel, flops=0.0):
        self.name, self.graph, self.bytes = name, graph, bytes_
        self.launches, self.kernel, self.flops = launches, kernel, flops


def capture_graph(calls):
    """Warm the calls once, then capture them into one CUDA graph."""
    for c in calls:
        c()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for c in calls:
            c()
    return g


class Workload:
    """A workload: device inputs, the graphs of one step, the host copies of
    the end-to-end leg and the oracle sample of the CPU legs."""
    name = ""
    SOURCES = ("tq_linear.cu", "tq_gemv_a.cu", "tq_gemv_b.cu", "tq_gemm_tc.cu",
               "tq_linear_simple.cu")

    def h2d(self):
        for dst, src in self.inputs:
            dst.copy_(src, non_blocking=True)
        return sum(src.numel() * src.element_size() for _, src in self.inputs)

    def d2h(self):
        for dst, src in self.outputs:
            dst.copy_(src, non_blocking=True)
        return sum(src.numel() * src.element_size() for _, src in self.outputs)

    def pin_io(self, xs, ys):
        """xs: device inputs refreshed from pinned host copies every step;
        ys: device results read back every step."""
        self.inputs = [(x, x.cpu().pin_memory()) for x in xs]
        self.outputs = [(torch.empty_like(y, device="cpu").pin_memory(), y)
                        for y in ys]


class FmtB4096(Workload):
    """Format B 4096 x 4096 layers, ladder 3^-(k-1), alpha 0.02, no rho, x at
    batch 1 and 4. `layers` distinct code copies rotate (> 3x L2)."""
    name = "fmt_b_4096"
    N = K = 4096
    BATCHES = (1, 4)
    MAX_ROWS = 4096

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
        self.x = {b: I.x_normal(b, self.K, 20 + b).to(dev)
                  for b in self.BATCHES}
        self.y = {b: torch.zeros(self.layers, b, self.N, device=dev)
                  for b in self.BATCHES}
        self.pin_io(list(self.x.values()), list(self.y.values()))

    def capture(self, tq):
        steps = []
        for b in self.BATCHES:
            calls = [lambda i=i, b=b: tq.tq_linear(self.w[i], self.x[b],
                                                   self.y[b][i])
                     for i in range(self.layers)]
            steps.append(Step(f"batch{b}", capture_graph(calls),
                              self.layers * self.weight_bytes(), self.layers,
                              f"linear_b_batch{b}",
                              2.0 * b * self.N * self.K * self.layers))
        return steps

    # -- oracle legs --
    def oracle_setup(self):
        from oracle import oref
        self.oref = oref
        self.codes_h = I.codes_uniform(self.N, self.K, 1).numpy()
        self.lut_h = oref.build_lut(I.ALPHA, I.ladder_pow3().numpy())
        self.xb_h = {b: I.bits(I.x_normal(b, self.K, 20 + b))
                     for b in self.BATCHES}

    def oracle_jobs(self, rows, r0=0):
        """Independent oracle calls of one pass over rows [r0, r0 + rows) at
        every batch: (callable, algorithmic bytes)."""
        c = self.codes_h[r0:r0 + rows]
        return [(lambda b=b: self.oref.linear_B(c, self.lut_h, self.xb_h[b]),
                 len(c) * self.K) for b in self.BATCHES]

    def sample_desc(self, rows):
        return (f"{rows} of {self.N} rows of one {self.N}x{self.K} layer at "
                f"batch {' and '.join(map(str, self.BATCHES))}")


class FmtBGemma(Workload):
    """Format B Gemma-shaped layers with rho: up 21504x5376 and down
    5376x21504 (one rho per row), q, k, v 8192x5376 (one rho per 128-row
    head); x at batch 1, 4 and 16. 364 MB resident (> 2x L2); each graph runs
    one batch over all five layers, so a layer's codes are evicted between
    its reads."""
    name = "fmt_b_gemma"
    BATCHES = (1, 4, 16)
    MAX_ROWS = 21504
    N = 21504  # rows of the sampled layer for the CPU legs
    K = 5376

    def describe(self):
        return {"workload": f"{self.name}: Format B up 21504x5376 and down "
                "5376x21504 with fp16 rho per row, q/k/v 8192x5376 with fp16 "
                "rho per 128-row head, rho ~ U(0.5,1.5), alpha=0.02, ladder "
                "a_k=3^-(k-1); x bf16 N(0,1) at batch 1, 4 and 16",
                "bytes_resident": sum(l.n * l.k for l in I.FMT_B_GEMMA_LAYERS),
                "l2": "5 distinct layers, 364 MB resident",
                "batches": list(self.BATCHES), "parallelism": "replicas"}

    def setup(self, tq, dev):
        lut = tq.tq_build_lut(I.ALPHA, I.ladder_pow3().numpy())
        self.lut_d = torch.from_numpy(lut).to(dev)
        self.layers = I.FMT_B_GEMMA_LAYERS
        self.w, self.keep = [], []
        for l in self.layers:
            idx = [q.name for q in self.layers].index(l.name)
            s = I.SEEDS["fmt_b_gemma"] * 1000 + idx
            codes = I.codes_uniform(l.n, l.k, s, device=dev)
            rho = I.rho_uniform(I.rho_count(l.n, l.rps), s + 500) \
                .view(torch.int16).to(dev)
            self.keep += [codes, rho]
            self.w.append(tq.weights_b(codes, self.lut_d, rho, l.rps))
        self.x = {(b, k): I.x_normal(b, k, 30 + b).to(dev)
                  for b in self.BATCHES for k in {l.k for l in self.layers}}
        self.y = {(b, i): torch.zeros(b, l.n, device=dev)
                  for b in self.BATCHES for i, l in enumerate(self.layers)}
        self.pin_io(list(self.x.values()), list(self.y.values()))

    def capture(self, tq):
        steps = []
        for b in self.BATCHES:
            calls = [lambda i=i, l=l, b=b: tq.tq_linear(
                self.w[i], self.x[(b, l.k)], self.y[(b, i)])
                for i, l in enumerate(self.layers)]
            nbytes = sum(l.n * l.k + 972 + 2 * I.rho_count(l.n, l.rps)
                         for l in self.layers)
            steps.append(Step(f"batch{b}", capture_graph(calls), nbytes,
                              len(self.layers), f"linear_b_gemma_batch{b}",
                              2.0 * b * sum(l.n * l.k for l in self.layers)))
        return steps

    def oracle_setup(self):
        from oracle import oref
        self.oref = oref
        cfg = I.fmt_b_gemma_layer(I.FMT_B_GEMMA_LAYERS[0])
        self.codes_h = cfg["codes"].numpy()
        self.rho_h = I.bits(cfg["rho"])
        self.lut_h = oref.build_lut(I.ALPHA, I.ladder_pow3().numpy())
        self.xb_h = {b: I.bits(I.x_normal(b, self.K, 30 + b))
                     for b in self.BATCHES}

    def oracle_jobs(self, rows, r0=0):
        c = self.codes_h[r0:r0 + rows]
        rho = self.rho_h[r0:r0 + rows]
        return [(lambda b=b: self.oref.linear_B(
            c, self.lut_h, self.xb_h[b], rho, 1), len(c) * self.K)
            for b in self.BATCHES]

    def sample_desc(self, rows):
        return (f"{rows} of 21504 rows of the up layer (21504x5376, rho per "
                f"row) at batch 1, 4 and 16")


class FmtALarge(Workload):
    """Format A 28672 x 8192 (bf16 0.02 * StudentT(5)), G = 64: quantize and
    pack both planes, then the fused matmul with one and with two planes at
    batch 1, 8, 32 and 64. The quantize graph moves 2 B/weight in and the
    package out; each linear graph reads the package once."""
    name = "fmt_a_large"
    N, K, G = 28672, 8192, 64
    MAX_ROWS = 64
    BATCHES = (1, 8, 32, 64)

    def describe(self):
        return {"workload": f"{self.name}: Format A W {self.N}x{self.K} bf16 = "
                "0.02*StudentT(5), G=64, two planes: tq_quantize_pack, then "
                "tq_linear with 1 and 2 planes at batch 1, 8, 32, 64",
                "bytes_resident": 2 * self.N * self.K + 2 * 55050240,
                "l2": "470 MB bf16 W and 110 MB package resident (> L2)",
                "batches": list(self.BATCHES), "parallelism": "replicas"}

    def setup(self, tq, dev):
        self.W = I.fmt_a_large()["W"].to(dev)
        gpr, nb = self.K // self.G, 13
        self.codes = torch.empty(2 * self.N * gpr * nb, dtype=torch.uint8,
                                 device=dev)
        self.scales = torch.empty(2 * self.N * gpr, dtype=torch.int16,
                                  device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.w = {p: tq.weights_a(self.codes, self.scales, self.N, self.K,
                                  self.G, p) for p in (1, 2)}
        self.x = {b: I.x_normal(b, self.K, 40 + b).to(dev)
                  for b in self.BATCHES}
        self.y = {(p, b): torch.zeros(b, self.N, device=dev)
                  for p in (1, 2) for b in self.BATCHES}
        self.pin_io(list(self.x.values()), list(self.y.values()))
        self.tq = tq

    def capture(self, tq):
        steps = []
        plane_bytes = self.N * (self.K // self.G) * 15
        q = capture_graph([lambda: tq.tq_quantize_pack(
            self.W, self.G, 2, self.codes, self.scales, self.status)])
        steps.append(Step("quantize2", q, 2 * self.N * self.K + 2 * plane_bytes,
                          1, "quantize_pack_a"))
        for p in (1, 2):
            for b in self.BATCHES:
                g = capture_graph([lambda p=p, b=b: tq.tq_linear(
                    self.w[p], self.x[b], self.y[(p, b)])])
                steps.append(Step(f"linear_p{p}_b{b}", g, p * plane_bytes, 1,
                                  f"linear_a_p{p}_batch{b}",
                                  2.0 * b * p * self.N * self.K))
        return steps

    def oracle_setup(self):
        from oracle import oref
        self.oref = oref
        rows = 64
        Wh = I.bits(I.student_t_bf16(rows, self.K, seed=3))
        self.Wh = Wh
        self.pkg = oref.quantize_pack_A(Wh, self.G, 2)
        self.xb_h = {b: I.bits(I.x_normal(b, self.K, 40 + b))
                     for b in self.BATCHES}

    def oracle_jobs(self, rows, r0=0):
        rows = max(0, min(rows, 64 - r0))
        codes, scales = self.pkg
        codes = codes[:, r0:r0 + rows]
        scales = scales[:, r0:r0 + rows]
        Wr = self.Wh[r0:r0 + rows]
        plane = rows * (self.K // self.G) * 15
        jobs = [(lambda: self.oref.quantize_pack_A(Wr, self.G, 2),
                 2 * rows * self.K + 2 * plane)]
        for p in (1, 2):
            for b in self.BATCHES:
                jobs.append((lambda p=p, b=b: self.oref.linear_A(
                    codes[:p], scales[:p], rows, self.K, self.xb_h[b], self.G,
                    p), p * plane))
        return jobs

    def sample_desc(self, rows):
        return (f"{min(rows, 64)} rows x 8192 of the Format A workload: "
                "quantize both planes, then linear with 1 and 2 planes at "
                "batch 1, 8, 32, 64")


class DecodeStep(Workload):
    """60 blocks x {q, k, v 8192x5376; o 5376x8192; gate, up 21504x5376; down
    5376x21504} Format B layers (31.4 GB of codes), alpha 0.02, no rho, one
    x per distinct k and batch. One step = the 420 ordered tq_linear calls at
    every batch of `batches` (one CUDA graph per batch); tokens/s of a batch
    = batch / its graph time. The step's result read back in the end-to-end
    leg is the last layer's output at every batch."""
    name = "decode_step"
    SOURCES = Workload.SOURCES
    MAX_ROWS = 256

    def __init__(self, batches=I.DECODE_BATCHES, blocks=I.GEMMA_BLOCKS):
        self.BATCHES = tuple(batches)
        self.blocks = blocks

    def describe(self):
        bs = ", ".join(map(str, self.BATCHES))
        return {"workload": f"{self.name}: {self.blocks} blocks x 7 Format B "
                "layers (q,k,v 8192x5376; o 5376x8192; gate,up 21504x5376; "
                "down 5376x21504), codes uniform 0..242, ladder "
                "a_k=3^-(k-1), alpha=0.02, no rho; x bf16 N(0,1); one graph "
                f"of the {7 * self.blocks} ordered layers per batch, batch "
                f"{bs}",
                "layers": 7 * self.blocks,
                "bytes_resident": sum(l.n * l.k for _, l in
                                      I.decode_step_layers(self.blocks)),
                "l2": "31.4 GB of codes resident (250x L2): every launch "
                      "streams its layer from HBM",
                "batches": list(self.BATCHES), "parallelism": "replicas"}

    def setup(self, tq, dev):
        lut = tq.tq_build_lut(I.ALPHA, I.ladder_pow3().numpy())
        self.lut_d = torch.from_numpy(lut).to(dev)
        self.layers = I.decode_step_layers(self.blocks)
        self.codes = [I.codes_uniform(l.n, l.k, s, device=dev)
                      for s, l in self.layers]
        self.w = [tq.weights_b(c, self.lut_d) for c in self.codes]
        ks = sorted({l.k for _, l in self.layers})
        self.x = {(b, k): I.x_normal(b, k, 50 + b).to(dev)
                  for b in self.BATCHES for k in ks}
        # one output buffer per (batch, position in the block): layers are
        # not chained, the last layer's output is the step's result
        self.y = {(b, j): torch.zeros(b, l.n, device=dev)
                  for b in self.BATCHES
                  for j, l in enumerate(I.BLOCK_LAYERS)}
        last = len(I.BLOCK_LAYERS) - 1
        self.pin_io(list(self.x.values()),
                    [self.y[(b, last)] for b in self.BATCHES])

    def step_bytes(self):
        return sum(l.n * l.k + 972 for _, l in self.layers)

    def capture(self, tq):
        steps = []
        nl = len(I.BLOCK_LAYERS)
        for b in self.BATCHES:
            calls = [lambda i=i, l=l, b=b: tq.tq_linear(
                self.w[i], self.x[(b, l.k)], self.y[(b, i % nl)])
                for i, (_, l) in enumerate(self.layers)]
            steps.append(Step(f"batch{b}", capture_graph(calls),
                              self.step_bytes(), len(calls),
                              f"linear_b_decode_batch{b}",
                              2.0 * b * sum(l.n * l.k for _, l in
                                            self.layers)))
        return steps

    def extra(self, steps, per_ms):
        """tokens/s per batch: batch / the time of its 420-layer graph."""
        return {"tokens_per_s": {f"batch{b}": b / (p / 1e3)
                                 for b, p in zip(self.BATCHES, per_ms)}}

    def oracle_setup(self):
        from oracle import oref
        self.oref = oref
        self.sample = [(l, I.codes_uniform(256, l.k, s).numpy())
                       for s, l in I.decode_step_layers(1)]
        self.lut_h = oref.build_lut(I.ALPHA, I.ladder_pow3().numpy())
        self.xb = {(b, l.k): I.bits(I.x_normal(b, l.k, 50 + b))
                   for b in self.BATCHES for l, _ in self.sample}

    def oracle_jobs(self, rows, r0=0):
        """Independent oracle calls of one pass over rows [r0, r0 + rows) of
        each of the 7 layer shapes of one block, at every batch: (callable,
        bytes)."""
        rows = max(0, min(rows, 256 - r0))
        jobs = []
        for b in self.BATCHES:
            for l, codes in self.sample:
                jobs.append((lambda c=codes[r0:r0 + rows],
                             x=self.xb[(b, l.k)]:
                             self.oref.linear_B(c, self.lut_h, x),
                             rows * l.k))
        return jobs

    def sample_desc(self, rows):
        return (f"{min(rows, 256)} rows of each of the 7 layer shapes of one "
                f"block at batch {', '.join(map(str, self.BATCHES))}")


class Layer(Workload):
    """One layer shape on its own (`--fmt`, `--n`, `--k`, `--planes`,
    `--batch`): Format B codes uniform on 0..242 with the 3^-(k-1) ladder
    (alpha 0.02, no rho), or a Format A package (G = 64) quantized on the GPU
    from bf16 0.02*StudentT(5) weights; x bf16 N(0,1). Enough distinct copies
    of the package rotate that they exceed 3x L2. Used for per-kernel
    profiles and sweeps."""
    name = "layer"
    MAX_ROWS = 256

    def __init__(self, fmt="B", n=8192, k=5376, batches=(1,), planes=1,
                 lut_rows=0):
        self.fmt, self.n, self.k = fmt.upper(), n, k
        self.BATCHES = tuple(batches)
        self.planes = planes
        self.lut_rows = lut_rows if self.fmt == "B" else 0
        self.books = -(-n // lut_rows) if self.lut_rows else 1
        if self.fmt == "A":
            self.pkg = planes * n * (k // 64) * 15
        elif self.fmt == "B7":
            self.pkg = n * 14 * (k // 16) + 512
        else:
            self.pkg = n * k + 972 * self.books
        self.copies = max(1, -(-3 * L2_BYTES // self.pkg))

    def describe(self):
        what = (f"Format A {self.n}x{self.k}, G=64, {self.planes} plane(s), "
                "quantized from bf16 0.02*StudentT(5)" if self.fmt == "A" else
                f"7-bit alphabet {self.n}x{self.k}, codes uniform over 45 "
                "seeded words of the 243, 7-bit indices into the used-code "
                "table, ladder a_k=3^-(k-1), alpha=0.02, no rho"
                if self.fmt == "B7" else
                f"Format B {self.n}x{self.k}, codes uniform 0..242, ladder "
                "a_k=3^-(k-1), alpha=0.02, no rho" if not self.lut_rows else
                f"Format B {self.n}x{self.k}, codes uniform 0..242, adaptive "
                f"alphabet: one code book per {self.lut_rows} rows (ladder "
                "amplitudes U(0.01, 1) per block, seeded), alpha=0.02, no rho")
        return {"workload": f"{self.name}: {what}; x bf16 N(0,1) at batch "
                f"{', '.join(map(str, self.BATCHES))}",
                "layers_rotated": self.copies,
                "bytes_resident": self.copies * self.pkg,
                "l2": "rotating distinct copies, resident bytes > 3x L2",
                "batches": list(self.BATCHES), "parallelism": "replicas"}

    def setup(self, tq, dev):
        n, k = self.n, self.k
        if self.fmt == "A":
            W = I.student_t_bf16(n, k, seed=3).to(dev)
            nb = self.planes * n * (k // 64)
            c0 = torch.empty(nb * 13, dtype=torch.uint8, device=dev)
            s0 = torch.empty(nb + 8, dtype=torch.int16, device=dev)
            st = torch.zeros(1, dtype=torch.int32, device=dev)
            tq.tq_quantize_pack(W, 64, self.planes, c0, s0, st)
            del W
            self.keep = [(c0.clone(), s0.clone()) for _ in range(self.copies)]
            self.w = [tq.weights_a(c, s, n, k, 64, self.planes)
                      for c, s in self.keep]
        elif self.fmt == "B7":
            lut = tq.tq_build_lut(I.ALPHA, I.ladder_pow3().numpy())
            self.keep = []
            for i in range(self.copies):
                c = torch.from_numpy(self.codes45(n, k, 5 + i)).to(dev)
                used = torch.empty(128, dtype=torch.uint8, device=dev)
                cnt = torch.zeros(1, dtype=torch.int32, device=dev)
                pk = torch.empty(n, 14 * (k // 16), dtype=torch.uint8,
                                 device=dev)
                tq.tq_pack7(c, used, cnt, pk)
                l7 = torch.from_numpy(tq.tq_build_lut7(
                    lut, used.cpu().numpy())).to(dev)
                del c
                self.keep.append((pk, l7))
            self.w = [tq.weights_b7(pk, l7, n, k) for pk, l7 in self.keep]
        else:
            self.lut_d = torch.from_numpy(self.book_array(tq.tq_build_lut)).to(dev)
            self.keep = [I.codes_uniform(n, k, 5 + i, device=dev)
                         for i in range(self.copies)]
            self.w = [tq.weights_b(c, self.lut_d, lut_rows=self.lut_rows)
                      for c in self.keep]
        self.x = {b: I.x_normal(b, k, 60 + b).to(dev) for b in self.BATCHES}
        self.y = {b: torch.zeros(b, n, device=dev) for b in self.BATCHES}
        self.pin_io(list(self.x.values()), list(self.y.values()))

    @staticmethod
    def codes45(n, k, seed):
        """Codes uniform over 45 seeded words of the 243."""
        rng = np.random.default_rng(seed)
        words = rng.choice(243, 45, replace=False).astype(np.uint8)
        return words[rng.integers(0, 45, (n, k))]

    def book_array(self, build):
        """The layer's code book, or one per block (seeded ladders)."""
        if not self.lut_rows:
            return build(I.ALPHA, I.ladder_pow3().numpy())
        rng = np.random.default_rng(17)
        lad = rng.uniform(0.01, 1.0, (self.books, 5)).astype(np.float32)
        return np.stack([build(I.ALPHA, lad[b]) for b in range(self.books)])

    def capture(self, tq):
        steps = []
        for b in self.BATCHES:
            calls = [lambda i=i, b=b: tq.tq_linear(self.w[i], self.x[b],
                                                   self.y[b])
                     for i in range(self.copies)]
            steps.append(Step(f"batch{b}", capture_graph(calls),
                              self.copies * self.pkg, self.copies,
                              f"linear_{self.fmt.lower()}_layer_batch{b}",
                              2.0 * b * self.planes * self.n * self.k *
                              self.copies))
        return steps

    def oracle_setup(self):
        from oracle import oref
        self.oref = oref
        rows = 256
        if self.fmt == "A":
            Wh = I.bits(I.student_t_bf16(rows, self.k, seed=3))
            self.pkg_h = oref.quantize_pack_A(Wh, 64, self.planes)
        elif self.fmt == "B7":
            self.lut_h = oref.build_lut(I.ALPHA, I.ladder_pow3().numpy())
            self.b7_h = oref.pack7(self.codes45(rows, self.k, 5))
        else:
            self.codes_h = I.codes_uniform(rows, self.k, 5).numpy()
            self.lut_h = self.book_array(oref.build_lut)
        self.xb = {b: I.bits(I.x_normal(b, self.k, 60 + b))
                   for b in self.BATCHES}

    def oracle_jobs(self, rows, r0=0):
        rows = max(0, min(rows, 256 - r0))
        jobs = []
        for b in self.BATCHES:
            if self.fmt == "B7":
                used, _, pk = self.b7_h
                pr = pk[r0:r0 + rows]
                jobs.append((lambda b=b, pr=pr, used=used: self.oref.linear_B7(
                    pr, used, len(pr), self.k, self.lut_h, self.xb[b]),
                    rows * 14 * (self.k // 16)))
            elif self.fmt == "A":
                c, s = self.pkg_h
                c, s = c[:, r0:r0 + rows], s[:, r0:r0 + rows]
                jobs.append((lambda b=b, c=c, s=s: self.oref.linear_A(
                    c, s, rows, self.k, self.xb[b], 64, self.planes),
                    self.planes * rows * (self.k // 64) * 15))
            else:
                c = self.codes_h[r0:r0 + rows]
                # the sample's rows r0.. decode with their own books
                lr = self.lut_rows
                L = self.lut_h if not lr else \
                    self.lut_h[r0 // lr:][:-(-rows // lr) + 1]
                jobs.append((lambda b=b, c=c, L=L: self.oref.linear_B(
                    c, L, self.xb[b], lut_rows=lr), rows * self.k))
        return jobs

    def sample_desc(self, rows):
        return (f"{min(rows, 256)} rows of the {self.n}x{self.k} layer at "
                f"batch {', '.join(map(str, self.BATCHES))}")


class FmtASmall(Workload):
    """Format A 512 x 1024 seed-0 workload (L2-resident; small)."""
    name = "fmt_a_small"
    N, K, G = 512, 1024, 64
    MAX_ROWS = 512
    BATCHES = (1,)

    def describe(self):
        return {"workload": f"{self.name}: Format A W 512x1024 bf16 "
                "0.02*N(0,1) with 1% x10 outliers and one zero group per "
                "64-row block, G=64; quantize + pack, then tq_linear at "
                "batch 1 (L2-resident)", "batches": [1],
                "l2": "122,880-byte package: L2-resident",
                "parallelism": "replicas"}

    def setup(self, tq, dev):
        cfg = I.fmt_a_small()
        self.W = cfg["W"].to(dev)
        self.codes = torch.empty(512 * 16 * 13, dtype=torch.uint8, device=dev)
        self.scales = torch.empty(512 * 16, dtype=torch.int16, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.wa = tq.weights_a(self.codes, self.scales, 512, 1024, 64, 1)
        self.x = cfg["x"].to(dev)
        self.y = torch.zeros(1, 512, device=dev)
        self.pin_io([self.x], [self.y])

    def capture(self, tq):
        q = capture_graph([lambda: tq.tq_quantize_pack(
            self.W, 64, 1, self.codes, self.scales, self.status)])
        l = capture_graph([lambda: tq.tq_linear(self.wa, self.x, self.y)])
        return [Step("quantize", q, 2 * 512 * 1024 + 122880, 1,
                     "quantize_pack_a"),
                Step("linear", l, 122880, 1, "linear_a_small_batch1",
                     2.0 * 512 * 1024)]

    def oracle_setup(self):
        from oracle import oref
        self.oref = oref
        cfg = I.fmt_a_small()
        self.Wh = I.bits(cfg["W"])
        self.xb = I.bits(cfg["x"])
        self.pkg = oref.quantize_pack_A(self.Wh, 64, 1)

    def oracle_jobs(self, rows, r0=0):
        rows = max(0, min(rows, 512 - r0))
        codes, scales = self.pkg
        codes, scales = codes[:, r0:r0 + rows], scales[:, r0:r0 + rows]
        Wr = self.Wh[r0:r0 + rows]
        return [(lambda: self.oref.quantize_pack_A(Wr, 64, 1),
                 rows * 1024 * 2 + rows * 16 * 15),
                (lambda: self.oref.linear_A(codes, scales, rows, 1024,
                                            self.xb), rows * 16 * 15)]

    def sample_desc(self, rows):
        return f"{min(rows, 512)} rows of the 512x1024 workload"


class EncodeB(Workload):
    """Format B encoder (tq_encode_b) on the Gemma-shaped layers: up
    21504x5376 with one scale per row and q 8192x5376 with one scale per
    128-row head, W = bf16(0.02 StudentT(5)), the page's fitted ladder
    (1, 0.33, 0.115, 0.037, 0.012), zero bias 0.5. Algorithmic bytes: W read
    once (2 B/weight), codes written (1 B/weight) and rho."""
    name = "encode_b"
    MAX_ROWS = 256
    BATCHES = ()
    LADDER = (1.0, 0.33, 0.115, 0.037, 0.012)
    SHAPES = ((21504, 5376, 1), (8192, 5376, 128))
    SOURCES = ("tq_encode.cu",)

    def describe(self):
        return {"workload": f"{self.name}: Format B encoder, up 21504x5376 "
                "(rho per row) and q 8192x5376 (rho per 128-row head), W "
                "bf16 0.02*StudentT(5), ladder (1, 0.33, 0.115, 0.037, "
                "0.012), zeta 0.5",
                "l2": "231 MB and 88 MB of W per launch (> L2)",
                "batches": [], "parallelism": "replicas"}

    def setup(self, tq, dev):
        self.W, self.codes, self.rho = [], [], []
        for i, (n, k, rps) in enumerate(self.SHAPES):
            self.W.append(I.student_t_bf16(n, k, seed=80 + i).to(dev))
            self.codes.append(torch.empty(n, k, dtype=torch.uint8, device=dev))
            self.rho.append(torch.empty((n + rps - 1) // rps,
                                        dtype=torch.int16, device=dev))
        self.alpha = torch.zeros(len(self.SHAPES), device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.pin_io([self.W[1]], [self.alpha])

    def capture(self, tq):
        steps = []
        for i, (n, k, rps) in enumerate(self.SHAPES):
            g = capture_graph([lambda i=i, rps=rps: tq.tq_encode_b(
                self.W[i], self.LADDER, 0.5, rps, self.codes[i], self.rho[i],
                self.alpha[i:i + 1], self.status)])
            nbytes = 3 * n * k + 2 * ((n + rps - 1) // rps)
            steps.append(Step(f"encode_{n}x{k}_rps{rps}", g, nbytes, 3,
                              "encode_b"))
        return steps

    def oracle_setup(self):
        from oracle import oref
        self.oref = oref
        self.sample = [I.bits(I.student_t_bf16(256, k, seed=80 + i))
                       for i, (n, k, rps) in enumerate(self.SHAPES)]

    def oracle_jobs(self, rows, r0=0):
        rows = max(0, min(rows, 256 - r0))
        lad = np.array(self.LADDER, np.float32)
        jobs = []
        for (n, k, rps), Wh in zip(self.SHAPES, self.sample):
            Wr = Wh[r0:r0 + rows]
            jobs.append((lambda Wr=Wr, rps=rps: self.oref.encode_B(
                Wr, lad, 0.5, rps if rps == 1 else 0), 3 * rows * k))
        return jobs

    def sample_desc(self, rows):
        return f"{min(rows, 256)} rows of each encoder layer shape"


class ExpertsA(Workload):
    """Expert-indexed Format A layer (tq_linear_experts): 128 experts of
    768 x 2048 (a mixture-of-experts FFN projection), G = 64, the 32 hot
    experts 0..31 with a second plane; 64 routed rows per call (8 tokens x
    8 experts), ids seeded uniform on 0..127; weights bf16 0.02*StudentT(5)
    quantized on the GPU. Algorithmic bytes: the packages (codes + scales,
    both planes of hot experts) of the distinct experts a call touches."""
    name = "experts_a"
    MAX_ROWS = 64
    E, N, K, HOT, TOKENS = 128, 768, 2048, 32, 64
    BATCHES = (64,)
    SOURCES = ("tq_gemv_a.cu", "tq_api.cu")

    def __init__(self):
        gpr = self.K // 64
        self.per = self.N * gpr  # groups per expert plane
        self.pkg = (self.E + self.HOT) * self.per * 15
        self.copies = max(1, -(-3 * L2_BYTES // self.pkg))
        g = torch.Generator().manual_seed(41)
        self.ids_h = torch.randint(0, self.E, (self.TOKENS,), generator=g,
                                   dtype=torch.int32)
        used = sorted(set(self.ids_h.tolist()))
        self.call_bytes = sum((2 if e < self.HOT else 1) * self.per * 15
                              for e in used)

    def describe(self):
        return {"workload": f"{self.name}: {self.E} Format A experts of "
                f"{self.N}x{self.K}, G=64, experts 0..{self.HOT - 1} with two "
                f"planes, {self.TOKENS} routed rows per call (ids uniform), "
                "weights bf16 0.02*StudentT(5); x bf16 N(0,1)",
                "layers_rotated": self.copies,
                "bytes_resident": self.copies * self.pkg,
                "l2": "rotating distinct copies, resident bytes > 3x L2",
                "batches": [self.TOKENS], "parallelism": "replicas"}

    def setup(self, tq, dev):
        E, N, K, H = self.E, self.N, self.K, self.HOT
        W = I.student_t_bf16(E * N, K, seed=43).to(dev)
        ng = E * N * (K // 64)
        c = torch.empty(2 * ng * 13, dtype=torch.uint8, device=dev)
        s = torch.empty(2 * ng + 8, dtype=torch.int16, device=dev)
        st = torch.zeros(1, dtype=torch.int32, device=dev)
        tq.tq_quantize_pack(W, 64, 2, c, s, st)
        del W
        c1, s1 = c[:ng * 13], s[:ng]
        c2, s2 = c[ng * 13:ng * 13 + H * self.per * 13], s[ng:ng + H * self.per]
        self.keep = [(c1.clone(), s1.clone(), c2.clone(), s2.clone())
                     for _ in range(self.copies)]
        del c, s
        self.w = [tq.experts_a(a, b, E, N, K, H, cc, d)
                  for a, b, cc, d in self.keep]
        self.ids = self.ids_h.to(dev)
        self.x = I.x_normal(self.TOKENS, K, 47).to(dev)
        self.y = torch.zeros(self.TOKENS, N, device=dev)
        self.pin_io([self.x], [self.y])

    def capture(self, tq):
        calls = [lambda i=i: tq.tq_linear_experts(self.w[i], self.ids, self.x,
                                                  self.y)
                 for i in range(self.copies)]
        return [Step(f"tokens{self.TOKENS}", capture_graph(calls),
                     self.copies * self.call_bytes, self.copies,
                     f"linear_experts_a_tokens{self.TOKENS}",
                     2.0 * self.TOKENS * self.N * self.K * self.copies)]

    def oracle_setup(self):
        from oracle import oref
        self.oref = oref
        # rows 0..63 of a hot and of a cold expert (both planes of the hot)
        rows, K = 64, self.K
        c, s = oref.quantize_pack_A(
            I.bits(I.student_t_bf16(2 * rows, K, seed=43)), 64, 2)
        c, s = np.asarray(c).reshape(2, -1), np.asarray(s).reshape(2, -1)
        per = rows * (K // 64)
        self.pkg_h = (c[0], s[0], c[1][:per * 13], s[1][:per])
        self.xb = I.bits(I.x_normal(2, K, 47))

    def oracle_jobs(self, rows, r0=0):
        c1, s1, c2, s2 = self.pkg_h
        ids = np.array([0, 1], np.int32)
        return [(lambda: self.oref.linear_experts_A(
            c1, s1, c2, s2, 2, 1, 64, self.K, ids, self.xb),
            3 * 64 * (self.K // 64) * 15)]

    def sample_desc(self, rows):
        return "64 rows of a hot and of a cold expert, one token each"


def make_workload(args):
    batches = tuple(args.batch) if args.batch else None
    if args.workload == "decode_step":
        return DecodeStep(batches=batches or I.DECODE_BATCHES)
    if args.workload == "layer":
        return Layer(args.fmt, args.n, args.k, batches or (1,), args.planes,
                     getattr(args, "lut_rows", 0))
    return WORKLOADS[args.workload]()


WORKLOADS = {"fmt_b_4096": FmtB4096, "fmt_b_gemma": FmtBGemma,
             "fmt_a_large": FmtALarge, "decode_step": DecodeStep,
             "fmt_a_small": FmtASmall, "layer": Layer, "encode_b": EncodeB,
             "experts_a": ExpertsA}


# ---- the oracle on the host cores ---------------------------------------------------

def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class OracleRunner:
    """Runs one pass of a workload's oracle sample: on one thread, or with
    the sample's rows split across `threads` host threads (the oracle's C
    calls release the GIL; rows are independent, so the results are the
    same)."""

    def __init__(self, wl, threads):
        import concurrent.futures as cf
        self.wl, self.threads = wl, threads
        self.pool = cf.ThreadPoolExecutor(threads) if threads > 1 else None

    def run(self, rows):
        """One pass over `rows` rows of the sample; returns its bytes."""
        if self.pool is None:
            jobs = self.wl.oracle_jobs(rows, 0)
            for f, _ in jobs:
                f()
            return sum(nb for _, nb in jobs)
        per = max(1, rows // self.threads)
        jobs = []
        for r0 in range(0, rows, per):
            jobs += self.wl.oracle_jobs(min(per, rows - r0), r0)
        for fut in [self.pool.submit(f) for f, _ in jobs]:
            fut.result()
        return sum(nb for _, nb in jobs)

    def close(self):
        if self.pool is not None:
            self.pool.shutdown()


def time_oracle(wl, seconds, threads):
    """Time the oracle on whole passes for about `seconds`: returns (bytes,
    seconds, rows per pass, passes)."""
    runner = OracleRunner(wl, threads)
    rows = min(wl.MAX_ROWS, 8 * threads)
    t0 = time.perf_counter()
    runner.run(rows)
    dt = time.perf_counter() - t0
    rows = int(max(1, min(wl.MAX_ROWS, rows * seconds / max(dt, 1e-6) / 4)))
    total_bytes, t_total, passes = 0, 0.0, 0
    while t_total < seconds:
        t0 = time.perf_counter()
        total_bytes += runner.run(rows)
        t_total += time.perf_counter() - t0
        passes += 1
    runner.close()
    return total_bytes, t_total, rows, passes


def cpu_baseline(wl, seconds):
    """The oracle as it stands, timed on the host: one thread, then all the
    threads this process may run on. The all-threads leg is the value."""
    wl.oracle_setup()
    legs = {}
    for name, threads in (("single_thread", 1), ("all_cores", host_threads())):
        nbytes, secs, rows, passes = time_oracle(wl, seconds, threads)
        legs[name] = {"value": nbytes / secs / 1e9, "cores": threads,
                      "sample": f"{passes} passes over " + wl.sample_desc(rows)
                                + f" ({secs:.1f} s, {threads} thread(s))"}
    top = legs["all_cores"]
    return {"value": top["value"], "unit": "GB/s", "cores": top["cores"],
            "kind": "oracle", "sample": top["sample"],
            "single_thread": legs["single_thread"],
            "cpu_model": cpu_model(),
            "hardware_concurrency": os.cpu_count()}


def run_reference(args, world, rank):
    if rank != 0:
        return
    wl = make_workload(args)
    wl.oracle_setup()
    threads = host_threads()
    runner = OracleRunner(wl, threads)
    # size each step so that the whole run ends within args.ref_seconds
    probe = min(wl.MAX_ROWS, 4 * threads)
    t0 = time.perf_counter()
    runner.run(probe)
    per_row = (time.perf_counter() - t0) / probe
    budget = args.ref_seconds / max(1, args.steps + args.warmup)
    rows = int(max(1, min(wl.MAX_ROWS, budget / max(per_row, 1e-9))))
    for _ in range(args.warmup):
        runner.run(rows)
    t0 = time.perf_counter()
    nbytes = 0
    for _ in range(args.steps):
        nbytes += runner.run(rows)
    dt = time.perf_counter() - t0
    runner.close()
    value = nbytes / dt / 1e9
    sample = wl.sample_desc(rows) + f" per step, {threads} host thread(s)"
    line = {"impl": "reference", "metric": METRIC, "value": value,
            "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "config": wl.describe(),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads,
                             "kind": "oracle", "sample": sample,
                             "cpu_model": cpu_model()},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_tq(args, world, rank, local):
    from packed_weight_matmul_b200 import tq
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = make_workload(args)
    wl.setup(tq, dev)
    if args.force_path:
        tq.tq_testing_force_linear_path(args.force_path)
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

    # read-only streaming reference on this GPU, in the same run
    read_ref = hbm_read_reference()

    if rank != 0:
        return
    pk = peaks()
    # dominant kernel: the graph with the largest share of the step
    dom = int(np.argmax(per))
    s = steps[dom]
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": wl.describe(),
        "pct_hbm_peak": 100.0 * value / world / pk["hbm_gbs"],
        "pct_hbm_nominal": 100.0 * value / world / HBM_NOMINAL_GBS,
        "hbm_read_ref": read_ref,
        "pct_hbm_read_ref": (100.0 * value / world / read_ref["gbs"]
                             if read_ref.get("gbs") else None),
        "roofline": roofline(s, per[dom], pk, wl),
        "per_graph_ms": {st.name: float(p) for st, p in zip(steps, per)},
        "per_graph_gbs": {st.name: st.bytes / (p / 1e3) / 1e9
                          for st, p in zip(steps, per)},
        "per_graph_roof_frac": {st.name: roofline(st, p, pk, wl)["frac"]
                                for st, p in zip(steps, per)},
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "clocks": clk,
        "gpu_launches": int(sum(st.launches for st in steps) * args.steps),
    }
    if args.force_path:
        line["config"]["forced_path"] = {1: "cuda cores",
                                         2: "tensor cores"}[args.force_path]
    if hasattr(wl, "extra"):
        line.update(wl.extra(steps, per))
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds)
    print(json.dumps(line), flush=True)


HBM_NOMINAL_GBS = 8000.0  # B200 HBM3e, nominal


def hbm_read_reference(nbytes=2 ** 31, reps=5):
    """Read bandwidth of this GPU measured in the same run: a torch fp32
    reduction over a 2 GiB buffer (it reads every byte once and writes one
    value), CUDA events, median of `reps` after two warm-up passes. A
    measurement reference for the % figures, not part of the library."""
    try:
        buf = torch.ones(nbytes // 4, dtype=torch.float32, device="cuda")
        for _ in range(2):
            buf.sum()
        times = []
        for _ in range(reps):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            buf.sum()
            b.record()
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b))
        del buf
        torch.cuda.empty_cache()
        t_ms = float(np.median(times))
        return {"gbs": nbytes / (t_ms / 1e3) / 1e9, "bytes": nbytes,
                "method": "torch.sum over a 2 GiB fp32 buffer (read once), "
                          "CUDA events, median of 5"}
    except Exception as e:  # the reference is optional; the line is not
        return {"gbs": None, "error": str(e)[:200]}


def roofline(step, ms, pk, wl):
    """Roofline of one graph's kernel: achieved = its algorithmic bytes (or
    flops) per launch / its average CUDA-event launch time, against the lower
    of the HBM roof (measured copy bandwidth) and the tensor roof (sustained
    dense bf16 throughput, expressed in packed bytes through the graph's
    flops per byte)."""
    per_launch_s = ms / 1e3 / step.launches
    bytes_per_launch = step.bytes / step.launches
    flops_per_launch = step.flops / step.launches
    hbm = pk["hbm_gbs"]
    tensor_tflops = pk["bf16_tflops_sustained"]
    tensor_gbs = (tensor_tflops * 1e12 * bytes_per_launch / flops_per_launch
                  / 1e9 if flops_per_launch > 0 else float("inf"))
    traffic = ncu_traffic(step.kernel, wl.SOURCES, bytes_per_launch)
    out = {"traffic": traffic, "kernel": step.kernel, "peak_src": pk["src"],
           "algorithmic_bytes_per_launch": bytes_per_launch,
           "algorithmic_flops_per_launch": flops_per_launch,
           "launch_us": per_launch_s * 1e6}
    if tensor_gbs < hbm:
        achieved = flops_per_launch / per_launch_s / 1e12
        out.update({"bound": "tensor", "achieved": achieved,
                    "peak": tensor_tflops, "unit": "TFLOP/s",
                    "frac": achieved / tensor_tflops,
                    "peak_kind": "dense bf16, sustained"})
    else:
        achieved = bytes_per_launch / per_launch_s / 1e9
        out.update({"bound": "hbm", "achieved": achieved, "peak": hbm,
                    "unit": "GB/s", "frac": achieved / hbm,
                    "peak_kind": "HBM copy"})
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["tq", "reference"], default="tq")
    ap.add_argument("--workload", choices=sorted(WORKLOADS),
                    default="decode_step")
    ap.add_argument("--batch", type=int, nargs="+", default=None,
                    help="batches of the decode_step and layer workloads "
                         "(default 1 4 16 64 and 1)")
    ap.add_argument("--fmt", choices=["A", "B", "B7", "a", "b", "b7"],
                    default="B",
                    help="layer workload: weight format")
    ap.add_argument("--n", type=int, default=8192, help="layer workload: rows")
    ap.add_argument("--k", type=int, default=5376,
                    help="layer workload: columns")
    ap.add_argument("--planes", type=int, default=1,
                    help="layer workload: Format A planes")
    ap.add_argument("--force-path", type=int, default=0, choices=[0, 1, 2, 3],
                    help="kernel family for comparisons: 0 automatic, "
                         "1 CUDA cores, 2 tensor cores")
    ap.add_argument("--lut-rows", type=int, default=0,
                    help="layer workload, Format B: rows per code book "
                         "(adaptive alphabet); 0 = one code book")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-seconds", type=float, default=90.0,
                    help="host time the reference arm spends in total")
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

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

    def oracle_pass(self, rows):
        """One oracle pass over `rows` rows at every batch; returns bytes."""
        for b in self.BATCHES:
            self.oref.linear_B(self.codes_h[:rows], self.lut_h, self.xb_h[b])
        return len(self.BATCHES) * rows * self.K

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

    def oracle_pass(self, rows):
        for b in self.BATCHES:
            self.oref.linear_B(self.codes_h[:rows], self.lut_h, self.xb_h[b],
                               self.rho_h, 1)
        return len(self.BATCHES) * rows * self.K

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

    def oracle_pass(self, rows):
        rows = min(rows, 64)
        codes, scales = self.oref.quantize_pack_A(self.Wh[:rows], self.G, 2)
        nbytes = 2 * rows * self.K + 2 * rows * (self.K // self.G) * 15
        for p in (1, 2):
            for b in self.BATCHES:
                self.oref.linear_A(codes[:p], scales[:p], rows, self.K,
                                   self.xb_h[b], self.G, p)
                nbytes += p * rows * (self.K // self.G) * 15
        return nbytes

    def sample_desc(self, rows):
        return (f"{min(rows, 64)} rows x 8192 of the Format A workload: "
                "quantize both planes, then linear with 1 and 2 planes at "
                "batch 1, 8, 32, 64")


class DecodeStep(Workload):
    """60 blocks x {q, k, v 8192x5376; o 5376x8192; gate, up 21504x5376; down
    5376x21504} Format B layers (31.4 GB of codes), alpha 0.02, no rho, one
    x per distinct k, at one batch (--batch, default 1). One step = the 420
    ordered tq_linear calls; tokens/s = batch / step time."""
    name = "decode_step"
    SOURCES = Workload.SOURCES
    MAX_ROWS = 256

    def __init__(self, batch=1, blocks=I.GEMMA_BLOCKS):
        self.batch = batch
        self.blocks = blocks
        self.BATCHES = (batch,)

    def describe(self):
        return {"workload": f"{self.name}: {self.blocks} blocks x 7 Format B "
                "layers (q,k,v 8192x5376; o 5376x8192; gate,up 21504x5376; "
                "down 5376x21504), codes uniform 0..242, alpha=0.02, no rho; "
                f"x bf16 N(0,1) at batch {self.batch}",
                "bytes_resident": sum(l.n * l.k for _, l in
                                      I.decode_step_layers(self.blocks)),
                "l2": "31.4 GB resident: every launch reads from HBM",
                "batches": [self.batch], "parallelism": "replicas"}

    def setup(self, tq, dev):
        lut = tq.tq_build_lut(I.ALPHA, I.ladder_pow3().numpy())
        self.lut_d = torch.from_numpy(lut).to(dev)
        self.layers = I.decode_step_layers(self.blocks)
        self.codes = [I.codes_uniform(l.n, l.k, s, device=dev)
                      for s, l in self.layers]
        self.w = [tq.weights_b(c, self.lut_d) for c in self.codes]
        ks = sorted({l.k for _, l in self.layers})
        self.x = {k: I.x_normal(self.batch, k, 50 + k % 97).to(dev)
                  for k in ks}
        self.y = [torch.zeros(self.batch, l.n, device=dev)
                  for _, l in self.layers]
        self.pin_io(list(self.x.values()), self.y)

    def capture(self, tq):
        calls = [lambda i=i, l=l: tq.tq_linear(self.w[i], self.x[l.k],
                                                self.y[i])
                 for i, (_, l) in enumerate(self.layers)]
        nbytes = sum(l.n * l.k + 972 for _, l in self.layers)
        return [Step(f"batch{self.batch}", capture_graph(calls), nbytes,
                     len(calls), f"linear_b_decode_batch{self.batch}",
                     2.0 * self.batch * sum(l.n * l.k for _, l in
                                            self.layers))]

    def oracle_setup(self):
        from oracle import oref
        self.oref = oref
        self.sample = [(l, I.codes_uniform(256, l.k, s).numpy())
                       for s, l in I.decode_step_layers(1)]
        self.lut_h = oref.build_lut(I.ALPHA, I.ladder_pow3().numpy())
        self.xb = {l.k: I.bits(I.x_normal(self.batch, l.k, 1))
                   for l, _ in self.sample}

    def oracle_pass(self, rows):
        rows = min(rows, 256)
        nbytes = 0
        for l, codes in self.sample:
            self.oref.linear_B(codes[:rows], self.lut_h, self.xb[l.k])
            nbytes += rows * l.k
        return nbytes

    def sample_desc(self, rows):
        return (f"{min(rows, 256)} rows of each of the 7 layer shapes of one "
                f"block at batch {self.batch}")


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

    def oracle_pass(self, rows):
        rows = min(rows, 512)
        codes, scales = self.oref.quantize_pack_A(self.Wh[:rows], 64, 1)
        self.oref.linear_A(codes, scales, rows, 1024, self.xb)
        return rows * 1024 * 2 + 2 * rows * 16 * 15

    def sample_desc(self, rows):
        return f"{min(rows, 512)} rows of the 512x1024 workload"


def make_workload(args):
    if args.workload == "decode_step":
        return DecodeStep(batch=args.batch)
    return WORKLOADS[args.workload]()


WORKLOADS = {"fmt_b_4096": FmtB4096, "fmt_b_gemma": FmtBGemma,
             "fmt_a_large": FmtALarge, "decode_step": DecodeStep,
             "fmt_a_small": FmtASmall}


# ---- the two arms ------------------------------------------------------------------------

def time_oracle(wl, seconds):
    """Time the single-threaded oracle for about `seconds` on whole passes."""
    wl.oracle_setup()
    rows = 64
    t0 = time.perf_counter()
    wl.oracle_pass(rows)
    dt = time.perf_counter() - t0
    rows = int(max(1, min(wl.MAX_ROWS, rows * seconds / max(dt, 1e-6) / 4)))
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
    wl = make_workload(args)
    wl.oracle_setup()
    # size each step so the whole run ends within about two minutes
    t0 = time.perf_counter()
    wl.oracle_pass(16)
    per_row = (time.perf_counter() - t0) / 16
    budget = args.ref_seconds / max(1, args.steps + args.warmup)
    rows = int(max(1, min(wl.MAX_ROWS, budget / max(per_row, 1e-9))))
    for _ in range(args.warmup):
        wl.oracle_pass(rows)
    t0 = time.perf_counter()
    nbytes = 0
    for _ in range(args.steps):
        nbytes += wl.oracle_pass(rows)
    dt = time.perf_counter() - t0
    value = nbytes / dt / 1e9
    sample = wl.sample_desc(rows) + " per step"
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
    wl = make_workload(args)
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
    if isinstance(wl, DecodeStep):
        line["tokens_per_s"] = world * wl.batch * args.steps / (elapsed_ms / 1e3)
        line["e2e_tokens_per_s"] = world * wl.batch * args.steps / (e2e_ms / 1e3)
    if world == 1 and not args.no_cpu_baseline:
        nbytes, secs, rows, passes = time_oracle(wl, args.cpu_seconds)
        line["cpu_baseline"] = {
            "value": nbytes / secs / 1e9, "unit": "GB/s", "cores": 1,
            "kind": "oracle",
            "sample": f"{passes} passes over " + wl.sample_desc(rows) +
                      f" "
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
    ap.add_argument("--batch", type=int, default=1,
                    help="batch of the decode_step workload")
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

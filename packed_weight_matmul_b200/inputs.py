"""Seeded synthetic inputs shaped like the pages' workloads.

This module only draws random numbers and lays them out; it holds none of the
packing, decoding or matmul arithmetic. The same arrays feed the CUDA library
and the CPU oracle. Random draws use torch's CPU generator (normal, uniform,
integer) or numpy's PCG64 generator (Student-t); fp32 samples become bf16 or
fp16 through torch's own round-to-nearest-even conversion.

Workloads (layer shapes follow the Gemma-4-31B-it linear layers of "A Discrete
Weight Language for Large Language Models", section 6.1: hidden 5376,
intermediate 21504, 60 blocks):

  fmt_a_small   W 512 x 1024 bf16 = bf16(0.02 N(0,1)), 1 % of entries x10,
                one all-zero 64-group per 64-row block; x 1 x 1024 N(0,1).
  fmt_b_4096    codes 4096 x 4096 uniform on 0..242, ladder a_k = 3^-(k-1),
                alpha 0.02, no rho; x at batch 1 and 4.
  fmt_b_gemma   rho ~ fp16(U(0.5, 1.5)); up 21504 x 5376 and down 5376 x 21504
                with one rho per row; q, k, v 8192 x 5376 with one rho per
                128-row head; x at batch 1, 4 and 16.
  fmt_a_large   W 28672 x 8192 = bf16(0.02 StudentT(nu=5)), G = 64, one or two
                planes; x at batch 1, 8, 32 and 64.
  decode_step   60 blocks x {q, k, v 8192 x 5376; o 5376 x 8192; gate, up
                21504 x 5376; down 5376 x 21504}, codes uniform on 0..242 per
                layer, alpha 0.02, no rho; x at batch 1, 4, 16 and 64.
"""
from dataclasses import dataclass
from typing import List, Tuple

import numpy as np
import torch

SEEDS = {"fmt_a_small": 0, "fmt_b_4096": 1, "fmt_b_gemma": 2,
         "fmt_a_large": 3, "decode_step": 4}


def generator(seed: int) -> torch.Generator:
    return torch.Generator().manual_seed(int(seed))


def to_bf16(t: torch.Tensor) -> torch.Tensor:
    return t.to(torch.float32).to(torch.bfloat16)


def bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a bf16 / fp16 tensor (for the oracle)."""
    assert t.dtype in (torch.bfloat16, torch.float16)
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def ladder_pow3() -> torch.Tensor:
    """a_k = fp32(3^-(k-1)), k = 1..5."""
    return torch.tensor([3.0 ** -(k - 1) for k in range(1, 6)],
                        dtype=torch.float64).to(torch.float32)


def x_normal(batch: int, k: int, seed: int) -> torch.Tensor:
    return to_bf16(torch.randn(batch, k, generator=generator(seed)))


def codes_uniform(n: int, k: int, seed: int, device="cpu") -> torch.Tensor:
    g = torch.Generator(device=device).manual_seed(int(seed))
    return torch.randint(0, 243, (n, k), generator=g, dtype=torch.uint8,
                         device=device)


def rho_uniform(count: int, seed: int) -> torch.Tensor:
    u = torch.rand(count, generator=generator(seed))
    return (0.5 + u).to(torch.float16)


# ---- format A, small: 512 x 1024 ----------------------------------------

def fmt_a_small(seed: int = SEEDS["fmt_a_small"], n=512, k=1024, G=64):
    g = generator(seed)
    w = 0.02 * torch.randn(n, k, generator=g)
    mask = torch.rand(n, k, generator=g) < 0.01
    w = torch.where(mask, w * 10.0, w)
    zero_groups = []
    for blk in range(0, n, 64):
        rows = min(64, n - blk)
        r = blk + int(torch.randint(0, rows, (1,), generator=g))
        gi = int(torch.randint(0, k // G, (1,), generator=g))
        w[r, gi * G:(gi + 1) * G] = 0.0
        zero_groups.append((r, gi))
    x = torch.randn(1, k, generator=g)
    return {"W": to_bf16(w), "x": to_bf16(x), "G": G,
            "zero_groups": zero_groups}


# ---- format A, large: Student-t ------------------------------------------

def student_t_bf16(n: int, k: int, seed: int, scale=0.02, nu=5.0,
                   chunk_rows=2048) -> torch.Tensor:
    rng = np.random.Generator(np.random.PCG64(seed))
    out = torch.empty(n, k, dtype=torch.bfloat16)
    for r0 in range(0, n, chunk_rows):
        r1 = min(n, r0 + chunk_rows)
        t = rng.standard_t(nu, size=(r1 - r0, k)).astype(np.float32)
        out[r0:r1] = to_bf16(torch.from_numpy(t) * scale)
    return out


def fmt_a_large(seed: int = SEEDS["fmt_a_large"], n=28672, k=8192):
    return {"W": student_t_bf16(n, k, seed), "G": 64,
            "batches": (1, 8, 32, 64)}


# ---- format B ---------------------------------------------------------------

ALPHA = 0.02


def fmt_b_4096(seed: int = SEEDS["fmt_b_4096"], n=4096, k=4096):
    return {"codes": codes_uniform(n, k, seed), "alpha": ALPHA,
            "ladder": ladder_pow3(), "batches": (1, 4)}


@dataclass
class Layer:
    name: str
    n: int
    k: int
    rps: int = 0  # rows per rho scale; 0 = no rho


GEMMA_HIDDEN, GEMMA_INTER, GEMMA_QKV_ROWS, GEMMA_BLOCKS = 5376, 21504, 8192, 60
HEAD_ROWS = 128

FMT_B_GEMMA_LAYERS = [
    Layer("up", GEMMA_INTER, GEMMA_HIDDEN, 1),
    Layer("down", GEMMA_HIDDEN, GEMMA_INTER, 1),
    Layer("q", GEMMA_QKV_ROWS, GEMMA_HIDDEN, HEAD_ROWS),
    Layer("k", GEMMA_QKV_ROWS, GEMMA_HIDDEN, HEAD_ROWS),
    Layer("v", GEMMA_QKV_ROWS, GEMMA_HIDDEN, HEAD_ROWS),
]


def rho_count(n: int, rps: int) -> int:
    return 0 if rps == 0 else (n + rps - 1) // rps


def fmt_b_gemma_layer(layer: Layer, seed: int = SEEDS["fmt_b_gemma"]):
    idx = [l.name for l in FMT_B_GEMMA_LAYERS].index(layer.name)
    s = seed * 1000 + idx
    return {"codes": codes_uniform(layer.n, layer.k, s),
            "rho": rho_uniform(rho_count(layer.n, layer.rps), s + 500),
            "rps": layer.rps, "alpha": ALPHA, "ladder": ladder_pow3(),
            "batches": (1, 4, 16)}


BLOCK_LAYERS = [
    Layer("q", GEMMA_QKV_ROWS, GEMMA_HIDDEN),
    Layer("k", GEMMA_QKV_ROWS, GEMMA_HIDDEN),
    Layer("v", GEMMA_QKV_ROWS, GEMMA_HIDDEN),
    Layer("o", GEMMA_HIDDEN, GEMMA_QKV_ROWS),
    Layer("gate", GEMMA_INTER, GEMMA_HIDDEN),
    Layer("up", GEMMA_INTER, GEMMA_HIDDEN),
    Layer("down", GEMMA_HIDDEN, GEMMA_INTER),
]


def decode_step_layers(blocks: int = GEMMA_BLOCKS) -> List[Tuple[int, Layer]]:
    """(layer seed, layer) for every linear of the decode step, in order."""
    out = []
    base = SEEDS["decode_step"] * 100000
    for b in range(blocks):
        for j, l in enumerate(BLOCK_LAYERS):
            out.append((base + b * len(BLOCK_LAYERS) + j, l))
    return out


DECODE_BATCHES = (1, 4, 16, 64)

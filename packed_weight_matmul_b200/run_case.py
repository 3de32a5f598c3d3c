"""Run one tq_linear configuration a few times on cuda:0, for profilers.

    python -m packed_weight_matmul_b200.run_case b 4096 4096 4 [reps]
    python -m packed_weight_matmul_b200.run_case a1 28672 8192 1 [reps]

Format b: uint8 codes uniform on 0..242 with the 3^-(k-1) ladder code book
(alpha 0.02, no rho). Format aP (P planes, G = 64): codes uniform on
0..242 and fp16 scales uniform on [0.01, 0.02). x is bf16 N(0,1). Every
launch reads the same weights; profilers flush caches between their passes.
"""
import sys

import torch

from . import inputs as I
from . import tq


def main(argv):
    fmt, n, k, batch = argv[0], int(argv[1]), int(argv[2]), int(argv[3])
    reps = int(argv[4]) if len(argv) > 4 else 3
    dev = torch.device("cuda:0")
    if fmt == "b":
        lut = torch.from_numpy(tq.tq_build_lut(I.ALPHA, I.ladder_pow3().numpy()))
        codes = I.codes_uniform(n, k, 5, device=dev)
        w = tq.weights_b(codes, lut.to(dev))
    elif fmt.startswith("a"):
        planes = int(fmt[1:]) if len(fmt) > 1 else 1
        G = 64
        gen = torch.Generator(device="cpu").manual_seed(7)
        codes = torch.randint(0, 243, (planes * n * (k // G) * 13,),
                              dtype=torch.uint8, generator=gen).to(dev)
        scales = (0.01 + 0.01 * torch.rand(planes * n * (k // G), generator=gen)
                  ).half().view(torch.int16).to(dev)
        w = tq.weights_a(codes, scales, n, k, G, planes)
    else:
        raise SystemExit(f"unknown format {fmt!r}")
    x = I.x_normal(batch, k, 1).to(dev)
    y = torch.empty(batch, n, device=dev)
    for _ in range(reps):
        tq.tq_linear(w, x, y)
    torch.cuda.synchronize()
    print("ok", float(y.abs().sum()))


if __name__ == "__main__":
    main(sys.argv[1:])

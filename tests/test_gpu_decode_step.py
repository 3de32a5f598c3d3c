"""GPU parity for the 60-block decode step's layer shapes and the empty-K edge.

The decode step (Gemma-4-31B-shaped linear layers of "A Discrete Weight
Language for Large Language Models", section 6.1) runs q/k/v 8192 x 5376,
o 5376 x 8192, gate/up 21504 x 5376 and down 5376 x 21504 in Format B with the
3^-(k-1) ladder, at batch 1, 4, 16 and 64. One layer of each shape, with
uniform seeded codes drawn here on the host (the bench draws its codes on the
device, from the same distribution), is checked on 64 seeded rows (the last
row included) against the fp64 oracle, through the same dispatch and launch
configuration the bench times at that shape and batch."""
import numpy as np
import pytest
import torch

from oracle import oref
from packed_weight_matmul_b200 import inputs as I
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lut():
    return oref.build_lut(I.ALPHA, I.ladder_pow3().numpy())


def _first_of_each_shape():
    seen, out = set(), []
    for seed, layer in I.decode_step_layers(1):
        if (layer.n, layer.k) not in seen:
            seen.add((layer.n, layer.k))
            out.append((seed, layer))
    return out


@pytest.mark.parametrize("seed,layer", _first_of_each_shape(),
                         ids=lambda v: getattr(v, "name", str(v)))
def test_decode_step_layer_sampled(lut, seed, layer):
    codes = I.codes_uniform(layer.n, layer.k, seed)
    w = U.weights_b_dev(codes, lut)
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(layer.n, 64, replace=False))
    rows[-1] = layer.n - 1
    codes_np = codes.numpy()
    absmax = U.absmax_rows_b(codes_np, lut, rows=rows)
    for batch in I.DECODE_BATCHES:
        x = I.x_normal(batch, layer.k, 50 + batch)
        xb = U.x_bits(x)
        y, _ = U.linear(w, x)
        ref = oref.linear_B(codes_np, lut, xb, None, 0, rows=rows)
        U.check_tolerance(y[:, rows], ref, xb, absmax,
                          f"decode {layer.name} b={batch}")


@pytest.mark.parametrize("fmt", ["A", "B"])
def test_empty_k_gives_zeros_and_keeps_padding(lut, fmt):
    n = 40
    # K = 0: valid (aligned, non-null) buffers that nothing may read
    dummy = torch.zeros(16, dtype=torch.uint8, device=U.DEV)
    if fmt == "A":
        sc = torch.zeros(8, dtype=torch.int16, device=U.DEV)
        w = U.tq().weights_a(dummy, sc, n, 0, 64, 1)
    else:
        L = torch.from_numpy(np.ascontiguousarray(lut, np.float32)).to(U.DEV)
        w = U.tq().weights_b(dummy, L, n=n, k=0)
    for batch in (1, 5, 64):
        ldy = n + 8
        y = torch.full((batch, ldy), -3.0, dtype=torch.float32, device=U.DEV)
        xd = torch.zeros(batch, 8, dtype=torch.bfloat16, device=U.DEV)
        U.tq().tq_linear(w, xd, y, batch=batch, ldx=8, ldy=ldy)
        torch.cuda.synchronize()
        yh = y.cpu().numpy()
        assert np.all(yh[:, :n] == 0.0)
        assert np.all(yh[:, n:] == -3.0)

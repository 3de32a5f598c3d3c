"""GPU parity of the adaptive alphabet (alphaneural.io page, section 8.3):
one Format B code book per block of lut_rows rows. tq_linear against the
fp64 oracle with per-block books (same tolerance as test_gpu_linear):
- block sizes that are multiples of 32 take the tensor-core kernel at every
  batch, with compact per-warp books;
- the others take the one-warp-per-row kernel;
- per-row books, rho, ragged rows and an invalid code are covered;
- tq_unpack is bit-exact against the oracle."""
import numpy as np
import pytest
import torch

from oracle import oref
from packed_weight_matmul_b200 import inputs as I
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


def _books(n, lut_rows, seed):
    """One ladder per block, amplitudes U(0.01, 1), alpha 0.02."""
    rng = np.random.default_rng(seed)
    nb = -(-n // lut_rows)
    ladders = rng.uniform(0.01, 1.0, (nb, 5)).astype(np.float32)
    return np.stack([oref.build_lut(np.float32(0.02), ladders[b])
                     for b in range(nb)])


def _weights(codes, luts, lut_rows, rho=None, rps=0):
    c = codes.to(U.DEV)
    L = torch.from_numpy(np.ascontiguousarray(luts.reshape(-1))).to(U.DEV)
    r = None
    if rho is not None:
        r = rho.view(torch.int16).to(U.DEV)
    n, k = codes.shape
    return U.tq().weights_b(c, L, r, rps, n=n, k=k, lut_rows=lut_rows)


@pytest.mark.parametrize("n,k,lut_rows,rps", [
    (300, 2064, 32, 0), (257, 4096, 64, 1), (130, 5376, 128, 128),
    (70, 528, 7, 0), (64, 64, 1, 1), (33, 1040, 32, 0)])
def test_adaptive_linear(n, k, lut_rows, rps):
    luts = _books(n, lut_rows, n + k)
    codes = I.codes_uniform(n, k, n * 3 + k)
    rho = I.rho_uniform(I.rho_count(n, rps), 2) if rps else None
    rho_bits = I.bits(rho) if rps else None
    w = _weights(codes, luts, lut_rows, rho, rps)
    absmax = np.abs(oref.weights_B(codes.numpy(), luts, rho_bits, rps,
                                   lut_rows=lut_rows)).max(axis=1)
    for batch in (1, 3, 4, 8, 16, 64):
        x = I.x_normal(batch, k, batch + 3)
        xb = U.x_bits(x)
        y, _ = U.linear(w, x)
        ref = oref.linear_B(codes.numpy(), luts, xb, rho_bits, rps,
                            lut_rows=lut_rows)
        U.check_tolerance(y, ref, xb, absmax,
                          f"adaptive {n}x{k} rows/book={lut_rows} b={batch}")


def test_adaptive_invalid_code_poisons_row():
    n, k = 128, 512
    luts = _books(n, 32, 4)
    codes = I.codes_uniform(n, k, 6)
    codes[40, 3] = 250
    w = _weights(codes, luts, 32)
    for batch in (1, 16):
        y, _ = U.linear(w, I.x_normal(batch, k, 2))
        assert np.all(np.isnan(y[:, 40]))
        assert np.all(np.isfinite(np.delete(y, 40, axis=1)))


@pytest.mark.parametrize("lut_rows", [1, 7, 32])
def test_adaptive_unpack_bit_exact(lut_rows):
    n, k = 100, 272
    luts = _books(n, lut_rows, 9)
    codes = I.codes_uniform(n, k, 10)
    rho = I.rho_uniform(I.rho_count(n, 1), 3)
    w = _weights(codes, luts, lut_rows, rho, 1)
    out = torch.empty(n, k, dtype=torch.int16, device=U.DEV)
    U.tq().tq_unpack(w, out)
    torch.cuda.synchronize()
    ref = oref.unpack_B(codes.numpy(), luts, I.bits(rho), 1,
                        lut_rows=lut_rows)
    assert np.array_equal(out.cpu().numpy().view(np.uint16), ref)

"""GPU parity of the two Format B operand paths of the tensor-core kernel.

A code book whose entries are all integer multiples m of one unit u (|m| <=
256, to 2^-20 of each entry) is decoded to the single exact operand bf16(m),
with u applied to the accumulator; any other code book is split into a bf16
hi + lo pair. These tests run both paths against the fp64 oracle (same
tolerance as test_gpu_linear), force the hi + lo path on a code book that
would take the single path (tq_testing_force_linear_path(3)), and check that
an entry just off the grid is not forced onto it: with every code of a row
equal and x all ones, an entry rounded onto the grid would miss by about
1e-3 * K * |w|, far outside the tolerance. A book with entry c = u * (c - 121)
(an ascending ternary ladder 1/81 .. 1, any alpha: the least significant trit
on the smallest step) is decoded without its table; every invalid byte value
243..255 must still make its row NaN on each path."""
import numpy as np
import pytest
import torch

from oracle import oref
from packed_weight_matmul_b200 import inputs as I
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

BATCHES = (5, 16, 33, 64)
# a ladder whose 243 sums are not on one grid (the encoder's test ladder)
LADDER_FREE = np.array([1.0, 0.33, 0.115, 0.037, 0.012], np.float32)
# an ascending ternary ladder: entry c = alpha * (c - 121) / 81
LADDER_ASC = np.array([1 / 81, 1 / 27, 1 / 9, 1 / 3, 1], np.float32)


@pytest.fixture
def force_path():
    def set_path(p):
        U.tq().tq_testing_force_linear_path(p)
    yield set_path
    U.tq().tq_testing_force_linear_path(0)


def _run(codes, lut, rho=None, rps=0, batches=BATCHES, seed=0, label=""):
    rho_bits = I.bits(rho) if rho is not None else None
    w = U.weights_b_dev(codes, lut, rho, rps)
    absmax = U.absmax_rows_b(codes.numpy(), lut, rho_bits, rps)
    for batch in batches:
        x = I.x_normal(batch, codes.shape[1], seed + batch)
        xb = U.x_bits(x)
        y, _ = U.linear(w, x)
        ref = oref.linear_B(codes.numpy(), lut, xb, rho_bits, rps)
        U.check_tolerance(y, ref, xb, absmax, f"{label} b={batch}")


@pytest.mark.parametrize("n,k,rps", [(130, 5376, 1), (300, 2064, 0),
                                     (257, 4096, 128)])
def test_off_grid_ladder_uses_hi_lo(n, k, rps):
    lut = oref.build_lut(I.ALPHA, LADDER_FREE)
    codes = I.codes_uniform(n, k, n + k)
    rho = I.rho_uniform(I.rho_count(n, rps), 3) if rps else None
    _run(codes, lut, rho, rps, label=f"free ladder {n}x{k}")


@pytest.mark.parametrize("path", [2, 3])
def test_grid_ladder_both_paths(force_path, path):
    lut = oref.build_lut(I.ALPHA, I.ladder_pow3().numpy())
    codes = I.codes_uniform(300, 4224, 77)
    force_path(path)
    _run(codes, lut, label=f"pow3 path {path}")


@pytest.mark.parametrize("path", [0, 3])
def test_entry_off_grid_is_not_rounded_onto_it(force_path, path):
    lut = oref.build_lut(I.ALPHA, I.ladder_pow3().numpy()).copy()
    lut[200] = np.float32(lut[200] * np.float32(1.001))
    n, k = 256, 4096
    codes = I.codes_uniform(n, k, 5)
    codes[7, :] = 200  # one row of a single code
    force_path(path)
    w = U.weights_b_dev(codes, lut)
    absmax = U.absmax_rows_b(codes.numpy(), lut)
    for batch in (8, 64):
        x = torch.ones(batch, k, dtype=torch.bfloat16)
        xb = U.x_bits(x)
        y, _ = U.linear(w, x)
        ref = oref.linear_B(codes.numpy(), lut, xb)
        U.check_tolerance(y, ref, xb, absmax, f"off-grid entry b={batch}")


def test_integer_ladder_and_zero_book():
    # ladder 81, 27, 9, 3, 1: the entries are the integers -121..121 * alpha
    lut = oref.build_lut(np.float32(0.75),
                         np.array([81, 27, 9, 3, 1], np.float32))
    codes = I.codes_uniform(200, 1040, 9)
    _run(codes, lut, batches=(6, 64), label="integer ladder")
    # alpha = 0: every entry is zero, and so is every output
    zero = oref.build_lut(np.float32(0.0), I.ladder_pow3().numpy())
    w = U.weights_b_dev(codes, zero)
    for batch in (6, 64):
        y, _ = U.linear(w, I.x_normal(batch, 1040, batch))
        assert np.all(y == 0.0)


@pytest.mark.parametrize("ladder,path", [("pow3", 0), ("pow3", 3),
                                         ("free", 0), ("asc", 0), ("asc", 3)])
def test_every_invalid_code_poisons_its_row(force_path, ladder, path):
    # one invalid byte (243..255) per row in rows 0..12, at k positions that
    # fall in both 64-k halves of a block, in different blocks and at the
    # last k; the ascending ternary ladder takes the table-free decode
    # (path 0), the ladder 3^-(k-1) the single-operand table (path 0) or the
    # hi + lo table (path 3), the free ladder the hi + lo table
    lad = {"pow3": I.ladder_pow3().numpy(), "free": LADDER_FREE,
           "asc": LADDER_ASC}[ladder]
    lut = oref.build_lut(I.ALPHA, lad)
    n, k = 141, 1024
    codes = I.codes_uniform(n, k, 31)
    bad_rows = list(range(13))
    for i in bad_rows:
        kk = k - 1 if i == 12 else (77 * i + 64 * (i % 2)) % k
        codes[i, kk] = 243 + i
    force_path(path)
    w = U.weights_b_dev(codes, lut)
    for batch in (5, 16, 64):
        y, _ = U.linear(w, I.x_normal(batch, k, batch))
        assert np.all(np.isnan(y[:, bad_rows])), f"b={batch}"
        assert np.all(np.isfinite(np.delete(y, bad_rows, axis=1))), f"b={batch}"


@pytest.mark.parametrize("path", [0, 3])
def test_integer_grid_that_is_not_the_ternary_ladder(force_path, path):
    # ladder 5, 4, 3, 2, 1: every entry is alpha times an integer (|m| <= 15)
    # but not alpha * (c - 121) / 81: the single-operand table path (path 0)
    # or the hi + lo pair (path 3)
    lut = oref.build_lut(I.ALPHA, np.array([5, 4, 3, 2, 1], np.float32))
    codes = I.codes_uniform(300, 2064, 17)
    force_path(path)
    _run(codes, lut, rho=I.rho_uniform(300, 4), rps=1,
         label=f"ladder 5..1 path {path}")


@pytest.mark.parametrize("path", [0, 3])
@pytest.mark.parametrize("n,k,rps", [(300, 2064, 0), (257, 4096, 1),
                                     (1000, 2048, 128)])
def test_ascending_ternary_ladder_table_free(force_path, path, n, k, rps):
    # entry c = alpha * (c - 121) / 81: the table-free decode (path 0) and the
    # hi + lo table (path 3), ragged rows and blocks, rho per row and per head
    lut = oref.build_lut(I.ALPHA, LADDER_ASC)
    m = np.rint(lut[:243] / (I.ALPHA / 81)).astype(np.int64)
    assert np.array_equal(m, np.arange(243) - 121)  # the book is c - 121
    codes = I.codes_uniform(n, k, n + 3 * k)
    rho = I.rho_uniform(I.rho_count(n, rps), 6) if rps else None
    force_path(path)
    _run(codes, lut, rho, rps, label=f"ascending ladder path {path} {n}x{k}")

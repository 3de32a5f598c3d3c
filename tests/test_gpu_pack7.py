"""GPU parity of the 7-bit truncated alphabet (alphaneural.io page, section
8.1): tq_pack7 bit-exact against the oracle (used-code table, count, packed
indices), the more-than-128-words status, tq_linear on a 7-bit layer against
the fp64 oracle (same tolerance as test_gpu_linear) through the
one-warp-per-row kernel and, for K a multiple of 128, the tensor-core kernel
(single-operand and hi + lo books, rho, ragged rows), and bit-exact unpack."""
import numpy as np
import pytest
import torch

from oracle import oref
from packed_weight_matmul_b200 import inputs as I
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


def _codes(n, k, distinct, seed):
    rng = np.random.default_rng(seed)
    words = rng.choice(243, distinct, replace=False)
    c = rng.choice(words, (n, k)).astype(np.uint8)
    c.reshape(-1)[:distinct] = words
    return c


def _pack_gpu(codes):
    n, k = codes.shape
    cd = torch.from_numpy(codes).to(U.DEV)
    used = torch.full((128,), 7, dtype=torch.uint8, device=U.DEV)
    cnt = torch.zeros(1, dtype=torch.int32, device=U.DEV)
    packed = torch.empty(n, 14 * (k // 16), dtype=torch.uint8, device=U.DEV)
    st = U.status_tensor()
    U.tq().tq_pack7(cd, used, cnt, packed, st)
    torch.cuda.synchronize()
    return (used.cpu().numpy(), int(cnt.item()), packed.cpu().numpy(),
            int(st.item()), packed)


@pytest.mark.parametrize("n,k,distinct", [(300, 2064, 45), (64, 512, 128),
                                          (5, 16, 1), (1000, 1024, 18)])
def test_pack7_bit_exact(n, k, distinct):
    codes = _codes(n, k, distinct, n + k)
    used, cnt, packed, st, _ = _pack_gpu(codes)
    r_used, r_cnt, r_packed = oref.pack7(codes)
    assert st == 0
    assert cnt == r_cnt == distinct
    assert np.array_equal(used, r_used)
    assert np.array_equal(packed, r_packed)


def test_pack7_too_many_words():
    codes = _codes(64, 256, 129, 1)
    _, cnt, _, st, _ = _pack_gpu(codes)
    assert cnt == 129 and st == U.tq().TQ_ERR_RANGE


@pytest.mark.parametrize("n,k,rps", [(300, 2064, 0), (130, 5376, 1),
                                     (257, 1040, 128)])
def test_linear_and_unpack_b7(n, k, rps):
    codes = _codes(n, k, 45, 3 * n + k)
    lut = oref.build_lut(I.ALPHA, I.ladder_pow3().numpy())
    used, _, packed_h, _, packed = _pack_gpu(codes)
    lut7 = U.tq().tq_build_lut7(lut, used)
    assert np.array_equal(lut7, lut[used])
    rho = I.rho_uniform(I.rho_count(n, rps), 4) if rps else None
    rho_bits = I.bits(rho) if rps else None
    L7 = torch.from_numpy(lut7).to(U.DEV)
    rd = rho.view(torch.int16).to(U.DEV) if rps else None
    w = U.tq().weights_b7(packed, L7, n, k, rd, rps)
    absmax = U.absmax_rows_b(codes, lut, rho_bits, rps)
    for batch in (1, 4, 9, 64):
        x = I.x_normal(batch, k, batch + 1)
        xb = U.x_bits(x)
        y, _ = U.linear(w, x)
        ref = oref.linear_B7(packed_h, used, n, k, lut, xb, rho_bits, rps)
        U.check_tolerance(y, ref, xb, absmax, f"B7 {n}x{k} b={batch}")
    out = torch.empty(n, k, dtype=torch.int16, device=U.DEV)
    U.tq().tq_unpack(w, out)
    torch.cuda.synchronize()
    ref = oref.unpack_B7(packed_h, used, n, k, lut, rho_bits, rps)
    assert np.array_equal(out.cpu().numpy().view(np.uint16), ref)


@pytest.fixture
def force_path():
    def set_path(p):
        U.tq().tq_testing_force_linear_path(p)
    yield set_path
    U.tq().tq_testing_force_linear_path(0)


# K a multiple of 128: batches from 3 take the tensor-core kernel (path 0) (one
# 112-byte run of 128 indices per row and k block); the balanced-ternary
# ladder puts every used word on one integer grid (single bf16 operand),
# the free ladder does not (hi + lo pair); path 3 forces the pair on the grid,
# path 2 the tensor-core kernel at batch 2
LADDER_FREE = np.array([1.0, 0.33, 0.115, 0.037, 0.012], np.float32)


@pytest.mark.parametrize("n,k,rps,ladder,distinct,path", [
    (300, 4096, 0, "pow3", 45, 0), (129, 1024, 1, "free", 128, 0),
    (1000, 2048, 128, "pow3", 100, 0), (257, 128, 0, "free", 3, 0),
    (300, 4096, 0, "pow3", 45, 3), (384, 5376, 1, "pow3", 1, 0),
    (200, 1024, 0, "free", 20, 2)])
def test_linear_b7_tensor_core(force_path, n, k, rps, ladder, distinct, path):
    codes = _codes(n, k, distinct, 7 * n + k)
    lad = I.ladder_pow3().numpy() if ladder == "pow3" else LADDER_FREE
    lut = oref.build_lut(I.ALPHA, lad)
    used, _, packed_h, _, packed = _pack_gpu(codes)
    lut7 = U.tq().tq_build_lut7(lut, used)
    rho = I.rho_uniform(I.rho_count(n, rps), 5) if rps else None
    rho_bits = I.bits(rho) if rps else None
    L7 = torch.from_numpy(lut7).to(U.DEV)
    rd = rho.view(torch.int16).to(U.DEV) if rps else None
    w = U.tq().weights_b7(packed, L7, n, k, rd, rps)
    absmax = U.absmax_rows_b(codes, lut, rho_bits, rps)
    force_path(path)
    for batch in (2, 5, 16, 33, 64):
        x = I.x_normal(batch, k, batch + 11)
        xb = U.x_bits(x)
        y, _ = U.linear(w, x)
        ref = oref.linear_B7(packed_h, used, n, k, lut, xb, rho_bits, rps)
        U.check_tolerance(y, ref, xb, absmax,
                          f"B7 TC {n}x{k} {ladder} path {path} b={batch}")


def test_linear_b7_tensor_core_matches_one_warp_per_row(force_path):
    # the same 7-bit layer through the tensor-core kernel and through the
    # one-warp-per-row kernel (force path 1), both within the oracle's
    # tolerance
    n, k = 256, 2048
    codes = _codes(n, k, 60, 99)
    lut = oref.build_lut(I.ALPHA, I.ladder_pow3().numpy())
    used, _, packed_h, _, packed = _pack_gpu(codes)
    lut7 = U.tq().tq_build_lut7(lut, used)
    w = U.tq().weights_b7(packed, torch.from_numpy(lut7).to(U.DEV), n, k,
                          None, 0)
    absmax = U.absmax_rows_b(codes, lut)
    x = I.x_normal(16, k, 5)
    xb = U.x_bits(x)
    ref = oref.linear_B7(packed_h, used, n, k, lut, xb, None, 0)
    y_tc, _ = U.linear(w, x)
    force_path(1)
    y_simple, _ = U.linear(w, x)
    U.check_tolerance(y_tc, ref, xb, absmax, "B7 tensor core")
    U.check_tolerance(y_simple, ref, xb, absmax, "B7 one warp per row")

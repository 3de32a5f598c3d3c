"""GPU parity of the 7-bit truncated alphabet (alphaneural.io page, section
8.1): tq_pack7 bit-exact against the oracle (used-code table, count, packed
indices), the more-than-128-words status, tq_linear on a 7-bit layer against
the fp64 oracle (same tolerance as test_gpu_linear) and bit-exact unpack."""
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

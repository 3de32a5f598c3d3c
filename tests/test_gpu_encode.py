"""GPU parity of the Format B encoder (tq_encode_b) with the oracle: codes,
rho and alpha bit-exact ("A Discrete Weight Language for Large Language
Models", sections 3.1 and 3.3), on layers of the Gemma-shaped workload (up
21504 x 5376 with one scale per row, q 8192 x 5376 with one per 128-row head),
ragged shapes, the page's fitted ladder and the 3^-(k-1) ladder, zero biases
0.5 and 0.65, all-zero rows and non-finite weights; then the codes it makes go
through tq_linear within the matmul tolerance."""
import numpy as np
import pytest
import torch

from oracle import oref
from packed_weight_matmul_b200 import inputs as I
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

FITTED = np.array([1.0, 0.33, 0.115, 0.037, 0.012], np.float32)


def encode(W, ladder, zeta, rps):
    n, k = W.shape
    Wd = W.to(U.DEV).contiguous()
    codes = torch.empty(n, k, dtype=torch.uint8, device=U.DEV)
    rho = (torch.empty((n + rps - 1) // rps, dtype=torch.int16, device=U.DEV)
           if rps else None)
    alpha = torch.empty(1, dtype=torch.float32, device=U.DEV)
    st = U.status_tensor()
    U.tq().tq_encode_b(Wd, ladder, zeta, rps, codes, rho, alpha, st)
    torch.cuda.synchronize()
    return (codes.cpu().numpy(),
            None if rho is None else rho.cpu().numpy().view(np.uint16),
            float(alpha.item()), int(st.item()))


def check(W, ladder, zeta, rps):
    codes, rho, alpha, st = encode(W, ladder, zeta, rps)
    rc, rr, ra = oref.encode_B(I.bits(W), ladder, zeta, rps)
    assert st == 0
    assert alpha == ra
    assert np.array_equal(codes, rc)
    if rps:
        assert np.array_equal(rho, rr)
    return codes, rho, alpha


@pytest.mark.parametrize("ladder", [FITTED, None], ids=["fitted", "pow3"])
@pytest.mark.parametrize("zeta", [0.5, 0.65])
@pytest.mark.parametrize("rps", [0, 1, 128, 3])
@pytest.mark.parametrize("n,k", [(1, 16), (37, 80), (300, 1024)])
def test_encode_ragged_bit_exact(ladder, zeta, rps, n, k):
    lad = I.ladder_pow3().numpy() if ladder is None else ladder
    W = I.student_t_bf16(n, k, seed=n + k + rps)
    check(W, lad, zeta, rps)


@pytest.mark.parametrize("n,k,rps", [(21504, 5376, 1), (8192, 5376, 128)],
                         ids=["up_per_row", "q_per_head"])
def test_encode_gemma_layers_bit_exact(n, k, rps):
    W = I.student_t_bf16(n, k, seed=7 + rps)
    check(W, FITTED, 0.5, rps)


def test_encode_zero_rows_and_matrix():
    W = I.student_t_bf16(64, 128, seed=3).float()
    W[5] = 0.0
    W[60:64] = 0.0
    W = W.to(torch.bfloat16)
    codes, rho, _ = check(W, FITTED, 0.5, 1)
    assert np.all(codes[5] == 121) and rho[5] == 0
    codes, rho, _ = check(W, FITTED, 0.5, 4)
    assert np.all(codes[60:] == 121) and rho[15] == 0
    Z = torch.zeros(8, 32, dtype=torch.bfloat16)
    codes, _, alpha, st = encode(Z, FITTED, 0.5, 0)
    assert st == 0 and alpha == 0.0 and np.all(codes == 121)


def test_encode_reports_nonfinite():
    W = I.student_t_bf16(16, 64, seed=4)
    W[7, 9] = float("inf")
    _, _, _, st = encode(W, FITTED, 0.5, 1)
    assert st == oref.ERR_NONFINITE


def test_encoded_codes_through_linear():
    n, k = 1024, 2048
    W = I.student_t_bf16(n, k, seed=9)
    codes, rho, alpha = check(W, FITTED, 0.5, 1)
    lut = oref.build_lut(alpha, FITTED)
    w = U.weights_b_dev(codes, lut, rho, 1)
    absmax = U.absmax_rows_b(codes, lut, rho, 1)
    for batch in (1, 4, 16, 64):
        x = I.x_normal(batch, k, 70 + batch)
        xb = U.x_bits(x)
        y, _ = U.linear(w, x)
        ref = oref.linear_B(codes, lut, xb, rho, 1)
        U.check_tolerance(y, ref, xb, absmax, f"encoded b={batch}")

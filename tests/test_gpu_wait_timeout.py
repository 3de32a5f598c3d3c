"""GPU: a bounded in-kernel wait that runs out ends the tensor-core kernel
cleanly. Through the test hook of include/tq_testing.h the decoder warps
withhold their first "operand stage ready" signal, so the MMA issuer's wait
(shortened to 20 ms) runs out with no fault: the kernel must write NaN to
every output, free its tensor memory and return, and the next ordinary call
on the same context must give correct results. Covered with and without a
split of K over a cluster (then the CTAs also leave through the cluster exit
protocol)."""
import numpy as np
import pytest
import torch

from oracle import oref
from packed_weight_matmul_b200 import inputs as I
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


@pytest.fixture
def hook():
    tq = U.tq()
    yield tq
    tq.tq_testing_linear_wait_fault(False, 0)


@pytest.mark.parametrize("n,k", [(200, 128),    # one block: no split of K
                                 (128, 2048)])  # one tile: K split over a cluster
@pytest.mark.parametrize("fmt", ["A", "B"])
def test_wait_timeout_gives_nan_then_context_recovers(hook, fmt, n, k):
    batch = 16  # tensor-core path for both formats
    if fmt == "B":
        codes = I.codes_uniform(n, k, 11)
        lut = oref.build_lut(I.ALPHA, I.ladder_pow3().numpy())
        w = U.weights_b_dev(codes, lut)
        absmax = U.absmax_rows_b(codes.numpy(), lut)
        ref = lambda xb: oref.linear_B(codes.numpy(), lut, xb)
    else:
        W = I.student_t_bf16(n, k, seed=12)
        codes, scales = oref.quantize_pack_A(I.bits(W), 64, 1)
        w = U.weights_a_dev(codes, scales, n, k)
        absmax = U.absmax_rows_a(codes, scales, n, k, 64, 1)
        ref = lambda xb: oref.linear_A(codes, scales, n, k, xb)
    x = I.x_normal(batch, k, 13)
    hook.tq_testing_linear_wait_fault(True, 20_000_000)
    y, _ = U.linear(w, x, y_fill=0.0)
    assert np.all(np.isnan(y)), "a timed-out kernel must leave NaN outputs"
    hook.tq_testing_linear_wait_fault(False, 0)
    y, _ = U.linear(w, x)
    xb = U.x_bits(x)
    U.check_tolerance(y, ref(xb), xb, absmax, f"{fmt} after a time-out")

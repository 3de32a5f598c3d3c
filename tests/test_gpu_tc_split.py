"""GPU parity of the tensor-core kernel's persistent clusters with a split of
K (alphaneural.io page, section 4.2; precisit.com page, "Three values and a
shared scale"). Through tq_testing_tc_split a small shape is planned with
clusters of ks CTAs and fewer clusters than row tiles, so that every
cluster walks several tiles and adds each tile's ks partial tiles through
distributed shared memory while the next tile streams in. Checked against
the fp64 oracle (same tolerance as test_gpu_linear) on every output, for
both formats, ragged rows and uneven K slices; two calls give bit-identical
outputs (the partials are added in rank order); and a bounded wait that
runs out with several tiles per cluster still ends with NaN outputs and a
usable context."""
import numpy as np
import pytest
import torch

from oracle import oref
from packed_weight_matmul_b200 import inputs as I
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

LADDER_FREE = np.array([1.0, 0.33, 0.115, 0.037, 0.012], np.float32)


@pytest.fixture
def split():
    def set_split(ks, clusters):
        U.tq().tq_testing_tc_split(ks, clusters)
    U.tq().tq_testing_force_linear_path(2)
    yield set_split
    U.tq().tq_testing_tc_split(0, 0)
    U.tq().tq_testing_force_linear_path(0)
    U.tq().tq_testing_linear_wait_fault(False, 0)


def _layer_b(n, k, ladder, rps, seed):
    codes = I.codes_uniform(n, k, seed)
    lad = I.ladder_pow3().numpy() if ladder == "pow3" else LADDER_FREE
    lut = oref.build_lut(I.ALPHA, lad)
    rho = I.rho_uniform(I.rho_count(n, rps), seed + 1) if rps else None
    rho_bits = I.bits(rho) if rps else None
    w = U.weights_b_dev(codes, lut, rho, rps)
    absmax = U.absmax_rows_b(codes.numpy(), lut, rho_bits, rps)
    ref = lambda xb: oref.linear_B(codes.numpy(), lut, xb, rho_bits, rps)
    return w, absmax, ref


def _layer_a(n, k, planes, seed):
    W = I.student_t_bf16(n, k, seed=seed)
    codes, scales = oref.quantize_pack_A(I.bits(W), 64, planes)
    w = U.weights_a_dev(codes, scales, n, k, 64, planes)
    absmax = U.absmax_rows_a(codes, scales, n, k, 64, planes)
    ref = lambda xb: oref.linear_A(codes, scales, n, k, xb, 64, planes)
    return w, absmax, ref


@pytest.mark.parametrize("n,k,ladder,rps,ks,clusters", [
    (1000, 2048, "pow3", 0, 2, 3),    # 8 tiles over 3 clusters
    (1000, 2048, "free", 1, 3, 2),    # slices of 5, 5 and 6 blocks
    (300, 4096, "pow3", 128, 8, 1),   # one cluster of 8 walks 3 tiles
    (1000, 2048, "free", 0, 1, 3),    # no split, 3 persistent CTAs
    (700, 1040, "pow3", 1, 4, 2)])    # ragged last block and tile
def test_split_format_b(split, n, k, ladder, rps, ks, clusters):
    w, absmax, ref = _layer_b(n, k, ladder, rps, n + k + ks)
    split(ks, clusters)
    for batch in (5, 16, 64):
        x = I.x_normal(batch, k, batch + ks)
        xb = U.x_bits(x)
        y, _ = U.linear(w, x)
        U.check_tolerance(y, ref(xb), xb, absmax,
                          f"B {n}x{k} ks={ks} clusters={clusters} b={batch}")
        y2, _ = U.linear(w, x)
        assert np.array_equal(y.view(np.uint32), y2.view(np.uint32)), \
            "the split's sums must not depend on timing"


@pytest.mark.parametrize("planes,ks,clusters", [(1, 2, 2), (2, 4, 1)])
def test_split_format_a(split, planes, ks, clusters):
    n, k = 520, 2048
    w, absmax, ref = _layer_a(n, k, planes, 7 + planes)
    split(ks, clusters)
    for batch in (2, 16, 64):
        x = I.x_normal(batch, k, batch)
        xb = U.x_bits(x)
        y, _ = U.linear(w, x)
        U.check_tolerance(y, ref(xb), xb, absmax,
                          f"A{planes} ks={ks} clusters={clusters} b={batch}")


def test_split_wait_timeout_gives_nan_then_recovers(split):
    n, k = 300, 2048  # 3 tiles walked by one cluster of 2
    w, absmax, ref = _layer_b(n, k, "pow3", 0, 21)
    split(2, 1)
    x = I.x_normal(16, k, 13)
    U.tq().tq_testing_linear_wait_fault(True, 20_000_000)
    y, _ = U.linear(w, x, y_fill=0.0)
    assert np.all(np.isnan(y)), "a timed-out kernel must leave NaN outputs"
    U.tq().tq_testing_linear_wait_fault(False, 0)
    y, _ = U.linear(w, x)
    xb = U.x_bits(x)
    U.check_tolerance(y, ref(xb), xb, absmax, "split after a time-out")


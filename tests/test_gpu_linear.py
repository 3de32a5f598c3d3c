"""GPU parity of tq_linear against the fp64 oracle over the same decoded
weights: |y - y_oracle| <= 2e-3 * ||x_b||_2 * max_k |w[n][k]| for every output
(a row with max |w| = 0 must give exactly 0), at sizes that span several tiles
and ragged tails, on both sides of every batch dispatch threshold, with
row-offset views and padded strides; at the full workload sizes on sampled
rows."""
import numpy as np
import pytest
import torch

from oracle import oref
from packed_weight_matmul_b200 import inputs as I
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

BATCHES = [1, 2, 3, 4, 5, 8, 9, 15, 16, 17, 32, 33, 64, 65]


def _pkg_a(n, k, G=64, planes=1, seed=0):
    W = I.student_t_bf16(n, k, seed=seed)
    codes, scales = oref.quantize_pack_A(I.bits(W), G, planes)
    return codes, scales


# ---- Format A -----------------------------------------------------------------

def test_linear_a_small_workload_all_batches():
    cfg = I.fmt_a_small()
    codes, scales = oref.quantize_pack_A(I.bits(cfg["W"]), 64, 1)
    w = U.weights_a_dev(codes, scales, 512, 1024)
    absmax = U.absmax_rows_a(codes, scales, 512, 1024, 64, 1)
    assert np.sum(absmax == 0) == 0  # zero groups, but no zero rows
    for batch in BATCHES:
        x = cfg["x"] if batch == 1 else I.x_normal(batch, 1024, 100 + batch)
        xb = U.x_bits(x)
        y, _ = U.linear(w, x)
        ref = oref.linear_A(codes, scales, 512, 1024, xb)
        U.check_tolerance(y, ref, xb, absmax, f"A small batch={batch}")


@pytest.mark.parametrize("G,planes", [(64, 1), (64, 2), (128, 1), (128, 2)])
@pytest.mark.parametrize("n,k", [(1, 128), (7, 256), (130, 1280),
                                 (257, 4224)])
def test_linear_a_ragged(G, planes, n, k):
    codes, scales = _pkg_a(n, k, G, planes, seed=n + k)
    w = U.weights_a_dev(codes, scales, n, k, G, planes)
    absmax = U.absmax_rows_a(codes, scales, n, k, G, planes)
    for batch in (1, 4, 9, 16, 40):
        x = I.x_normal(batch, k, batch)
        xb = U.x_bits(x)
        y, _ = U.linear(w, x)
        ref = oref.linear_A(codes, scales, n, k, xb, G, planes)
        U.check_tolerance(y, ref, xb, absmax, f"A G={G} p={planes} "
                          f"{n}x{k} b={batch}")


def test_linear_a_zero_rows_are_exact_zero():
    n, k = 40, 512
    W = I.student_t_bf16(n, k, seed=2)
    W[[3, 17, 39]] = 0
    codes, scales = oref.quantize_pack_A(I.bits(W), 64, 2)
    w = U.weights_a_dev(codes, scales, n, k, 64, 2)
    for batch in (1, 8, 16, 64):
        x = I.x_normal(batch, k, 3)
        y, _ = U.linear(w, x)
        assert np.all(y[:, [3, 17, 39]] == 0.0)


def test_linear_a_views_and_strides():
    N, k, G = 96, 1024, 64  # 208-byte rows: every row offset is aligned
    codes, scales = _pkg_a(N, k, G, 2, seed=4)
    cd, sd = U.to_dev_u8(codes), U.to_dev_u16(scales)
    gpr, nb = k // G, 13
    r0, n = 10, 50
    w = U.tq().weights_a(cd[r0 * gpr * nb:], sd[r0 * gpr:], n, k, G, 2,
                         codes_plane_stride=N * gpr * nb,
                         scales_plane_stride=N * gpr)
    rows = np.arange(r0, r0 + n)
    absmax = U.absmax_rows_a(codes, scales, N, k, G, 2, rows=rows)
    for batch in (1, 5, 16, 33):
        x = I.x_normal(batch, k, 7)
        xb = U.x_bits(x)
        y, yfull = U.linear(w, x, ldx=k + 24, ldy=n + 12, y_fill=-7.0)
        assert np.all(yfull[:, n:] == -7.0)  # padding untouched
        ref = oref.linear_A(codes, scales, N, k, xb, G, 2, rows=rows)
        U.check_tolerance(y, ref, xb, absmax, f"A view b={batch}")
    # a view whose row offset breaks the 16-byte rule is rejected
    codes1, scales1 = _pkg_a(8, 320, 64, 1, seed=1)  # 65-byte rows
    cd1, sd1 = U.to_dev_u8(codes1), U.to_dev_u16(scales1)
    bad = U.tq().weights_a(cd1[65:], sd1[5:], 7, 320)
    x = torch.zeros(1, 320, dtype=torch.bfloat16, device=U.DEV)
    y = torch.zeros(1, 8, dtype=torch.float32, device=U.DEV)
    st = U.tq().tq_linear(bad, x, y, check=False)
    assert st == U.tq().TQ_ERR_ALIGNMENT


@pytest.fixture(scope="module")
def large_pkg():
    W = I.fmt_a_large()["W"]
    codes, scales = oref.quantize_pack_A(I.bits(W), 64, 2)
    return codes, scales


@pytest.mark.parametrize("planes", [1, 2])
def test_linear_a_large_workload_sampled(large_pkg, planes):
    codes2, scales2 = large_pkg
    codes, scales = codes2[:planes], scales2[:planes]
    n, k = 28672, 8192
    w = U.weights_a_dev(codes, scales, n, k, 64, planes)
    rng = np.random.default_rng(planes)
    rows = np.sort(rng.choice(n, 192, replace=False))
    rows[-1] = n - 1
    absmax = U.absmax_rows_a(codes, scales, n, k, 64, planes, rows=rows)
    for batch in (1, 8, 32, 64):
        x = I.x_normal(batch, k, 1000 + batch)
        xb = U.x_bits(x)
        y, _ = U.linear(w, x)
        ref = oref.linear_A(codes, scales, n, k, xb, 64, planes, rows=rows)
        U.check_tolerance(y[:, rows], ref, xb, absmax,
                          f"A large p={planes} b={batch}")


# ---- Format B -------------------------------------------------------------------

@pytest.fixture(scope="module")
def lut():
    return oref.build_lut(I.ALPHA, I.ladder_pow3().numpy())


def test_linear_b_4096_workload(lut):
    cfg = I.fmt_b_4096()
    codes = cfg["codes"]
    w = U.weights_b_dev(codes, lut)
    absmax = U.absmax_rows_b(codes.numpy(), lut)
    for batch in BATCHES:
        x = I.x_normal(batch, 4096, 10 + batch)
        xb = U.x_bits(x)
        y, _ = U.linear(w, x)
        rows = None if batch <= 4 else np.arange(0, 4096, 17)
        ref = oref.linear_B(codes.numpy(), lut, xb, rows=rows)
        yy = y if rows is None else y[:, rows]
        am = absmax if rows is None else absmax[rows]
        U.check_tolerance(yy, ref, xb, am, f"B 4096 b={batch}")


@pytest.mark.parametrize("rps", [0, 1, 2, 128])
@pytest.mark.parametrize("n,k", [(1, 16), (5, 48), (33, 528), (130, 5376),
                                 (300, 2064)])
def test_linear_b_ragged(lut, rps, n, k):
    codes = I.codes_uniform(n, k, n * 31 + k)
    rho = I.rho_uniform(I.rho_count(n, rps), 5) if rps else None
    rho_bits = I.bits(rho) if rps else None
    w = U.weights_b_dev(codes, lut, rho, rps)
    absmax = U.absmax_rows_b(codes.numpy(), lut, rho_bits, rps)
    for batch in (1, 3, 8, 16, 24, 64):
        x = I.x_normal(batch, k, batch + 50)
        xb = U.x_bits(x)
        y, _ = U.linear(w, x)
        ref = oref.linear_B(codes.numpy(), lut, xb, rho_bits, rps)
        U.check_tolerance(y, ref, xb, absmax, f"B {n}x{k} rps={rps} "
                          f"b={batch}")


def test_linear_b_invalid_code_poisons_row(lut):
    codes = I.codes_uniform(64, 256, 1)
    codes[9, 100] = 250
    w = U.weights_b_dev(codes, lut)
    for batch in (1, 16):
        y, _ = U.linear(w, I.x_normal(batch, 256, 2))
        assert np.all(np.isnan(y[:, 9]))
        assert np.all(np.isfinite(np.delete(y, 9, axis=1)))


def test_linear_b_views_and_strides(lut):
    N, k, rps = 512, 1024, 128
    codes = I.codes_uniform(N, k, 8)
    rho = I.rho_uniform(I.rho_count(N, rps), 8)
    r0, n = 256, 200
    cd = codes.to(U.DEV)
    L = torch.from_numpy(lut).to(U.DEV)
    rd = rho.view(torch.int16).to(U.DEV)
    w = U.tq().weights_b(cd[r0:], L, rd[r0 // rps:], rps, n=n, k=k)
    rows = np.arange(r0, r0 + n)
    rho_bits = I.bits(rho)
    absmax = U.absmax_rows_b(codes.numpy(), lut, rho_bits, rps, rows=rows)
    for batch in (1, 4, 16, 33):
        x = I.x_normal(batch, k, 9)
        xb = U.x_bits(x)
        y, yfull = U.linear(w, x, ldx=k + 8, ldy=n + 4, y_fill=3.0)
        assert np.all(yfull[:, n:] == 3.0)
        ref = oref.linear_B(codes.numpy(), lut, xb, rho_bits, rps, rows=rows)
        U.check_tolerance(y, ref, xb, absmax, f"B view b={batch}")


@pytest.mark.parametrize("layer", I.FMT_B_GEMMA_LAYERS, ids=lambda l: l.name)
def test_linear_b_gemma_layers_sampled(lut, layer):
    cfg = I.fmt_b_gemma_layer(layer)
    codes, rho, rps = cfg["codes"], cfg["rho"], cfg["rps"]
    rho_bits = I.bits(rho)
    w = U.weights_b_dev(codes, lut, rho, rps)
    rng = np.random.default_rng(len(layer.name))
    rows = np.sort(rng.choice(layer.n, 160, replace=False))
    rows[0], rows[-1] = 0, layer.n - 1
    absmax = U.absmax_rows_b(codes.numpy(), lut, rho_bits, rps, rows=rows)
    for batch in (1, 4, 16):
        x = I.x_normal(batch, layer.k, batch)
        xb = U.x_bits(x)
        y, _ = U.linear(w, x)
        ref = oref.linear_B(codes.numpy(), lut, xb, rho_bits, rps, rows=rows)
        U.check_tolerance(y[:, rows], ref, xb, absmax,
                          f"B {layer.name} b={batch}")


def test_linear_deterministic(lut):
    codes = I.codes_uniform(4096, 4096, 1)
    w = U.weights_b_dev(codes, lut)
    ca, sa = _pkg_a(2048, 2048, 64, 2, seed=3)
    wa = U.weights_a_dev(ca, sa, 2048, 2048, 64, 2)
    for ww, k in ((w, 4096), (wa, 2048)):
        for batch in (1, 8, 16, 64):
            x = I.x_normal(batch, k, 4)
            y1, _ = U.linear(ww, x)
            y2, _ = U.linear(ww, x)
            assert np.array_equal(y1, y2)

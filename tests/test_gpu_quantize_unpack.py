"""GPU parity: tq_quantize_pack and tq_unpack must be bit-exact against the
oracle (codes, scales, unpacked bf16), report data errors through the status
word, and be deterministic."""
import numpy as np
import pytest
import torch

from oracle import oref
from packed_weight_matmul_b200 import inputs as I
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


def test_quantize_small_workload_bit_exact():
    cfg = I.fmt_a_small()
    codes, scales, st = U.quantize(cfg["W"], 64, 1)
    assert st == 0
    rc, rs = oref.quantize_pack_A(I.bits(cfg["W"]), 64, 1)
    assert np.array_equal(codes, rc)
    assert np.array_equal(scales, rs)
    for r, g in cfg["zero_groups"]:
        assert scales[0, r, g] == 0 and np.all(codes[0, r, g] == 121)


@pytest.mark.parametrize("G", [64, 128])
@pytest.mark.parametrize("planes", [1, 2])
@pytest.mark.parametrize("n,k", [(1, 128), (3, 256), (17, 384), (129, 1024),
                                 (257, 640)])
def test_quantize_ragged_bit_exact(G, planes, n, k):
    if k % G:
        pytest.skip("k not a multiple of G")
    W = I.student_t_bf16(n, k, seed=n * 7 + k)
    codes, scales, st = U.quantize(W, G, planes)
    assert st == 0
    rc, rs = oref.quantize_pack_A(I.bits(W), G, planes)
    assert np.array_equal(codes, rc)
    assert np.array_equal(scales, rs)


def test_quantize_edge_values_bit_exact():
    # ties at s/2, subnormal bf16, an underflowing group, huge finite values
    rows = []
    vals = [0.5] * 8 + [-0.5] * 8 + [7.0] * 6 + [1.5, -1.5, 0.50390625,
                                                  -0.50390625, 0.49609375]
    vals += [0.0] * (64 - len(vals) - 1)
    vals.append(64.0 - sum(abs(v) for v in vals))
    rows.append(vals)
    rows.append([2.0 ** -40 * (-1) ** j for j in range(64)])
    rows.append([2.0 ** -130 * (j + 1) for j in range(64)])  # subnormals
    rows.append([3.0e38 * (-1) ** j for j in range(64)])  # huge: RANGE
    rows.append([1.0e4 * (j % 7 - 3) for j in range(64)])
    W = torch.tensor(rows, dtype=torch.float32).to(torch.bfloat16)
    ok_rows = W[[0, 1, 2, 4]].contiguous()
    for planes in (1, 2):
        codes, scales, st = U.quantize(ok_rows, 64, planes)
        rc, rs = oref.quantize_pack_A(I.bits(ok_rows), 64, planes)
        assert st == 0
        assert np.array_equal(codes, rc) and np.array_equal(scales, rs)
    _, _, st = U.quantize(W[3:4].contiguous(), 64, 1)
    assert st == oref.ERR_RANGE


def test_quantize_nonfinite_reported():
    W = I.student_t_bf16(8, 256, seed=5)
    W[5, 77] = float("nan")
    _, _, st = U.quantize(W, 64, 1)
    assert st == oref.ERR_NONFINITE
    W = I.student_t_bf16(8, 256, seed=5)
    W[2, 3] = float("inf")
    _, _, st = U.quantize(W, 64, 2)
    assert st == oref.ERR_NONFINITE


@pytest.fixture(scope="module")
def large():
    return I.fmt_a_large()


def test_quantize_large_workload_both_planes_bit_exact(large):
    W = large["W"]
    codes, scales, st = U.quantize(W, 64, 2)
    assert st == 0
    rc, rs = oref.quantize_pack_A(I.bits(W), 64, 2)
    assert np.array_equal(scales, rs)
    assert np.array_equal(codes, rc)
    # deterministic: a second run is bit-identical
    codes2, scales2, _ = U.quantize(W, 64, 2)
    assert np.array_equal(codes, codes2) and np.array_equal(scales, scales2)


def _unpack(w, n, k):
    out = torch.empty(n, k, dtype=torch.int16, device=U.DEV)
    st = U.status_tensor()
    U.tq().tq_unpack(w, out, st)
    torch.cuda.synchronize()
    return out.cpu().numpy().view(np.uint16), int(st.item())


@pytest.mark.parametrize("G,planes,n,k", [(64, 1, 512, 1024), (64, 2, 3, 64),
                                          (64, 2, 300, 2048),
                                          (128, 1, 5, 384), (128, 2, 33, 1280)])
def test_unpack_a_bit_exact(G, planes, n, k):
    W = I.student_t_bf16(n, k, seed=G + planes + n)
    codes, scales = oref.quantize_pack_A(I.bits(W), G, planes)
    w = U.weights_a_dev(codes, scales, n, k, G, planes)
    got, st = _unpack(w, n, k)
    assert st == 0
    assert np.array_equal(got, oref.unpack_A(codes, scales, n, k, G, planes))


def test_unpack_a_large_two_planes_bit_exact(large):
    W = large["W"][:4096]
    n, k = W.shape
    codes, scales = oref.quantize_pack_A(I.bits(W), 64, 2)
    got, st = _unpack(U.weights_a_dev(codes, scales, n, k, 64, 2), n, k)
    assert st == 0
    assert np.array_equal(got, oref.unpack_A(codes, scales, n, k, 64, 2))


def test_unpack_a_rejects_bad_bytes():
    n, k = 4, 256
    codes, scales = oref.quantize_pack_A(I.bits(I.student_t_bf16(n, k, 1)))
    bad = codes.copy()
    bad[0, 2, 1, 5] = 247  # >= 243
    _, st = _unpack(U.weights_a_dev(bad, scales, n, k), n, k)
    assert st == oref.ERR_BAD_CODE
    bad = codes.copy()
    b = int(bad[0, 1, 3, 12])
    bad[0, 1, 3, 12] = b - 81  # padding digit 1 -> 0
    _, st = _unpack(U.weights_a_dev(bad, scales, n, k), n, k)
    assert st == oref.ERR_BAD_CODE


@pytest.mark.parametrize("rps", [0, 1, 128, 3])
def test_unpack_b_bit_exact(rps):
    g = torch.Generator().manual_seed(rps)
    n, k = 384, 528
    codes = torch.randint(0, 243, (n, k), generator=g, dtype=torch.uint8)
    lut = oref.build_lut(0.02, I.ladder_pow3().numpy())
    rho = I.rho_uniform(I.rho_count(n, rps), rps + 9) if rps else None
    w = U.weights_b_dev(codes, lut, rho, rps)
    got, st = _unpack(w, n, k)
    assert st == 0
    rho_bits = I.bits(rho) if rps else None
    ref = oref.unpack_B(codes.numpy(), lut, rho_bits, rps)
    assert np.array_equal(got, ref)


def test_unpack_b_rejects_bad_codes():
    codes = I.codes_uniform(64, 64, 3)
    codes[10, 20] = 255
    lut = oref.build_lut(0.02, I.ladder_pow3().numpy())
    _, st = _unpack(U.weights_b_dev(codes, lut), 64, 64)
    assert st == oref.ERR_BAD_CODE


# ---- tq_unpack at the workloads' full sizes ---------------------------------
# The decoded bf16 weights must be bit-exact on every workload: a lossless
# round trip ("Does your weight format deserve a kernel?", "Five trits in a
# byte"). Inputs come from the oracle and the seeded generators only.

def test_unpack_a_large_all_rows_two_planes_bit_exact(large):
    W = large["W"]
    n, k = W.shape
    codes, scales = oref.quantize_pack_A(I.bits(W), 64, 2)
    got, st = _unpack(U.weights_a_dev(codes, scales, n, k, 64, 2), n, k)
    assert st == 0
    assert np.array_equal(got, oref.unpack_A(codes, scales, n, k, 64, 2))
    # plane 1 alone (the plane stride leaves plane 2 unread)
    got1, st1 = _unpack(U.weights_a_dev(codes[:1], scales[:1], n, k, 64, 1),
                        n, k)
    assert st1 == 0
    assert np.array_equal(got1, oref.unpack_A(codes[:1], scales[:1], n, k, 64,
                                              1))


def test_unpack_b_4096_bit_exact():
    cfg = I.fmt_b_4096()
    codes = cfg["codes"]
    lut = oref.build_lut(cfg["alpha"], cfg["ladder"].numpy())
    got, st = _unpack(U.weights_b_dev(codes, lut), 4096, 4096)
    assert st == 0
    assert np.array_equal(got, oref.unpack_B(codes.numpy(), lut))


@pytest.mark.parametrize("layer", I.FMT_B_GEMMA_LAYERS,
                         ids=lambda l: l.name)
def test_unpack_b_gemma_layers_with_rho_bit_exact(layer):
    cfg = I.fmt_b_gemma_layer(layer)
    codes, rho, rps = cfg["codes"], cfg["rho"], cfg["rps"]
    lut = oref.build_lut(cfg["alpha"], cfg["ladder"].numpy())
    got, st = _unpack(U.weights_b_dev(codes, lut, rho, rps), layer.n, layer.k)
    assert st == 0
    ref = oref.unpack_B(codes.numpy(), lut, I.bits(rho), rps)
    assert np.array_equal(got, ref)


def _decode_step_shapes():
    seen, out = set(), []
    for seed, layer in I.decode_step_layers(1):
        if (layer.n, layer.k) not in seen:
            seen.add((layer.n, layer.k))
            out.append((seed, layer))
    return out


@pytest.mark.parametrize("seed,layer", _decode_step_shapes(),
                         ids=lambda v: getattr(v, "name", str(v)))
def test_unpack_b_decode_step_layer_bit_exact(seed, layer):
    codes = I.codes_uniform(layer.n, layer.k, seed)
    lut = oref.build_lut(I.ALPHA, I.ladder_pow3().numpy())
    got, st = _unpack(U.weights_b_dev(codes, lut), layer.n, layer.k)
    assert st == 0
    assert np.array_equal(got, oref.unpack_B(codes.numpy(), lut))

"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these tests compares the oracle with itself: each checks it against a
value printed on a page (tests/golden), a closed form, an invariant, a library
routine (numpy / torch / math.fsum) that implements the same IEEE rounding, or
a brute-force computation on tiny exact inputs.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

from packed_weight_matmul_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            out[key] = [float(v) if "." in v else int(v) for v in vals]
    return out


def digits_of(codes, count=5):
    """Independent scalar base-3 decoding ((b // 3^i) % 3), vectorised."""
    c = np.asarray(codes, dtype=np.int64)[..., None]
    return (c // (3 ** np.arange(count))) % 3


def trits_of_package(codes, G):
    """codes [..., nb] -> trits [..., G] by the scalar decoding above."""
    d = digits_of(codes).reshape(*codes.shape[:-1], -1)
    return d[..., :G] - 1


def pack_independent(trits):
    """Pack a [..., G] trit array with a plain python base-3 sum."""
    G = trits.shape[-1]
    nb = (G + 4) // 5
    pad = np.ones((*trits.shape[:-1], nb * 5), np.int64)
    pad[..., :G] = trits + 1
    pad = pad.reshape(*trits.shape[:-1], nb, 5)
    return (pad * (3 ** np.arange(5))).sum(-1).astype(np.uint8)


def f16_bits_to_f64(h):
    return np.asarray(h, np.uint16).view(np.float16).astype(np.float64)


def torch_bf16_bits(x_f32):
    t = torch.from_numpy(np.ascontiguousarray(x_f32, np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# ---- IEEE rounding -----------------------------------------------------------

def test_f16_decode_all_patterns(oref):
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oref.f16_to_f64_array(h)
    ref = h.view(np.float16).astype(np.float64)
    fin = np.isfinite(ref)
    assert np.array_equal(ours[fin], ref[fin])
    assert np.array_equal(np.signbit(ours[fin]), np.signbit(ref[fin]))
    assert np.all(np.isnan(ours[np.isnan(ref)]))
    assert np.array_equal(ours[np.isinf(ref)], ref[np.isinf(ref)])


def test_f16_rounding_every_boundary(oref):
    # every non-negative finite fp16 value, each midpoint to the next value
    # (65536 stands for the first value past the largest finite one), and the
    # fp64 neighbours of every midpoint; then the same with negative sign.
    v = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    nxt = np.append(v[1:], 65536.0)
    mid = (v + nxt) / 2.0
    xs = np.concatenate([v, mid, np.nextafter(mid, np.inf),
                         np.nextafter(mid, -np.inf), [1e-300, 2.0 ** -26,
                                                      1e6, 65519.99]])
    xs = np.concatenate([xs, -xs])
    ours = oref.f64_to_f16_array(xs)
    with np.errstate(over="ignore"):
        ref = xs.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)
    assert oref.f64_to_f16(65520.0) == 0x7C00  # ties to even -> infinity
    assert oref.f64_to_f16(65519.0) == 0x7BFF


def test_bf16_rounding_every_boundary(oref):
    base = np.arange(0, 0x7F80, dtype=np.uint64) << 16
    offs = np.array([0, 1, 0x7FFF, 0x8000, 0x8001, 0xFFFF], np.uint64)
    pat = (base[:, None] + offs[None, :]).ravel().astype(np.uint32)
    pat = np.concatenate([pat, pat | np.uint32(0x80000000)])
    xs = pat.view(np.float32)
    ours = oref.f32_to_bf16_array(xs)
    assert np.array_equal(ours, torch_bf16_bits(xs))


# ---- base-3 packing ------------------------------------------------------------

def test_p2_worked_example(oref):
    g = read_golden("p2_pack_example.txt")
    trits = np.array(g["trits"], np.int8)
    packed = oref.pack_trits(trits, len(trits))
    assert list(packed) == g["byte"]
    assert list(oref.unpack_trits(packed, len(trits))) == g["trits"]


def test_all_243_words_are_a_bijection(oref):
    seen = {}
    for t in itertools.product((-1, 0, 1), repeat=5):
        b = int(oref.pack_trits(np.array(t, np.int8), 5)[0])
        assert b == sum((ti + 1) * 3 ** i for i, ti in enumerate(t))
        assert tuple(oref.unpack_trits([b], 5)) == t
        assert tuple(digits_of([b])[0] - 1) == t
        seen[b] = t
    assert sorted(seen) == list(range(243))


def test_bytes_243_to_255_rejected(oref):
    for b in range(243, 256):
        _, st = oref.unpack_trits([b], 5, check=False)
        assert st == oref.ERR_BAD_CODE
    for b in range(243):
        _, st = oref.unpack_trits([b], 5, check=False)
        assert st == oref.OK


@pytest.mark.parametrize("G", [1, 2, 4, 5, 7, 63, 64, 65, 128])
def test_round_trip_and_padding(oref, G):
    rng = np.random.default_rng(G)
    cases = [rng.integers(-1, 2, G) for _ in range(20)]
    cases += [np.full(G, v) for v in (-1, 0, 1)]
    nb = (G + 4) // 5
    for t in cases:
        t = t.astype(np.int8)
        packed = oref.pack_trits(t, G)
        assert len(packed) == nb
        assert np.array_equal(packed, pack_independent(t.astype(np.int64)))
        assert np.array_equal(oref.unpack_trits(packed, G), t)
        used = G - 5 * (nb - 1)  # trits in the last byte
        last_digits = digits_of(packed[-1:])[0]
        assert np.all(last_digits[used:] == 1)  # padding decodes to zero
        if used < 5:
            bad = packed.copy()
            d = used  # first padding digit: 1 -> 0 (or 2) changes the byte
            bad[-1] = int(bad[-1]) - 3 ** d
            _, st = oref.unpack_trits(bad, G, check=False)
            assert st == oref.ERR_BAD_CODE


# ---- byte accounting -------------------------------------------------------------

def test_byte_accounting(oref):
    g = read_golden("p2_byte_accounting.txt")
    G = g["G"][0]
    assert oref.bytes_per_group(G) == g["code_bytes"][0]
    assert oref.packed_bytes(oref.FMT_A, 1, G, G, 1) == g["group_bytes"][0]
    assert 8 * oref.packed_bytes(oref.FMT_A, 1, G, G, 1) / G == \
        g["bits_per_weight"][0]
    for G in (64, 128, 5, 32, 320):
        formula = 8 * (math.ceil(G / 5) + 2) / G
        n, k = 3, 4 * G
        got = oref.packed_bytes(oref.FMT_A, n, k, G, 1)
        assert 8 * got / (n * k) == formula
        assert oref.packed_bytes(oref.FMT_A, n, k, G, 2) == 2 * got
    assert 8 * oref.packed_bytes(oref.FMT_A, 1, 128, 128, 1) / 128 == 1.75
    # the workload sizes
    assert oref.packed_bytes(oref.FMT_A, 512, 1024, 64, 1) == 122_880
    assert oref.packed_bytes(oref.FMT_A, 28672, 8192, 64, 1) == 55_050_240
    assert oref.packed_bytes(oref.FMT_B, 4096, 4096, 0, 1) == 4096 * 4096 + 972


def test_format_b_storage_matches_page(oref):
    g = read_golden("p1_storage.txt")
    n, k = g["rho_layer_rows"][0], g["rho_layer_cols"][0]
    rho_bytes = 2 * n
    assert rho_bytes / oref.packed_bytes(oref.FMT_B, n, k, 0, 1) < \
        g["rho_overhead_max_fraction"][0]
    total = sum(l.n * l.k for _, l in I.decode_step_layers())
    assert total == 31_378_636_800
    # same order as the page's 31.0 GB for 410 layers, scaled to 420 layers
    per_layer_page = g["packed_weight_gb"][0] * 1e9 / g["packed_layers"][0]
    assert abs(total / (per_layer_page * len(I.decode_step_layers())) - 1) \
        < 0.05


# ---- format A quantization -------------------------------------------------

@pytest.fixture(scope="module")
def small(oref):
    cfg = I.fmt_a_small()
    Wb = I.bits(cfg["W"])
    codes, scales = oref.quantize_pack_A(Wb, cfg["G"], 1)
    return cfg, Wb, codes, scales


def test_zero_groups(oref, small):
    cfg, Wb, codes, scales = small
    assert len(cfg["zero_groups"]) == 8
    unpacked = oref.unpack_A(codes, scales, 512, 1024, 64, 1)
    for r, g in cfg["zero_groups"]:
        assert scales[0, r, g] == 0
        assert np.all(codes[0, r, g] == 121)  # every digit 1, padding too
        assert np.all(unpacked[r, g * 64:(g + 1) * 64] == 0x0000)  # +0.0


def test_underflowing_mean_is_a_zero_group(oref):
    W = np.full((1, 64), 2.0 ** -40, np.float32)
    W[0, ::2] *= -1
    codes, scales = oref.quantize_pack_A(torch_bf16_bits(W), 64, 1)
    assert scales[0, 0, 0] == 0
    assert np.all(codes == 121)


def test_ties_round_to_even(oref):
    # s = fp16(64 / 64) = 1 exactly; |W| = s/2 is a tie that rounds to 0,
    # 1.5 s rounds to 2 and clips to 1, values above s/2 give +-1.
    vals = [0.5] * 8 + [-0.5] * 8 + [7.0] * 6 + [1.5, -1.5] + \
        [0.50390625, -0.50390625] + [0.49609375] + [0.0] * 37
    extra = 64.0 - sum(abs(v) for v in vals)
    vals[-1] = extra
    W = np.array([vals], np.float32)
    assert math.fsum(abs(v) for v in vals) == 64.0
    codes, scales = oref.quantize_pack_A(torch_bf16_bits(W), 64, 1)
    assert scales[0, 0, 0] == 0x3C00
    t = trits_of_package(codes[0, 0, 0], 64)
    expect = [0] * 16 + [1] * 6 + [1, -1] + [1, -1] + [0] + [0] * 36 + [1]
    assert list(t) == expect


def test_scale_is_fp16_of_exact_mean(oref, small):
    _, Wb, codes, scales = small
    W = Wb.view(np.uint16)
    Wf = torch.from_numpy(W.view(np.int16)).view(torch.bfloat16).float() \
        .numpy().astype(np.float64).reshape(512, 16, 64)
    means = np.array([[math.fsum(np.abs(Wf[r, g])) / 64 for g in range(16)]
                      for r in range(512)])
    assert np.array_equal(scales[0], means.astype(np.float16).view(np.uint16))


def test_trits_follow_the_rounding_rule(oref, small):
    _, Wb, codes, scales = small
    Wf = torch.from_numpy(Wb.view(np.int16)).view(torch.bfloat16).float() \
        .numpy().astype(np.float64).reshape(512, 16, 64)
    s = f16_bits_to_f64(scales[0])[..., None]
    t = trits_of_package(codes[0], 64)
    with np.errstate(divide="ignore", invalid="ignore"):
        expect = np.clip(np.rint(Wf / s), -1, 1)  # rint: ties to even
    expect[np.broadcast_to(s == 0, expect.shape)] = 0
    assert np.array_equal(t, expect)
    assert np.all(np.abs(Wf - s * t) <= np.maximum(s / 2, np.abs(Wf) - s) + 0)


def test_unpack_is_bf16_of_scale_times_trit(oref, small):
    _, Wb, codes, scales = small
    s = f16_bits_to_f64(scales[0])[..., None].astype(np.float32)
    t = trits_of_package(codes[0], 64).astype(np.float32)
    expect = torch_bf16_bits((s * t).reshape(512, 1024))
    assert np.array_equal(oref.unpack_A(codes, scales, 512, 1024), expect)


def test_nonfinite_and_range(oref):
    base = np.full((1, 64), 0.25, np.float32)
    for bad in (np.inf, -np.inf, np.nan):
        W = base.copy()
        W[0, 17] = bad
        _, st = oref.quantize_pack_A(torch_bf16_bits(W), 64, 1, check=False)
        assert st == oref.ERR_NONFINITE
    W = np.full((1, 64), 65536.0, np.float32)  # mean rounds to fp16 inf
    _, st = oref.quantize_pack_A(torch_bf16_bits(W), 64, 1, check=False)
    assert st == oref.ERR_RANGE
    W = np.full((1, 64), 65280.0, np.float32)  # largest bf16 below 65520
    (codes, scales), st = oref.quantize_pack_A(torch_bf16_bits(W), 64, 1,
                                               check=False)
    assert st == oref.OK and scales[0, 0, 0] == 0x7BF8  # 65280 in fp16


def test_second_plane_fits_the_fp32_residual(oref):
    W = I.student_t_bf16(96, 8192, seed=3)
    Wb = I.bits(W)
    c1, s1 = oref.quantize_pack_A(Wb, 64, 1)
    c2, s2 = oref.quantize_pack_A(Wb, 64, 2)
    assert np.array_equal(c2[0], c1[0]) and np.array_equal(s2[0], s1[0])
    Wf = W.float().numpy().reshape(96, 128, 64)
    t1 = trits_of_package(c2[0], 64).astype(np.float32)
    sc1 = f16_bits_to_f64(s2[0])[..., None].astype(np.float32)
    R = (Wf - sc1 * t1).astype(np.float32)  # IEEE single arithmetic
    R64 = R.astype(np.float64)
    means = np.array([[math.fsum(np.abs(R64[r, g])) / 64 for g in range(128)]
                      for r in range(96)])
    assert np.array_equal(s2[1], means.astype(np.float16).view(np.uint16))
    sc2 = f16_bits_to_f64(s2[1])[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        expect = np.clip(np.rint(R64 / sc2), -1, 1)
    expect[np.broadcast_to(sc2 == 0, expect.shape)] = 0
    assert np.array_equal(trits_of_package(c2[1], 64), expect)
    # the second plane reduces the reconstruction error
    W64 = W.double().numpy()
    e1 = np.linalg.norm(W64 - oref.weights_A(c1, s1, 96, 8192, 64, 1))
    e2 = np.linalg.norm(W64 - oref.weights_A(c2, s2, 96, 8192, 64, 2))
    assert e2 < e1


# ---- format B code book ----------------------------------------------------

def test_lut_balanced_ternary_closed_form(oref):
    alpha = np.float32(0.02)
    lut = oref.build_lut(alpha, I.ladder_pow3().numpy())
    assert np.all(np.isnan(lut[243:]))
    d = digits_of(np.arange(243)) - 1  # c_1 .. c_5
    m = (d * (3 ** np.arange(4, -1, -1))).sum(-1)  # c_1 weighs 81
    assert sorted(m) == list(range(-121, 122))
    exact = float(alpha) * m / 81.0
    ulp = np.spacing(np.abs(lut[:243]).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(lut[:243] - exact) <= 2 * ulp)
    assert lut[121] == 0.0
    assert np.array_equal(lut[242 - np.arange(243)], -lut[:243])


def test_lut_digit_order_with_unit_ladders(oref):
    for i in range(5):
        ladder = np.zeros(5, np.float32)
        ladder[i] = 1.0
        lut = oref.build_lut(1.0, ladder)
        expect = (np.arange(243) // 3 ** i) % 3 - 1
        assert np.array_equal(lut[:243], expect.astype(np.float32))


def test_unpack_B(oref):
    g = torch.Generator().manual_seed(11)
    codes = torch.randint(0, 243, (6, 48), generator=g, dtype=torch.uint8)
    lut = oref.build_lut(0.02, I.ladder_pow3().numpy())
    rho = (0.5 + torch.rand(3, generator=g)).to(torch.float16)
    rho_f32 = rho.float().numpy()
    c = codes.numpy()
    got = oref.unpack_B(c, lut, I.bits(rho), 2)
    prod = (rho_f32[np.arange(6) // 2][:, None] * lut[c]).astype(np.float32)
    assert np.array_equal(got, torch_bf16_bits(prod))
    assert np.array_equal(oref.unpack_B(c, lut), torch_bf16_bits(lut[c]))
    bad = c.copy()
    bad[4, 7] = 250
    _, st = oref.unpack_B(bad, lut, check=False)
    assert st == oref.ERR_BAD_CODE


# ---- brute-force matmuls on exact inputs ---------------------------------------

def dyadic_x(batch, k, ldx, seed):
    rng = np.random.default_rng(seed)
    x = np.zeros((batch, ldx), np.float32)
    x[:, :k] = rng.integers(-64, 65, (batch, k)) / 8.0
    x[:, k:] = 1e30  # past K: must never be read
    return torch_bf16_bits(x), x[:, :k].astype(np.float64)


@pytest.mark.parametrize("planes", [1, 2])
def test_linear_A_brute_force(oref, planes):
    n, k, G, batch = 5, 192, 64, 3
    rng = np.random.default_rng(planes)
    trits = rng.integers(-1, 2, (planes, n, k // G, G))
    s_vals = np.array([0.0, 0.125, 0.75, 1.5, 3.0, 2.0 ** -10], np.float16)
    scales = rng.choice(s_vals, (planes, n, k // G)).view(np.uint16)
    codes = pack_independent(trits)
    xb, x = dyadic_x(batch, k, k + 8, planes)
    w = (f16_bits_to_f64(scales)[..., None] * trits).sum(0).reshape(n, k)
    y = oref.linear_A(codes, scales, n, k, xb, G, planes)
    assert np.array_equal(y, x @ w.T)  # every product and sum is exact
    rows = [4, 0, 2]
    y_rows = oref.linear_A(codes, scales, n, k, xb, G, planes, rows=rows)
    assert np.array_equal(y_rows, y[:, rows])
    assert np.array_equal(oref.weights_A(codes, scales, n, k, G, planes), w)


def test_linear_B_brute_force(oref):
    n, k, batch, rps = 7, 80, 4, 2
    ladder = np.array([1, 0.5, 0.25, 0.125, 0.0625], np.float32)
    lut = oref.build_lut(0.5, ladder)  # every entry a short dyadic number
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 243, (n, k)).astype(np.uint8)
    rho = np.array([1.5, 0.75, 0.5, 1.25], np.float16)
    xb, x = dyadic_x(batch, k, k + 3, 9)
    d = digits_of(codes) - 1
    w_nr = 0.5 * (d * ladder.astype(np.float64)).sum(-1)  # independent decode
    assert np.array_equal(lut[codes].astype(np.float64), w_nr)
    w = rho.astype(np.float64)[np.arange(n) // rps][:, None] * w_nr
    y = oref.linear_B(codes, lut, xb, rho.view(np.uint16), rps)
    assert np.array_equal(y, x @ w.T)
    y0 = oref.linear_B(codes, lut, xb)
    assert np.array_equal(y0, x @ w_nr.T)
    rows = [6, 1]
    assert np.array_equal(
        oref.linear_B(codes, lut, xb, rho.view(np.uint16), rps, rows=rows),
        y[:, rows])


# ---- Format B encoder ("A Discrete Weight Language...", sections 3.1, 3.3) --

def balanced_ternary_word(m):
    """Digits d_1..d_5 in {-1, 0, 1} with m = sum d_i 3^(5-i) (integer
    arithmetic, most significant first), |m| <= 121."""
    d = []
    for i in range(5):
        p = 3 ** (4 - i)
        q = int(round(m / p))
        q = max(-1, min(1, q))
        d.append(q)
        m -= q * p
    assert m == 0
    return d


def code_of_word(d):
    return sum((di + 1) * 3 ** i for i, di in enumerate(d))


def bf16_bits_of(values):
    t = torch.tensor(values, dtype=torch.float32).to(torch.bfloat16)
    return I.bits(t)


def test_encode_balanced_ternary_closed_form(oref):
    # integers m in [-121, 121] are exact in bf16; alpha = max |W| = 121, so
    # r_0 = m / 121 and the ladder s_i = 3^(5-i) / 121 makes the greedy path
    # spell the balanced-ternary digits of m (every decision has a margin of
    # at least s_5 / 2, far above fp32 rounding)
    ms = np.arange(-121, 122)
    W = bf16_bits_of(ms.astype(np.float32)[None, :])
    ladder = np.array([3.0 ** (4 - i) / 121.0 for i in range(5)], np.float32)
    for zeta in (0.0, 0.25, 0.5):
        codes, rho, alpha = oref.encode_B(W, ladder, zeta, 0)
        assert alpha == 121.0 and rho is None
        want = [code_of_word(balanced_ternary_word(int(m))) for m in ms]
        assert codes[0].tolist() == want
    assert codes[0][121] == 121  # m = 0: the all-zero word


def test_encode_tie_goes_to_zero_and_zero_bias(oref):
    ladder = np.array([1.0, 0.5, 0.25, 0.125, 0.0625], np.float32)
    # alpha = 1; r_0 = 0.5 = s_1 / 2 exactly: a tie, c_1 = 0 (then c_2 = +1)
    W = bf16_bits_of(np.array([[1.0, 0.5, 0.50390625, -0.5, 0.7, 0.0]],
                              np.float32))
    codes, _, _ = oref.encode_B(W, ladder, 0.5, 0)
    c0 = codes[0].astype(np.int64)
    first = c0 % 3 - 1  # c_1 (least significant digit)
    second = (c0 // 3) % 3 - 1
    assert first.tolist() == [1, 0, 1, 0, 1, 0]
    assert second[1] == 1 and second[3] == -1
    # zeta = 0.8 prefers 0 while |r| < 0.8 s_1: 0.7 and 0.50390625 give 0
    codes, _, _ = oref.encode_B(W, ladder, 0.8, 0)
    assert (codes[0].astype(np.int64) % 3 - 1).tolist() == [1, 0, 0, 0, 0, 0]


def _decode_words(codes, ladder):
    d = digits_of(codes) - 1  # [..., 5] with c_1 first
    return (d * np.asarray(ladder, np.float64)).sum(axis=-1)


@pytest.mark.parametrize("ladder,bound", [
    ([1.0, 1 / 3, 1 / 9, 1 / 27, 1 / 81], 1 / 162),
    ([1.0, 0.5, 0.25, 0.125, 0.0625], 1 / 32)])
def test_encode_greedy_residual_bound(oref, ladder, bound):
    # s_{i+1} <= s_i / 2 and |r_0| <= 1: each greedy step leaves
    # |r_i| <= s_i / 2, so |x / a - sum c_i s_i| <= s_5 / 2
    lad = np.array(ladder, np.float32)
    W = I.student_t_bf16(64, 256, seed=31)
    Wb = I.bits(W)
    codes, rho, alpha = oref.encode_B(Wb, lad, 0.5, 0)
    x = W.double().numpy()
    assert alpha == float(np.abs(x).max())
    err = np.abs(x / alpha - _decode_words(codes, lad))
    assert err.max() <= bound * (1 + 1e-5)
    # per-row scale: the same bound against each row's own maximum
    codes, rho, alpha = oref.encode_B(Wb, lad, 0.5, 1)
    rowmax = np.abs(x).max(axis=1, keepdims=True)
    err = np.abs(x / rowmax - _decode_words(codes, lad))
    assert err.max() <= bound * (1 + 1e-5)


def test_encode_row_and_head_scales(oref):
    lad = I.ladder_pow3().numpy()
    W = I.student_t_bf16(8, 128, seed=32).float()
    W[3] = 0.0                       # an all-zero row
    W[5] *= 8.0                      # exact power-of-two rescales
    W[6] *= 0.25
    Wb = I.bits(W.to(torch.bfloat16))
    x = W.to(torch.bfloat16).double().numpy()
    codes, rho, alpha = oref.encode_B(Wb, lad, 0.5, 1)
    rowmax = np.abs(x).max(axis=1)
    assert alpha == rowmax.max()
    # rho = fp16(alpha_n / alpha), through numpy's IEEE float16 rounding
    want = np.where(rowmax > 0, rowmax / alpha, 0.0).astype(np.float16)
    assert np.array_equal(rho, want.view(np.uint16))
    assert np.all(codes[3] == 121) and rho[3] == 0
    # scaling a row by a power of two leaves its words unchanged
    base = I.student_t_bf16(8, 128, seed=32)
    cb, _, _ = oref.encode_B(I.bits(base), lad, 0.5, 1)
    assert np.array_equal(codes[5], cb[5]) and np.array_equal(codes[6], cb[6])
    # per-head: one scale per 4 rows
    codes4, rho4, _ = oref.encode_B(Wb, lad, 0.5, 4)
    hmax = np.abs(x).reshape(2, 4, 128).max(axis=(1, 2))
    assert np.array_equal(rho4, (hmax / alpha).astype(np.float16).view(np.uint16))
    err = np.abs(x / np.repeat(hmax, 4)[:, None] - _decode_words(codes4, lad))
    assert err.max() <= 1 / 162 * (1 + 1e-5)


def test_encode_zero_matrix_and_nonfinite(oref):
    lad = I.ladder_pow3().numpy()
    codes, rho, alpha = oref.encode_B(np.zeros((2, 16), np.uint16), lad, 0.5, 1)
    assert alpha == 0.0 and np.all(codes == 121) and np.all(rho == 0)
    W = I.bits(I.student_t_bf16(2, 16, seed=1))
    W[1, 3] = 0x7FC0  # bf16 NaN
    _, st = oref.encode_B(W, lad, 0.5, 0, check=False)
    assert st == oref.ERR_NONFINITE


# ---- expert-indexed matmul (FUCINA README, "The method") -------------------

def test_linear_experts_A_brute_force(oref):
    # 5 experts, the first 2 hot (both planes); tokens routed to every expert,
    # some twice; exact dyadic inputs, so every product and sum is exact
    E, hot, n, k, G, tokens = 5, 2, 4, 128, 64, 7
    rng = np.random.default_rng(41)
    t1 = rng.integers(-1, 2, (E, n, k // G, G))
    t2 = rng.integers(-1, 2, (hot, n, k // G, G))
    s_vals = np.array([0.0, 0.125, 0.75, 1.5, 3.0, 2.0 ** -10], np.float16)
    s1 = rng.choice(s_vals, (E, n, k // G)).view(np.uint16)
    s2 = rng.choice(s_vals, (hot, n, k // G)).view(np.uint16)
    c1, c2 = pack_independent(t1), pack_independent(t2)
    ids = np.array([0, 4, 1, 3, 1, 2, 0], np.int32)
    xb, x = dyadic_x(tokens, k, k + 4, 17)
    w1 = (f16_bits_to_f64(s1)[..., None] * t1).reshape(E, n, k)
    w2 = (f16_bits_to_f64(s2)[..., None] * t2).reshape(hot, n, k)
    y = oref.linear_experts_A(c1, s1, c2, s2, E, hot, n, k, ids, xb, G)
    for t, e in enumerate(ids):
        w = w1[e] + (w2[e] if e < hot else 0.0)  # plane 2 only for hot ones
        assert np.array_equal(y[t], w @ x[t]), (t, e)
    # no hot experts: plane 1 everywhere
    y0 = oref.linear_experts_A(c1, s1, None, None, E, 0, n, k, ids, xb, G)
    for t, e in enumerate(ids):
        assert np.array_equal(y0[t], w1[e] @ x[t])
    _, st = oref.linear_experts_A(c1, s1, c2, s2, E, hot, n, k,
                                  np.array([5], np.int32), xb[:1], G,
                                  check=False)
    assert st == oref.ERR_INVALID_ARG


# ---- adaptive alphabets (one code book per block of rows, section 8.3) -------

def _block_weights_numpy(codes, alpha, ladders, lut_rows):
    """fp32(alpha * sum_i c_i a_{b,i}) per weight, from the code's base-3
    digits (first digit least significant) and the ladder of the row's
    block b = n // lut_rows; the sum in fp64 over ascending i."""
    c = codes.astype(np.int64)
    blk = np.arange(codes.shape[0]) // lut_rows
    lad = ladders.astype(np.float64)[blk]  # [n][5]
    s = np.zeros(codes.shape, np.float64)
    for i in range(5):
        s = s + ((c // 3 ** i) % 3 - 1) * lad[:, i:i + 1]
    return (np.float64(alpha) * s).astype(np.float32).astype(np.float64)


@pytest.mark.parametrize("n,lut_rows", [(70, 32), (64, 32), (5, 1), (9, 4)])
def test_adaptive_alphabet_per_block_code_books(oref, n, lut_rows):
    rng = np.random.default_rng(n * 7 + lut_rows)
    k = 48
    nb = -(-n // lut_rows)
    ladders = rng.uniform(0.01, 1.0, (nb, 5)).astype(np.float32)
    alpha = np.float32(0.03)
    luts = np.stack([oref.build_lut(alpha, ladders[b]) for b in range(nb)])
    codes = rng.integers(0, 243, (n, k)).astype(np.uint8)
    want = _block_weights_numpy(codes, alpha, ladders, lut_rows)
    got = oref.weights_B(codes, luts, lut_rows=lut_rows)
    assert np.array_equal(got, want)
    # unpack: bf16 of the same weights
    ub = oref.unpack_B(codes, luts, lut_rows=lut_rows)
    ref = torch.from_numpy(want.astype(np.float32)).to(torch.bfloat16)
    assert np.array_equal(ub, ref.view(torch.int16).numpy().view(np.uint16))
    # matmul against numpy over the same exact weights
    x = I.x_normal(3, k, 5)
    xb = I.bits(x)
    y = oref.linear_B(codes, luts, xb, lut_rows=lut_rows)
    x64 = x.double().numpy()
    np.testing.assert_allclose(y, x64 @ want.T, rtol=1e-12, atol=1e-15)


def test_adaptive_alphabet_equal_books_match_single_book(oref):
    rng = np.random.default_rng(2)
    codes = rng.integers(0, 243, (40, 32)).astype(np.uint8)
    lut = oref.build_lut(np.float32(0.02), I.ladder_pow3().numpy())
    luts = np.stack([lut] * 4)
    x = I.bits(I.x_normal(2, 32, 1))
    assert np.array_equal(oref.linear_B(codes, luts, x, lut_rows=10),
                          oref.linear_B(codes, lut, x))


# ---- 7-bit truncated alphabet (section 8.1) ---------------------------------

def _pack7_python(codes):
    """Independent restatement: the used table is np.unique (padded with the
    all-zero word 121), and each 16-index chunk is the little-endian 14-byte
    image of sum_j idx_j * 2^(7 j)."""
    used = np.unique(codes)
    idx = np.searchsorted(used, codes)
    n, k = codes.shape
    out = bytearray()
    for r in range(n):
        for ch in range(k // 16):
            v = 0
            for j in range(16):
                v |= int(idx[r, 16 * ch + j]) << (7 * j)
            out += v.to_bytes(14, "little")
    table = np.full(128, 121, np.uint8)
    table[:len(used)] = used
    return table, len(used), np.frombuffer(bytes(out), np.uint8).reshape(n, -1)


@pytest.mark.parametrize("n,k,distinct", [(3, 32, 45), (7, 64, 128), (1, 16, 1),
                                          (5, 48, 18)])
def test_pack7_layout_and_round_trip(oref, n, k, distinct):
    rng = np.random.default_rng(n * 100 + distinct)
    words = rng.choice(243, distinct, replace=False)
    codes = rng.choice(words, (n, k)).astype(np.uint8)
    codes.reshape(-1)[:distinct] = words  # every word present
    used, cnt, packed = oref.pack7(codes)
    t_used, t_cnt, t_packed = _pack7_python(codes)
    assert cnt == t_cnt == distinct
    assert np.array_equal(used, t_used)
    assert np.array_equal(packed, t_packed)
    assert np.array_equal(oref.unpack7_codes(packed, used, n, k), codes)


def test_pack7_too_many_words_and_shape(oref):
    codes = np.arange(129, dtype=np.uint8).repeat(16).reshape(129, 16)
    _, st = oref.pack7(codes, check=False)
    assert st == oref.ERR_RANGE
    codes = np.zeros((2, 24), np.uint8)
    _, st = oref.pack7(codes, check=False)
    assert st == oref.ERR_INVALID_ARG


def test_linear_b7_equals_format_b(oref):
    rng = np.random.default_rng(4)
    words = rng.choice(243, 45, replace=False)
    codes = rng.choice(words, (20, 64)).astype(np.uint8)
    lut = oref.build_lut(np.float32(0.02), I.ladder_pow3().numpy())
    used, _, packed = oref.pack7(codes)
    x = I.bits(I.x_normal(3, 64, 8))
    assert np.array_equal(oref.linear_B7(packed, used, 20, 64, lut, x),
                          oref.linear_B(codes, lut, x))

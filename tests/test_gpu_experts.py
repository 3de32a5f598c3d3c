"""GPU parity of tq_linear_experts (expert-indexed Format A matmul: the
second plane only on the hot-expert prefix 0 .. n_hot - 1, FUCINA README,
"The method") against the fp64 oracle oref_linear_experts_A, with the
tolerance of test_gpu_linear applied to each token with its own expert's
row maxima: ragged shapes, no / some / all hot experts, repeated and
unordered ids, padded strides, an invalid id (NaN row, status) and a
decode-sized layer."""
import numpy as np
import pytest
import torch

from oracle import oref
from packed_weight_matmul_b200 import inputs as I
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

G = 64


def _experts(E, n_hot, n, k, seed):
    """Per expert a two-plane package from the oracle's quantizer (plane 1 of
    a two-plane package is the one-plane package); plane 1 of every expert,
    plane 2 of the hot prefix."""
    c1, s1, c2, s2 = [], [], [], []
    for e in range(E):
        W = I.student_t_bf16(n, k, seed=seed * 131 + e)
        codes, scales = oref.quantize_pack_A(I.bits(W), G, 2)
        codes = np.asarray(codes).reshape(2, -1)
        scales = np.asarray(scales).reshape(2, -1)
        c1.append(codes[0]); s1.append(scales[0])
        if e < n_hot:
            c2.append(codes[1]); s2.append(scales[1])
    cat = lambda a: np.concatenate(a) if a else None
    return cat(c1), cat(s1), cat(c2), cat(s2)


def _absmax(c1, s1, c2, s2, E, n_hot, n, k):
    per = n * (k // G)
    out = []
    for e in range(E):
        c = c1[e * per * 13:(e + 1) * per * 13]
        s = s1[e * per:(e + 1) * per]
        if e < n_hot:
            c = np.concatenate([c, c2[e * per * 13:(e + 1) * per * 13]])
            s = np.concatenate([s, s2[e * per:(e + 1) * per]])
            out.append(U.absmax_rows_a(c, s, n, k, G, 2))
        else:
            out.append(U.absmax_rows_a(c, s, n, k, G, 1))
    return out


def _device(c1, s1, c2, s2, E, n_hot, n, k):
    d = [U.to_dev_u8(c1), U.to_dev_u16(s1),
         U.to_dev_u8(c2) if n_hot else None,
         U.to_dev_u16(s2) if n_hot else None]
    return U.tq().experts_a(d[0], d[1], E, n, k, n_hot, d[2], d[3])


def _run(E, n_hot, n, k, ids, seed=1, ldx=None, ldy=None):
    c1, s1, c2, s2 = _experts(E, n_hot, n, k, seed)
    w = _device(c1, s1, c2, s2, E, n_hot, n, k)
    T = len(ids)
    ldx = k if ldx is None else ldx
    ldy = n if ldy is None else ldy
    x = I.x_normal(T, k, seed + 7)
    xb = U.x_bits(x)
    xd = torch.full((T, ldx), float("nan"), dtype=torch.bfloat16,
                    device=U.DEV)
    xd[:, :k] = x.to(U.DEV)
    yd = torch.full((T, ldy), 5.0, dtype=torch.float32, device=U.DEV)
    idd = torch.tensor(ids, dtype=torch.int32, device=U.DEV)
    st = U.status_tensor()
    U.tq().tq_linear_experts(w, idd, xd, yd, ldx=ldx, ldy=ldy, status=st)
    torch.cuda.synchronize()
    y = yd.cpu().numpy()
    assert np.all(y[:, n:] == 5.0)  # padding untouched
    return y[:, :n], (c1, s1, c2, s2), xb, int(st.item())


def _check(y, pkg, xb, E, n_hot, n, k, ids, what):
    c1, s1, c2, s2 = pkg
    valid = [t for t, e in enumerate(ids) if 0 <= e < E]
    ref = oref.linear_experts_A(c1, s1, c2, s2, E, n_hot, n, k,
                                np.array([ids[t] for t in valid], np.int32),
                                xb[valid], G)
    am = _absmax(c1, s1, c2, s2, E, n_hot, n, k)
    for i, t in enumerate(valid):
        U.check_tolerance(y[t:t + 1], ref[i:i + 1], xb[t:t + 1], am[ids[t]],
                          f"{what} token {t} expert {ids[t]}")


@pytest.mark.parametrize("E,n_hot,n,k,ids", [
    (5, 2, 300, 1024, [0, 4, 1, 1, 2, 3, 0, 4, 2]),
    (3, 0, 130, 4224, [2, 2, 0, 1]),
    (2, 2, 257, 512, [1, 0, 1]),
    (1, 1, 64, 64, [0]),
    (4, 1, 1000, 2048, [3, 1, 0, 2, 3, 3, 1]),
])
def test_experts_ragged(E, n_hot, n, k, ids):
    y, pkg, xb, st = _run(E, n_hot, n, k, ids)
    assert st == 0
    _check(y, pkg, xb, E, n_hot, n, k, ids, f"E={E} hot={n_hot} {n}x{k}")


def test_experts_padded_strides():
    ids = [1, 0, 2, 1]
    y, pkg, xb, st = _run(3, 1, 200, 1024, ids, ldx=1024 + 24, ldy=200 + 3)
    assert st == 0
    _check(y, pkg, xb, 3, 1, 200, 1024, ids, "padded")


def test_experts_invalid_id_is_nan_and_reported():
    ids = [0, 7, 1, -1, 2]
    y, pkg, xb, st = _run(3, 1, 160, 1024, ids)
    assert st == U.tq().TQ_ERR_INVALID_ARG
    assert np.all(np.isnan(y[1])) and np.all(np.isnan(y[3]))
    assert np.all(np.isfinite(y[[0, 2, 4]]))
    _check(y, pkg, xb, 3, 1, 160, 1024, ids, "invalid id")


def test_experts_decode_layer_and_determinism():
    # a decode step's worth of routed tokens over a small expert layer
    rng = np.random.default_rng(3)
    E, n_hot, n, k = 16, 4, 768, 2048
    ids = [int(v) for v in rng.integers(0, E, 48)]
    c1, s1, c2, s2 = _experts(E, n_hot, n, k, 5)
    w = _device(c1, s1, c2, s2, E, n_hot, n, k)
    x = I.x_normal(len(ids), k, 9)
    xb = U.x_bits(x)
    xd = x.to(U.DEV)
    idd = torch.tensor(ids, dtype=torch.int32, device=U.DEV)
    ys = []
    for _ in range(2):
        yd = torch.empty(len(ids), n, dtype=torch.float32, device=U.DEV)
        U.tq().tq_linear_experts(w, idd, xd, yd)
        torch.cuda.synchronize()
        ys.append(yd.cpu().numpy())
    assert np.array_equal(ys[0], ys[1])
    _check(ys[0], (c1, s1, c2, s2), xb, E, n_hot, n, k, ids, "decode layer")

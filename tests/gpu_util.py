"""Helpers shared by the GPU parity tests: run the library through its C ABI
on seeded inputs, and compare with the oracle on the same host arrays."""
import numpy as np
import torch

from oracle import oref
from packed_weight_matmul_b200 import inputs as I

DEV = "cuda:0"
TOL = 2e-3  # |y - y_exact| <= TOL * ||x_b||_2 * max_k |w[n][k]|


def tq():
    from packed_weight_matmul_b200 import tq as _tq
    return _tq


def status_tensor():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def quantize(W, G=64, planes=1):
    """W: bf16 tensor (any device) -> (codes np [planes][n][k/G][nb],
    scales np uint16 [planes][n][k/G], status)."""
    n, k = W.shape
    nb = (G + 4) // 5
    Wd = W.to(DEV).contiguous()
    codes = torch.empty(planes * n * (k // G) * nb, dtype=torch.uint8,
                        device=DEV)
    scales = torch.empty(planes * n * (k // G), dtype=torch.int16, device=DEV)
    st = status_tensor()
    tq().tq_quantize_pack(Wd, G, planes, codes, scales, st)
    torch.cuda.synchronize()
    return (codes.view(planes, n, k // G, nb).cpu().numpy(),
            scales.view(planes, n, k // G).cpu().numpy().view(np.uint16),
            int(st.item()))


def to_dev_u8(a):
    return torch.from_numpy(np.ascontiguousarray(a).reshape(-1)).to(DEV)


def to_dev_u16(a):
    return torch.from_numpy(
        np.ascontiguousarray(a).view(np.int16).reshape(-1)).to(DEV)


def weights_a_dev(codes, scales, n, k, G=64, planes=1):
    c, s = to_dev_u8(codes), to_dev_u16(scales)
    return tq().weights_a(c, s, n, k, G, planes)


def weights_b_dev(codes, lut, rho=None, rps=0):
    c = codes.to(DEV) if torch.is_tensor(codes) else to_dev_u8(codes)
    n, k = codes.shape
    L = torch.from_numpy(np.ascontiguousarray(lut, np.float32)).to(DEV)
    r = None
    if rho is not None:
        r = rho.view(torch.int16).to(DEV) if torch.is_tensor(rho) else \
            to_dev_u16(rho)
    return tq().weights_b(c, L, r, rps, n=n, k=k)


def linear(w, x_bf16, ldx=None, ldy=None, y_fill=float("nan")):
    """Run tq_linear on x [batch][k] bf16 (host or device) with optional
    padded strides. Returns (y [batch][n] fp32 numpy, full padded y)."""
    batch, k = x_bf16.shape
    ldx = k if ldx is None else ldx
    ldy = w.n if ldy is None else ldy
    xd = torch.zeros(batch, ldx, dtype=torch.bfloat16, device=DEV)
    xd[:, :k] = x_bf16.to(DEV)
    if ldx > k:
        xd[:, k:] = float("nan")  # never read
    y = torch.full((batch, ldy), y_fill, dtype=torch.float32, device=DEV)
    tq().tq_linear(w, xd, y, batch=batch, ldx=ldx, ldy=ldy)
    torch.cuda.synchronize()
    yh = y.cpu().numpy()
    return yh[:, :w.n], yh


def check_tolerance(y_gpu, y_ref, x_bits, w_absmax, what=""):
    x64 = torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)) \
        .view(torch.bfloat16).double().numpy()
    xn = np.linalg.norm(x64, axis=1)
    tol = TOL * xn[:, None] * np.asarray(w_absmax)[None, :]
    err = np.abs(y_gpu.astype(np.float64) - y_ref)
    bad = ~(err <= tol)
    if bad.any():
        b, n = np.argwhere(bad)[0]
        raise AssertionError(
            f"{what}: {bad.sum()} outputs out of tolerance; first (b={b}, "
            f"n={n}): gpu={y_gpu[b, n]!r} ref={y_ref[b, n]!r} "
            f"tol={tol[b, n]!r}")
    return float(np.max(err / np.where(tol > 0, tol, 1)))


def absmax_rows_a(codes, scales, n, k, G, planes, rows=None):
    return np.abs(oref.weights_A(codes, scales, n, k, G, planes,
                                 rows=rows)).max(axis=1)


def absmax_rows_b(codes, lut, rho=None, rps=0, rows=None):
    return np.abs(oref.weights_B(codes, lut, rho, rps, rows=rows)).max(axis=1)


def x_bits(x):
    return I.bits(x.cpu())

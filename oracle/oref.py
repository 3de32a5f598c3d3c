"""ctypes wrapper of the CPU oracle (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline and
reference legs may import this module. It never touches the CUDA library.

Arrays are numpy: bf16 and fp16 values travel as their uint16 bit patterns.
Every function raises OracleError on a non-zero status unless `check=False`,
in which case it returns (result, status).
"""
import ctypes as C
import os

import numpy as np

from . import build as _build

OK, ERR_INVALID_ARG, ERR_SHAPE, ERR_UNSUPPORTED = 0, 1, 2, 4
ERR_BAD_CODE, ERR_NONFINITE, ERR_RANGE = 5, 6, 7
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "SHAPE", 4: "UNSUPPORTED",
                5: "BAD_CODE", 6: "NONFINITE", 7: "RANGE"}
FMT_A, FMT_B = 1, 2


class OracleError(RuntimeError):
    def __init__(self, status):
        super().__init__(f"oracle status {STATUS_NAMES.get(status, status)}")
        self.status = status


_lib = None


def lib(path: str = None):
    """Load (building if stale) the oracle library. `path` loads another
    build of the oracle sources, e.g. a deliberately mutated copy."""
    global _lib
    if path is not None:
        return _declare(C.CDLL(path))
    if _lib is None:
        override = os.environ.get("OREF_LIB")  # a mutated build, for tests
        if override:
            _lib = _declare(C.CDLL(override))
            return _lib
        if _build.needs_build():
            _build.build()
        _lib = _declare(C.CDLL(_build.LIB))
    return _lib


def _declare(L):
    i64, i32, u16 = C.c_int64, C.c_int32, C.c_uint16
    P = C.c_void_p
    L.oref_f64_to_f16.restype = u16
    L.oref_f64_to_f16.argtypes = [C.c_double]
    L.oref_f16_to_f64.restype = C.c_double
    L.oref_f16_to_f64.argtypes = [u16]
    L.oref_f64_to_bf16.restype = u16
    L.oref_f64_to_bf16.argtypes = [C.c_double]
    L.oref_f32_to_bf16.restype = u16
    L.oref_f32_to_bf16.argtypes = [C.c_float]
    L.oref_bf16_to_f64.restype = C.c_double
    L.oref_bf16_to_f64.argtypes = [u16]
    for name in ("oref_f64_to_f16_n", "oref_f32_to_bf16_n",
                 "oref_f16_to_f64_n"):
        getattr(L, name).restype = None
        getattr(L, name).argtypes = [P, i64, P]
    L.oref_bytes_per_group.restype = i32
    L.oref_bytes_per_group.argtypes = [i32]
    L.oref_packed_bytes.restype = C.c_uint64
    L.oref_packed_bytes.argtypes = [i32, i64, i64, i32, i32]
    L.oref_pack_trits.restype = None
    L.oref_pack_trits.argtypes = [P, i32, P]
    L.oref_unpack_trits.restype = C.c_int
    L.oref_unpack_trits.argtypes = [P, i32, P]
    L.oref_quantize_pack_A.restype = C.c_int
    L.oref_quantize_pack_A.argtypes = [P, i64, i64, i32, i32, P, P]
    L.oref_unpack_A.restype = C.c_int
    L.oref_unpack_A.argtypes = [P, P, i64, i64, i32, i32, P]
    L.oref_weights_A.restype = C.c_int
    L.oref_weights_A.argtypes = [P, P, i64, i64, i32, i32, P, i64, P]
    L.oref_linear_A.restype = C.c_int
    L.oref_linear_A.argtypes = [P, P, i64, i64, i32, i32, P, i64, P, i64,
                                i64, P]
    L.oref_linear_experts_A.restype = C.c_int
    L.oref_linear_experts_A.argtypes = [P, P, P, P, i32, i32, i64, i64, i32,
                                        P, i64, P, i64, P]
    L.oref_build_lut.restype = C.c_int
    L.oref_build_lut.argtypes = [C.c_float, P, P]
    L.oref_unpack_B.restype = C.c_int
    L.oref_unpack_B.argtypes = [P, i64, i64, P, P, i32, P]
    L.oref_weights_B.restype = C.c_int
    L.oref_weights_B.argtypes = [P, i64, i64, P, P, i32, P, i64, P]
    L.oref_encode_B.restype = C.c_int
    L.oref_encode_B.argtypes = [P, i64, i64, P, C.c_float, i32, P, P, P]
    L.oref_unpack_Bx.restype = C.c_int
    L.oref_unpack_Bx.argtypes = [P, i64, i64, P, i64, P, i32, P]
    L.oref_weights_Bx.restype = C.c_int
    L.oref_weights_Bx.argtypes = [P, i64, i64, P, i64, P, i32, P, i64, P]
    L.oref_linear_Bx.restype = C.c_int
    L.oref_linear_Bx.argtypes = [P, i64, i64, P, i64, P, i32, P, i64, P, i64,
                                 i64, P]
    L.oref_pack7.restype = C.c_int
    L.oref_pack7.argtypes = [P, i64, i64, P, P, P]
    L.oref_unpack7_codes.restype = C.c_int
    L.oref_unpack7_codes.argtypes = [P, P, i64, i64, P]
    L.oref_linear_B.restype = C.c_int
    L.oref_linear_B.argtypes = [P, i64, i64, P, P, i32, P, i64, P, i64, i64,
                                P]
    return L


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def _ret(value, status, check):
    if check:
        if status != OK:
            raise OracleError(status)
        return value
    return value, status


# ---- scalar rounding ------------------------------------------------------

def f64_to_f16(x: float, L=None) -> int:
    return (L or lib()).oref_f64_to_f16(float(x))


def f16_to_f64(h: int, L=None) -> float:
    return (L or lib()).oref_f16_to_f64(int(h))


def f64_to_bf16(x: float, L=None) -> int:
    return (L or lib()).oref_f64_to_bf16(float(x))


def bf16_to_f64(b: int, L=None) -> float:
    return (L or lib()).oref_bf16_to_f64(int(b))


def f64_to_f16_array(x, L=None) -> np.ndarray:
    x = _c(x, np.float64)
    out = np.zeros(x.shape, np.uint16)
    (L or lib()).oref_f64_to_f16_n(_p(x), x.size, _p(out))
    return out


def f32_to_bf16_array(x, L=None) -> np.ndarray:
    x = _c(x, np.float32)
    out = np.zeros(x.shape, np.uint16)
    (L or lib()).oref_f32_to_bf16_n(_p(x), x.size, _p(out))
    return out


def f16_to_f64_array(h, L=None) -> np.ndarray:
    h = _c(h, np.uint16)
    out = np.zeros(h.shape, np.float64)
    (L or lib()).oref_f16_to_f64_n(_p(h), h.size, _p(out))
    return out


def bytes_per_group(G: int, L=None) -> int:
    return (L or lib()).oref_bytes_per_group(G)


def packed_bytes(fmt: int, n: int, k: int, G: int, planes: int, L=None) -> int:
    return (L or lib()).oref_packed_bytes(fmt, n, k, G, planes)


# ---- format A ---------------------------------------------------------------

def pack_trits(t, G: int, L=None) -> np.ndarray:
    t = _c(t, np.int8)
    out = np.zeros(bytes_per_group(G, L), np.uint8)
    (L or lib()).oref_pack_trits(_p(t), G, _p(out))
    return out


def unpack_trits(b, G: int, check=True, L=None):
    b = _c(b, np.uint8)
    t = np.zeros(G, np.int8)
    st = (L or lib()).oref_unpack_trits(_p(b), G, _p(t))
    return _ret(t, st, check)


def quantize_pack_A(W_bits, G: int = 64, planes: int = 1, check=True, L=None):
    """W_bits: uint16 [n][k] bf16 patterns -> (codes [planes][n][k/G][nb],
    scales uint16 [planes][n][k/G])."""
    W = _c(W_bits, np.uint16)
    n, k = W.shape
    nb = bytes_per_group(G, L)
    codes = np.zeros((planes, n, k // G, nb), np.uint8)
    scales = np.zeros((planes, n, k // G), np.uint16)
    st = (L or lib()).oref_quantize_pack_A(_p(W), n, k, G, planes, _p(codes),
                                           _p(scales))
    return _ret((codes, scales), st, check)


def unpack_A(codes, scales, n, k, G=64, planes=1, check=True, L=None):
    codes, scales = _c(codes, np.uint8), _c(scales, np.uint16)
    out = np.zeros((n, k), np.uint16)
    st = (L or lib()).oref_unpack_A(_p(codes), _p(scales), n, k, G, planes,
                                    _p(out))
    return _ret(out, st, check)


def weights_A(codes, scales, n, k, G=64, planes=1, rows=None, check=True,
              L=None):
    codes, scales = _c(codes, np.uint8), _c(scales, np.uint16)
    rows = _c(rows, np.int64)
    nr = n if rows is None else len(rows)
    out = np.zeros((nr, k), np.float64)
    st = (L or lib()).oref_weights_A(_p(codes), _p(scales), n, k, G, planes,
                                     _p(rows), nr, _p(out))
    return _ret(out, st, check)


def linear_A(codes, scales, n, k, x_bits, G=64, planes=1, rows=None,
             check=True, L=None):
    """y[b][i] (fp64) for x_bits uint16 [batch][ldx] (bf16)."""
    codes, scales = _c(codes, np.uint8), _c(scales, np.uint16)
    x = _c(x_bits, np.uint16)
    rows = _c(rows, np.int64)
    batch, ldx = x.shape
    nr = n if rows is None else len(rows)
    y = np.zeros((batch, nr), np.float64)
    st = (L or lib()).oref_linear_A(_p(codes), _p(scales), n, k, G, planes,
                                    _p(rows), nr, _p(x), batch, ldx, _p(y))
    return _ret(y, st, check)


# ---- format B ---------------------------------------------------------------

def build_lut(alpha: float, ladder, check=True, L=None):
    ladder = _c(ladder, np.float32)
    lut = np.zeros(256, np.float32)
    st = (L or lib()).oref_build_lut(C.c_float(alpha), _p(ladder), _p(lut))
    return _ret(lut, st, check)


def unpack_B(codes, lut, rho=None, rps=0, check=True, L=None, lut_rows=0):
    """lut: one code book [256], or with lut_rows > 0 one per block of
    lut_rows rows ([ceil(n / lut_rows)][256], section 8.3)."""
    codes = _c(codes, np.uint8)
    n, k = codes.shape
    lut, rho = _c(lut, np.float32), _c(rho, np.uint16)
    out = np.zeros((n, k), np.uint16)
    st = (L or lib()).oref_unpack_Bx(_p(codes), n, k, _p(lut), lut_rows,
                                     _p(rho), rps, _p(out))
    return _ret(out, st, check)


def weights_B(codes, lut, rho=None, rps=0, rows=None, check=True, L=None,
              lut_rows=0):
    codes = _c(codes, np.uint8)
    n, k = codes.shape
    lut, rho, rows = _c(lut, np.float32), _c(rho, np.uint16), _c(rows, np.int64)
    nr = n if rows is None else len(rows)
    out = np.zeros((nr, k), np.float64)
    st = (L or lib()).oref_weights_Bx(_p(codes), n, k, _p(lut), lut_rows,
                                      _p(rho), rps, _p(rows), nr, _p(out))
    return _ret(out, st, check)


def linear_B(codes, lut, x_bits, rho=None, rps=0, rows=None, check=True,
             L=None, lut_rows=0):
    codes = _c(codes, np.uint8)
    n, k = codes.shape
    lut, rho, rows = _c(lut, np.float32), _c(rho, np.uint16), _c(rows, np.int64)
    x = _c(x_bits, np.uint16)
    batch, ldx = x.shape
    nr = n if rows is None else len(rows)
    y = np.zeros((batch, nr), np.float64)
    st = (L or lib()).oref_linear_Bx(_p(codes), n, k, _p(lut), lut_rows,
                                     _p(rho), rps, _p(rows), nr, _p(x), batch,
                                     ldx, _p(y))
    return _ret(y, st, check)



def encode_B(W_bits, ladder, zeta=0.5, rps=0, check=True, L=None):
    """W_bits: uint16 [n][k] bf16 patterns -> (codes uint8 [n][k],
    rho uint16 [ceil(n / rps)] fp16 patterns or None, alpha float)."""
    W = _c(W_bits, np.uint16)
    n, k = W.shape
    ladder = _c(ladder, np.float32)
    codes = np.zeros((n, k), np.uint8)
    rho = np.zeros(((n + rps - 1) // rps,), np.uint16) if rps > 0 else None
    alpha = np.zeros(1, np.float32)
    st = (L or lib()).oref_encode_B(_p(W), n, k, _p(ladder), C.c_float(zeta),
                                    rps, _p(codes), _p(rho), _p(alpha))
    return _ret((codes, rho, float(alpha[0])), st, check)


def linear_experts_A(codes1, scales1, codes2, scales2, n_experts, n_hot, n, k,
                     ids, x_bits, G=64, check=True, L=None):
    """Expert-indexed Format A matmul: plane 1 of every expert in codes1 /
    scales1 ([E][n][k/G][nb], [E][n][k/G]), plane 2 of the n_hot hot experts
    in codes2 / scales2; token t uses expert ids[t]. Returns y [tokens][n]."""
    codes1, scales1 = _c(codes1, np.uint8), _c(scales1, np.uint16)
    codes2 = _c(codes2, np.uint8) if n_hot else None
    scales2 = _c(scales2, np.uint16) if n_hot else None
    ids = _c(ids, np.int32)
    x = _c(x_bits, np.uint16)
    tokens, ldx = x.shape
    y = np.zeros((tokens, n), np.float64)
    st = (L or lib()).oref_linear_experts_A(
        _p(codes1), _p(scales1), _p(codes2), _p(scales2), n_experts, n_hot,
        n, k, G, _p(ids), tokens, _p(x), ldx, _p(y))
    return _ret(y, st, check)


# ---- 7-bit truncated alphabet (section 8.1) ---------------------------------

def pack7(codes, check=True, L=None):
    """codes uint8 [n][k] (k % 16 == 0) -> (used uint8 [128], n_used,
    packed uint8 [n][14 k / 16])."""
    codes = _c(codes, np.uint8)
    n, k = codes.shape
    used = np.zeros(128, np.uint8)
    cnt = np.zeros(1, np.int32)
    packed = np.zeros((n, 14 * (k // 16)), np.uint8)
    st = (L or lib()).oref_pack7(_p(codes), n, k, _p(used), _p(cnt),
                                 _p(packed))
    return _ret((used, int(cnt[0]), packed), st, check)


def unpack7_codes(packed, used, n, k, check=True, L=None):
    packed, used = _c(packed, np.uint8), _c(used, np.uint8)
    codes = np.zeros((n, k), np.uint8)
    st = (L or lib()).oref_unpack7_codes(_p(packed), _p(used), n, k,
                                         _p(codes))
    return _ret(codes, st, check)


def linear_B7(packed, used, n, k, lut, x_bits, rho=None, rps=0, rows=None,
              check=True, L=None):
    """The 7-bit layer's matmul: index i is the code used[i], then Format
    B's matmul over the same code book."""
    codes = unpack7_codes(packed, used, n, k, L=L)
    return linear_B(codes, lut, x_bits, rho, rps, rows, check, L)


def unpack_B7(packed, used, n, k, lut, rho=None, rps=0, check=True, L=None):
    codes = unpack7_codes(packed, used, n, k, L=L)
    return unpack_B(codes, lut, rho, rps, check, L)


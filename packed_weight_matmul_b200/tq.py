"""Thin ctypes binding of libtq.so (include/tq.h), for torch tensors.

Argument marshalling only: every step of the computation runs in the CUDA
library. The names follow the C entry points. Importing this module loads
libtq.so and raises TqError if it has not been built: there is no fallback.

Device tensors are passed by pointer; the CUDA stream defaults to torch's
current stream. A non-TQ_OK status raises TqError (status in `.status`).
"""
import ctypes as C
import os

import numpy as np
import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                        "libtq.so")

TQ_OK, TQ_ERR_INVALID_ARG, TQ_ERR_SHAPE, TQ_ERR_ALIGNMENT = 0, 1, 2, 3
TQ_ERR_UNSUPPORTED, TQ_ERR_BAD_CODE, TQ_ERR_NONFINITE = 4, 5, 6
TQ_ERR_RANGE, TQ_ERR_TIMEOUT, TQ_ERR_CUDA = 7, 8, 9
TQ_FMT_A, TQ_FMT_B, TQ_FMT_B7 = 1, 2, 3

# Every entry point declared in include/tq.h.
ENTRY_POINTS = ("tq_packed_bytes", "tq_build_lut", "tq_quantize_pack",
                "tq_unpack", "tq_linear", "tq_status_string",
                "tq_encode_b", "tq_testing_linear_wait_fault",
                "tq_testing_force_linear_path", "tq_testing_tc_self_check",
                "tq_testing_tc_trace", "tq_linear_experts", "tq_pack7",
                "tq_build_lut7", "tq_testing_tc_split")


class TqError(RuntimeError):
    def __init__(self, status, what=""):
        msg = _lib.tq_status_string(status).decode() if _lib else str(status)
        super().__init__(f"{what}: {msg}" if what else msg)
        self.status = status


class tq_weights(C.Structure):
    _fields_ = [("format", C.c_int32), ("group", C.c_int32),
                ("planes", C.c_int32), ("rows_per_scale", C.c_int32),
                ("n_rows", C.c_int64), ("k_cols", C.c_int64),
                ("codes", C.c_void_p), ("scales", C.c_void_p),
                ("lut", C.c_void_p), ("codes_plane_stride", C.c_int64),
                ("scales_plane_stride", C.c_int64),
                ("lut_rows", C.c_int64)]


class tq_experts(C.Structure):
    _fields_ = [("n_experts", C.c_int32), ("n_hot", C.c_int32),
                ("group", C.c_int32), ("reserved", C.c_int32),
                ("n_rows", C.c_int64), ("k_cols", C.c_int64),
                ("codes", C.c_void_p), ("scales", C.c_void_p),
                ("codes2", C.c_void_p), ("scales2", C.c_void_p)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m packed_weight_matmul_b200.build`")
    L = C.CDLL(LIB_PATH)
    i32, i64, P = C.c_int32, C.c_int64, C.c_void_p
    L.tq_packed_bytes.restype = C.c_size_t
    L.tq_packed_bytes.argtypes = [i32, i64, i64, i32, i32]
    L.tq_build_lut.restype = C.c_int
    L.tq_build_lut.argtypes = [C.c_float, P, P]
    L.tq_quantize_pack.restype = C.c_int
    L.tq_quantize_pack.argtypes = [P, i64, i64, i32, i32, P, P, P, P]
    L.tq_unpack.restype = C.c_int
    L.tq_unpack.argtypes = [C.POINTER(tq_weights), P, P, P]
    L.tq_linear.restype = C.c_int
    L.tq_linear.argtypes = [C.POINTER(tq_weights), P, i64, i64, P, i64, P]
    L.tq_encode_b.restype = C.c_int
    L.tq_encode_b.argtypes = [P, i64, i64, P, C.c_float, i32, P, P, P, P, P]
    L.tq_status_string.restype = C.c_char_p
    L.tq_status_string.argtypes = [C.c_int]
    L.tq_testing_linear_wait_fault.restype = C.c_int
    L.tq_testing_linear_wait_fault.argtypes = [i32, C.c_uint64]
    L.tq_testing_force_linear_path.restype = C.c_int
    L.tq_testing_force_linear_path.argtypes = [i32]
    L.tq_testing_tc_split.restype = C.c_int
    L.tq_testing_tc_split.argtypes = [i32, i32]
    L.tq_testing_tc_self_check.restype = C.c_int
    L.tq_testing_tc_self_check.argtypes = [i32, P, i32]
    L.tq_testing_tc_trace.restype = C.c_int
    L.tq_testing_tc_trace.argtypes = [P]
    L.tq_pack7.restype = C.c_int
    L.tq_pack7.argtypes = [P, i64, i64, P, P, P, P, P]
    L.tq_build_lut7.restype = C.c_int
    L.tq_build_lut7.argtypes = [P, P, P]
    L.tq_linear_experts.restype = C.c_int
    L.tq_linear_experts.argtypes = [C.POINTER(tq_experts), P, i64, P, i64, P,
                                    i64, P, P]
    return L


_lib = None
_lib = _load()


def lib():
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return stream


def _check(status, what):
    if status != TQ_OK:
        raise TqError(status, what)


# ---- host entry points --------------------------------------------------------

def tq_packed_bytes(fmt: int, n: int, k: int, group: int = 64,
                    planes: int = 1) -> int:
    return _lib.tq_packed_bytes(fmt, n, k, group, planes)


def tq_build_lut(alpha: float, ladder) -> np.ndarray:
    lad = np.ascontiguousarray(np.asarray(ladder, np.float32))
    assert lad.shape == (5,)
    out = np.zeros(256, np.float32)
    _check(_lib.tq_build_lut(C.c_float(alpha),
                             lad.ctypes.data_as(C.c_void_p),
                             out.ctypes.data_as(C.c_void_p)), "tq_build_lut")
    return out


def tq_build_lut7(lut, used) -> np.ndarray:
    """Host: LUT7[i] = lut[used[i]] for a 7-bit layer (128 entries)."""
    lut = np.ascontiguousarray(np.asarray(lut, np.float32))
    used = np.ascontiguousarray(np.asarray(used, np.uint8))
    assert lut.shape == (256,) and used.shape == (128,)
    out = np.zeros(128, np.float32)
    _check(_lib.tq_build_lut7(lut.ctypes.data_as(C.c_void_p),
                              used.ctypes.data_as(C.c_void_p),
                              out.ctypes.data_as(C.c_void_p)), "tq_build_lut7")
    return out


def tq_pack7(codes, used_out, n_used_out, packed_out, dev_status=None,
             stream=None, check=True):
    n, k = codes.shape
    st = _lib.tq_pack7(_ptr(codes), n, k, _ptr(used_out), _ptr(n_used_out),
                       _ptr(packed_out), _ptr(dev_status), _stream(stream))
    if check:
        _check(st, "tq_pack7")
    return st


def tq_linear_experts(w: "Experts", ids, x, y, n_tokens=None, ldx=None,
                      ldy=None, status=None, stream=None, check=True):
    if n_tokens is None:
        n_tokens = ids.shape[0]
    if ldx is None:
        ldx = x.stride(0)
    if ldy is None:
        ldy = y.stride(0)
    st = _lib.tq_linear_experts(C.byref(w.desc), _ptr(ids), n_tokens, _ptr(x),
                                ldx, _ptr(y), ldy, _ptr(status),
                                _stream(stream))
    if check:
        _check(st, "tq_linear_experts")
    return st


def tq_testing_linear_wait_fault(withhold_first_arrive: bool,
                                 wait_limit_ns: int = 0) -> None:
    """Test hook (include/tq_testing.h): make the tensor-core tq_linear
    kernels time out on purpose, with a short wait limit."""
    _check(_lib.tq_testing_linear_wait_fault(int(bool(withhold_first_arrive)),
                                             int(wait_limit_ns)),
           "tq_testing_linear_wait_fault")


def tq_testing_force_linear_path(path: int) -> None:
    """Test hook (include/tq_testing.h): 0 automatic dispatch, 1 CUDA-core
    kernels, 2 tensor-core kernel, 3 tensor-core kernel with the Format B
    code book always split into bf16 hi + lo operands."""
    _check(_lib.tq_testing_force_linear_path(int(path)),
           "tq_testing_force_linear_path")


def tq_testing_tc_split(ks: int, max_clusters: int = 0) -> None:
    """Test hook (include/tq_testing.h): split of K over clusters of ks
    CTAs (0 = planner's choice) and a cap on the number of clusters."""
    _check(_lib.tq_testing_tc_split(int(ks), int(max_clusters)),
           "tq_testing_tc_split")


def tq_testing_tc_self_check(enable: bool, read: bool = False,
                             reset: bool = False):
    """Test hook (include/tq_testing.h): select the self-checking
    tensor-core kernel; with read=True return its record (4 integers)."""
    rec = np.zeros(4, np.uint64)
    _check(_lib.tq_testing_tc_self_check(
        int(bool(enable)), rec.ctypes.data_as(C.c_void_p) if read else None,
        int(bool(reset))), "tq_testing_tc_self_check")
    return [int(v) for v in rec] if read else None


def tq_testing_tc_trace(buffer) -> None:
    """Test hook (include/tq_testing.h): progress trace of the self-checking
    tensor-core kernel into a pinned host tensor (int64), or None."""
    _check(_lib.tq_testing_tc_trace(None if buffer is None else
                                    buffer.data_ptr()),
           "tq_testing_tc_trace")


def tq_status_string(status: int) -> str:
    return _lib.tq_status_string(status).decode()


# ---- weight descriptors --------------------------------------------------------

class Weights:
    """A tq_weights descriptor that keeps its tensors alive."""

    def __init__(self, desc: tq_weights, keep):
        self.desc = desc
        self._keep = keep

    @property
    def n(self):
        return self.desc.n_rows

    @property
    def k(self):
        return self.desc.k_cols


def weights_a(codes, scales, n, k, group=64, planes=1, codes_plane_stride=0,
              scales_plane_stride=0) -> Weights:
    d = tq_weights(format=TQ_FMT_A, group=group, planes=planes,
                   rows_per_scale=0, n_rows=n, k_cols=k, codes=_ptr(codes),
                   scales=_ptr(scales), lut=None,
                   codes_plane_stride=codes_plane_stride,
                   scales_plane_stride=scales_plane_stride)
    return Weights(d, (codes, scales))


class Experts:
    """A tq_experts descriptor that keeps its tensors alive."""

    def __init__(self, desc: tq_experts, keep):
        self.desc = desc
        self._keep = keep

    @property
    def n(self):
        return self.desc.n_rows

    @property
    def k(self):
        return self.desc.k_cols


def experts_a(codes, scales, n_experts, n, k, n_hot=0, codes2=None,
              scales2=None, group=64) -> Experts:
    """Plane 1 of every expert in codes / scales ([E][N][K/G][13] bytes,
    [E][N][K/G] fp16); plane 2 of experts 0 .. n_hot - 1 in codes2 /
    scales2 (same layout)."""
    d = tq_experts(n_experts=n_experts, n_hot=n_hot, group=group, reserved=0,
                   n_rows=n, k_cols=k, codes=_ptr(codes), scales=_ptr(scales),
                   codes2=_ptr(codes2), scales2=_ptr(scales2))
    return Experts(d, (codes, scales, codes2, scales2))


def weights_b7(packed, lut7, n, k, rho=None, rows_per_scale=0) -> Weights:
    """7-bit layer: packed indices [n][14 k / 16] and LUT7 [128]."""
    d = tq_weights(format=TQ_FMT_B7, group=0, planes=1,
                   rows_per_scale=rows_per_scale if rho is not None else 0,
                   n_rows=n, k_cols=k, codes=_ptr(packed), scales=_ptr(rho),
                   lut=_ptr(lut7), codes_plane_stride=0, scales_plane_stride=0,
                   lut_rows=0)
    return Weights(d, (packed, lut7, rho))


def weights_b(codes, lut, rho=None, rows_per_scale=0, n=None, k=None,
              lut_rows=0) -> Weights:
    """lut: one code book (256 fp32), or with lut_rows > 0 one per block of
    lut_rows rows ([ceil(n / lut_rows)][256], the adaptive alphabet)."""
    if n is None:
        n, k = codes.shape
    d = tq_weights(format=TQ_FMT_B, group=0, planes=1,
                   rows_per_scale=rows_per_scale if rho is not None else 0,
                   n_rows=n, k_cols=k, codes=_ptr(codes), scales=_ptr(rho),
                   lut=_ptr(lut), codes_plane_stride=0, scales_plane_stride=0,
                   lut_rows=lut_rows)
    return Weights(d, (codes, lut, rho))


# ---- GPU entry points -----------------------------------------------------------

def tq_quantize_pack(W, group, planes, codes_out, scales_out, dev_status=None,
                     stream=None, n=None, k=None, check=True):
    if n is None:
        n, k = W.shape
    st = _lib.tq_quantize_pack(_ptr(W), n, k, group, planes, _ptr(codes_out),
                               _ptr(scales_out), _ptr(dev_status),
                               _stream(stream))
    if check:
        _check(st, "tq_quantize_pack")
    return st


def tq_encode_b(W, ladder, zeta, rows_per_scale, codes_out, rho_out,
                alpha_out, dev_status=None, stream=None, n=None, k=None,
                check=True):
    """Format B encoder: W bf16 [n][k] (device) -> codes_out uint8 [n][k],
    rho_out fp16 [ceil(n / rows_per_scale)] (None when rows_per_scale = 0),
    alpha_out fp32 [1] (all device). `ladder` is 5 host floats."""
    if n is None:
        n, k = W.shape
    lad = np.ascontiguousarray(np.asarray(ladder, np.float32))
    assert lad.shape == (5,)
    st = _lib.tq_encode_b(_ptr(W), n, k, lad.ctypes.data_as(C.c_void_p),
                          C.c_float(zeta), rows_per_scale, _ptr(codes_out),
                          _ptr(rho_out), _ptr(alpha_out), _ptr(dev_status),
                          _stream(stream))
    if check:
        _check(st, "tq_encode_b")
    return st


def tq_unpack(w: Weights, out, dev_status=None, stream=None, check=True):
    st = _lib.tq_unpack(C.byref(w.desc), _ptr(out), _ptr(dev_status),
                        _stream(stream))
    if check:
        _check(st, "tq_unpack")
    return st


def tq_linear(w: Weights, x, y, batch=None, ldx=None, ldy=None, stream=None,
              check=True):
    if batch is None:
        batch = x.shape[0]
    if ldx is None:
        ldx = x.stride(0) if x.dim() == 2 else w.k
    if ldy is None:
        ldy = y.stride(0) if y.dim() == 2 else w.n
    st = _lib.tq_linear(C.byref(w.desc), _ptr(x), batch, ldx, _ptr(y), ldy,
                        _stream(stream))
    if check:
        _check(st, "tq_linear")
    return st

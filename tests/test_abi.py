"""The C ABI library loads, exports every declared entry point, and its host
functions and argument checks behave as include/tq.h states. No GPU needed:
nothing here launches a kernel (every call either runs on the host or is
rejected by validation before any launch)."""
import ctypes as C
import os
import re

import numpy as np
import pytest

from packed_weight_matmul_b200 import inputs as I

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def tq():
    from packed_weight_matmul_b200 import build
    if build.needs_build():
        build.build()
    from packed_weight_matmul_b200 import tq as _tq
    return _tq


def declared_entry_points():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        if not h.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", h)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(tq_\w+)\s*\(", text))
    return names


def test_exports_every_declared_symbol(tq):
    names = declared_entry_points()
    assert names, "no entry points found in include/"
    assert names == set(tq.ENTRY_POINTS)
    L = C.CDLL(tq.LIB_PATH)
    for name in names:
        assert hasattr(L, name), f"{name} not exported"


def test_packed_bytes_matches_oracle(tq, oref):
    for fmt in (tq.TQ_FMT_A, tq.TQ_FMT_B):
        for n, k, G, planes in [(512, 1024, 64, 1), (28672, 8192, 64, 2),
                                (3, 256, 128, 1), (1, 64, 64, 2),
                                (7, 100, 64, 1), (0, 64, 64, 1)]:
            assert tq.tq_packed_bytes(fmt, n, k, G, planes) == \
                oref.packed_bytes(fmt, n, k, G, planes)


def test_build_lut_bit_exact(tq, oref):
    ladders = [I.ladder_pow3().numpy(),
               np.array([1.0, 0.33, 0.115, 0.037, 0.012], np.float32)]
    rng = np.random.default_rng(0)
    ladders += [rng.standard_normal(5).astype(np.float32) for _ in range(20)]
    for lad in ladders:
        for alpha in (0.02, 1.0, -3.5, 1e-30, 7e30):
            got = tq.tq_build_lut(alpha, lad)
            ref = oref.build_lut(alpha, lad)
            assert np.array_equal(got[:243].view(np.uint32),
                                  ref[:243].view(np.uint32))
            assert np.all(np.isnan(got[243:]))


def test_status_strings(tq):
    for s in range(10):
        assert tq.tq_status_string(s).startswith("TQ_")
    assert "unknown" in tq.tq_status_string(99)


def _wa(tq, **kw):
    d = dict(format=tq.TQ_FMT_A, group=64, planes=1, rows_per_scale=0,
             n_rows=4, k_cols=128, codes=0x10000, scales=0x20000, lut=None,
             codes_plane_stride=0, scales_plane_stride=0)
    d.update(kw)
    return tq.Weights(tq.tq_weights(**d), None)


def _wb(tq, **kw):
    d = dict(format=tq.TQ_FMT_B, group=0, planes=1, rows_per_scale=0,
             n_rows=4, k_cols=128, codes=0x10000, scales=None, lut=0x30000,
             codes_plane_stride=0, scales_plane_stride=0)
    d.update(kw)
    return tq.Weights(tq.tq_weights(**d), None)


def _linear(tq, w, x=0x40000, y=0x50000, batch=1, ldx=None, ldy=None):
    ldx = w.k if ldx is None else ldx
    ldy = w.n if ldy is None else ldy
    return tq.lib().tq_linear(C.byref(w.desc), x, batch, ldx, y, ldy, None)


def test_validation_before_launch(tq):
    # Fake (never dereferenced) device addresses: each call must be rejected
    # on the host, so no GPU is touched.
    E = tq
    assert _linear(tq, _wa(tq, codes=None)) == E.TQ_ERR_INVALID_ARG
    assert _linear(tq, _wa(tq, scales=None)) == E.TQ_ERR_INVALID_ARG
    assert _linear(tq, _wa(tq, planes=3)) == E.TQ_ERR_INVALID_ARG
    assert _linear(tq, _wa(tq, group=32)) == E.TQ_ERR_UNSUPPORTED
    assert _linear(tq, _wa(tq, k_cols=100)) == E.TQ_ERR_SHAPE
    assert _linear(tq, _wa(tq, codes=0x10008)) == E.TQ_ERR_ALIGNMENT
    assert _linear(tq, _wa(tq, scales=0x20002)) == E.TQ_ERR_ALIGNMENT
    assert _linear(tq, _wa(tq, scales=0x20008)) == E.TQ_ERR_ALIGNMENT  # A: 16 B
    assert _linear(tq, _wa(tq, format=7)) == E.TQ_ERR_INVALID_ARG
    assert _linear(tq, _wa(tq), x=None) == E.TQ_ERR_INVALID_ARG
    assert _linear(tq, _wa(tq), batch=0) == E.TQ_ERR_INVALID_ARG
    assert _linear(tq, _wa(tq), ldx=64) == E.TQ_ERR_SHAPE
    assert _linear(tq, _wa(tq), ldy=2) == E.TQ_ERR_SHAPE
    assert _linear(tq, _wa(tq), x=0x40002) == E.TQ_ERR_ALIGNMENT
    assert _linear(tq, _wa(tq), ldx=132) == E.TQ_ERR_ALIGNMENT
    assert _linear(tq, _wa(tq), y=0x50002) == E.TQ_ERR_ALIGNMENT
    assert _linear(tq, _wa(tq, planes=2, codes_plane_stride=10)) == \
        E.TQ_ERR_SHAPE
    assert _linear(tq, _wb(tq, lut=None)) == E.TQ_ERR_INVALID_ARG
    assert _linear(tq, _wb(tq, planes=2)) == E.TQ_ERR_INVALID_ARG
    assert _linear(tq, _wb(tq, rows_per_scale=1)) == E.TQ_ERR_INVALID_ARG
    assert _linear(tq, _wb(tq, rows_per_scale=-1)) == E.TQ_ERR_INVALID_ARG
    assert _linear(tq, _wb(tq, k_cols=120)) == E.TQ_ERR_SHAPE
    assert _linear(tq, _wb(tq, lut=0x30004)) == E.TQ_ERR_ALIGNMENT
    assert _linear(tq, _wb(tq, codes=0x10001)) == E.TQ_ERR_ALIGNMENT
    # zero rows: nothing to do, no launch
    assert _linear(tq, _wb(tq, n_rows=0), ldy=0) == E.TQ_OK
    L = tq.lib()
    assert L.tq_quantize_pack(None, 4, 128, 64, 1, 0x10000, 0x20000, None,
                              None) == E.TQ_ERR_INVALID_ARG
    assert L.tq_quantize_pack(0x10000, 4, 128, 48, 1, 0x10000, 0x20000, None,
                              None) == E.TQ_ERR_UNSUPPORTED
    assert L.tq_quantize_pack(0x10000, 4, 96, 64, 1, 0x10000, 0x20000, None,
                              None) == E.TQ_ERR_SHAPE
    assert L.tq_quantize_pack(0x10000, 4, 128, 64, 0, 0x10000, 0x20000, None,
                              None) == E.TQ_ERR_INVALID_ARG
    assert L.tq_quantize_pack(0x10002, 4, 128, 64, 1, 0x10000, 0x20000, None,
                              None) == E.TQ_ERR_ALIGNMENT
    assert L.tq_quantize_pack(0x10000, 0, 128, 64, 1, 0x10000, 0x20000, None,
                              None) == E.TQ_OK
    assert L.tq_unpack(C.byref(_wa(tq).desc), None, None, None) == \
        E.TQ_ERR_INVALID_ARG
    assert L.tq_unpack(C.byref(_wa(tq).desc), 0x60008, None, None) == \
        E.TQ_ERR_ALIGNMENT


def _we(tq, **kw):
    f = dict(n_experts=4, n_hot=1, group=64, reserved=0, n_rows=8, k_cols=128,
             codes=0x10000, scales=0x20000, codes2=0x30000, scales2=0x40000)
    f.update(kw)
    return tq.tq_experts(**f)


def _experts(tq, w, ids=0x50000, tokens=3, x=0x60000, ldx=128, y=0x70000,
             ldy=8, status=None):
    return tq.lib().tq_linear_experts(C.byref(w), ids, tokens, x, ldx, y, ldy,
                                      status, None)


def test_experts_validation_before_launch(tq):
    """tq_linear_experts rejects every bad argument on the host (fake,
    never dereferenced addresses: no GPU is touched)."""
    E = tq
    assert tq.lib().tq_linear_experts(None, 0x50000, 1, 0x60000, 128, 0x70000,
                                      8, None, None) == E.TQ_ERR_INVALID_ARG
    assert _experts(tq, _we(tq, n_experts=0)) == E.TQ_ERR_INVALID_ARG
    assert _experts(tq, _we(tq, n_hot=5)) == E.TQ_ERR_INVALID_ARG
    assert _experts(tq, _we(tq, n_hot=-1)) == E.TQ_ERR_INVALID_ARG
    assert _experts(tq, _we(tq, reserved=1)) == E.TQ_ERR_INVALID_ARG
    assert _experts(tq, _we(tq, group=128)) == E.TQ_ERR_UNSUPPORTED
    assert _experts(tq, _we(tq, k_cols=96)) == E.TQ_ERR_SHAPE
    assert _experts(tq, _we(tq, n_rows=0)) == E.TQ_ERR_SHAPE
    assert _experts(tq, _we(tq, codes=None)) == E.TQ_ERR_INVALID_ARG
    assert _experts(tq, _we(tq, codes2=None)) == E.TQ_ERR_INVALID_ARG
    assert _experts(tq, _we(tq, codes2=None, scales2=None, n_hot=0), ids=None,
                    tokens=0) == E.TQ_OK
    assert _experts(tq, _we(tq, codes=0x10008)) == E.TQ_ERR_ALIGNMENT
    assert _experts(tq, _we(tq, scales2=0x40004)) == E.TQ_ERR_ALIGNMENT
    assert _experts(tq, _we(tq), tokens=-1) == E.TQ_ERR_INVALID_ARG
    assert _experts(tq, _we(tq), tokens=70000) == E.TQ_ERR_UNSUPPORTED
    assert _experts(tq, _we(tq), ids=None) == E.TQ_ERR_INVALID_ARG
    assert _experts(tq, _we(tq), ldx=64) == E.TQ_ERR_SHAPE
    assert _experts(tq, _we(tq), ldy=4) == E.TQ_ERR_SHAPE
    assert _experts(tq, _we(tq), ids=0x50002) == E.TQ_ERR_ALIGNMENT
    assert _experts(tq, _we(tq), x=0x60002) == E.TQ_ERR_ALIGNMENT
    assert _experts(tq, _we(tq), ldx=132) == E.TQ_ERR_ALIGNMENT
    assert _experts(tq, _we(tq), status=0x80002) == E.TQ_ERR_ALIGNMENT


def test_lut_rows_validation(tq):
    """lut_rows: negative is rejected, and Format A must leave it 0."""
    E = tq
    assert _linear(tq, _wb(tq, lut_rows=-1)) == E.TQ_ERR_INVALID_ARG
    assert _linear(tq, _wa(tq, lut_rows=32)) == E.TQ_ERR_INVALID_ARG
    # a zero-row call with per-block books is valid and launches nothing
    assert _linear(tq, _wb(tq, n_rows=0, lut_rows=32), ldy=0) == E.TQ_OK


def test_pack7_and_b7_validation(tq):
    """tq_pack7 and 7-bit weights: bad arguments are rejected on the host
    (fake addresses, no GPU touched); the host book builder gathers."""
    E, L = tq, tq.lib()
    assert L.tq_pack7(None, 4, 32, 0x20000, 0x30000, 0x40000, None,
                      None) == E.TQ_ERR_INVALID_ARG
    assert L.tq_pack7(0x10000, 4, 24, 0x20000, 0x30000, 0x40000, None,
                      None) == E.TQ_ERR_SHAPE
    assert L.tq_pack7(0x10008, 4, 32, 0x20000, 0x30000, 0x40000, None,
                      None) == E.TQ_ERR_ALIGNMENT
    assert L.tq_pack7(0x10000, 4, 32, 0x20004, 0x30000, 0x40000, None,
                      None) == E.TQ_ERR_ALIGNMENT
    assert L.tq_pack7(0x10000, 4, 32, 0x20000, 0x30000, 0x40001, None,
                      None) == E.TQ_ERR_ALIGNMENT
    b7 = dict(format=tq.TQ_FMT_B7)
    assert _linear(tq, _wb(tq, **b7, lut_rows=32)) == E.TQ_ERR_INVALID_ARG
    assert _linear(tq, _wb(tq, **b7, k_cols=24)) == E.TQ_ERR_SHAPE
    assert _linear(tq, _wb(tq, **b7, codes=0x10001)) == E.TQ_ERR_ALIGNMENT
    assert _linear(tq, _wb(tq, **b7, lut=0x30008)) == E.TQ_ERR_ALIGNMENT
    assert tq.tq_packed_bytes(tq.TQ_FMT_B7, 3, 32) == 3 * 28 + 512
    lut = np.arange(256, dtype=np.float32)
    used = np.arange(128, dtype=np.uint8)[::-1].copy()
    assert np.array_equal(tq.tq_build_lut7(lut, used), lut[used])


def test_tc_split_hook_range(tq):
    # host-only: the hook stores the plan override; out-of-range values are
    # rejected and (0, 0) restores the planner's choice
    with pytest.raises(tq.TqError):
        tq.tq_testing_tc_split(9, 0)
    with pytest.raises(tq.TqError):
        tq.tq_testing_tc_split(-1, 0)
    with pytest.raises(tq.TqError):
        tq.tq_testing_tc_split(2, -1)
    tq.tq_testing_tc_split(3, 2)
    tq.tq_testing_tc_split(0, 0)

"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point the header declares, and rejects bad arguments before any
CUDA call; the host tilt helper agrees with the oracle."""
import ctypes
import os
import re

import numpy as np
import pytest

from mixed_precision_vit_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from mixed_precision_vit_b200 import build
    build.build()
    return L.load()


def _declared():
    src = open(os.path.join(ROOT, "include", "sc.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sc_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol(lib):
    declared = _declared()
    assert declared == sorted(L.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), name
    assert "sm_100a" in L.sc_version()


def test_kband_tilt_matches_oracle(lib, orc):
    from mixed_precision_vit_b200.sc import kband_tilt
    for ladder, nb, t, ceil in [([64, 96, 128, 192, 256], 16, 0.25, 256),
                                ([64, 96, 128, 192, 256], 16, 0.0, 256),
                                ([8, 16, 24], 5, -0.4, 32), ([10, 30], 7, 0.33, 64),
                                ([64, 96, 128, 192, 256], 3, 0.9, 256)]:
        assert np.array_equal(kband_tilt(ladder, nb, t, ceil), orc.kband_tilt(ladder, nb, t, ceil))


def test_kband_tilt_rejects(lib):
    from mixed_precision_vit_b200.sc import kband_tilt
    with pytest.raises(L.ScError) as e:
        kband_tilt([64, 300], 4, 0.1, 256)
    assert e.value.code == L.SC_ERR_TABLE
    with pytest.raises(L.ScError) as e:
        kband_tilt([64], 4, 1.0, 256)
    assert e.value.code == L.SC_ERR_ARG


def _status(fn, *args):
    return fn(*args)


def test_host_validation_before_any_cuda_call(lib):
    vp = ctypes.c_void_p
    lad = np.array([64, 96, 128], np.int32)
    bad_lad = np.array([96, 64], np.int32)
    h = vp()
    assert lib.sc_build_table(8, lad.ctypes.data, 3, None, 0, 0, 0, None) == L.SC_ERR_ARG
    assert lib.sc_build_table(9, lad.ctypes.data, 3, None, 0, 0, 0, ctypes.byref(h)) == L.SC_ERR_ARG
    assert lib.sc_build_table(8, bad_lad.ctypes.data, 2, None, 0, 0, 0, ctypes.byref(h)) == L.SC_ERR_TABLE
    big = np.array([64, 512], np.int32)
    assert lib.sc_build_table(8, big.ctypes.data, 2, None, 0, 0, 0, ctypes.byref(h)) == L.SC_ERR_TABLE
    # band table: identity broken, ceiling exceeded, width mismatch
    bl = np.full((4, 3), 64, np.int32)
    bl[:, 1] = 96
    bl[:, 2] = 128
    bl[0, 0] = 65
    assert lib.sc_build_table(8, lad.ctypes.data, 3, bl.ctypes.data, 4, 16, 64, ctypes.byref(h)) == L.SC_ERR_TABLE
    bl[0, 0] = 64
    bl[0, 2] = 300
    assert lib.sc_build_table(8, lad.ctypes.data, 3, bl.ctypes.data, 4, 16, 64, ctypes.byref(h)) == L.SC_ERR_TABLE
    bl[0, 2] = 128
    assert lib.sc_build_table(8, lad.ctypes.data, 3, bl.ctypes.data, 4, 16, 65, ctypes.byref(h)) == L.SC_ERR_TABLE
    assert "width" in L.sc_last_error() or "contraction_d" in L.sc_last_error()
    # quantise / assign / matmul argument checks
    assert lib.sc_quantize(None, 4, 4, 4, 1, 16, 2, 8, 0, None, None, None, None, None) == L.SC_ERR_ARG
    assert lib.sc_quantize(None, 4, 4, 3, 1, 16, 0, 8, 0, None, None, None, None, None) == L.SC_ERR_ARG
    tau_bad = np.array([0.2, 0.8], np.float32)
    assert lib.sc_assign_rows(None, 4, 1, tau_bad.ctypes.data, 3, None, None, None, None) == L.SC_ERR_ARG
    assert "non-increasing" in L.sc_last_error()
    assert lib.sc_matmul(None, None, None, None, None, None, None, None, None, None, None, None, None) == L.SC_ERR_ARG
    d = L.ScMatmulDesc(4, 4, 0, 1, 0, 0, 0.0)
    assert lib.sc_matmul(ctypes.byref(d), None, None, None, None, None, None, None, None, None, None, None, None) == L.SC_ERR_ARG
    # chunked quantisation: chunk must divide the row
    assert lib.sc_quantize_chunked(None, 4, 10, 10, 1, 40, 4, 8, 0, None, None, None, None, None) == L.SC_ERR_ARG
    assert "divide" in L.sc_last_error()
    assert lib.sc_quantize_chunked(None, 4, 8, 8, 1, 32, 0, 8, 0, None, None, None, None, None) == L.SC_ERR_ARG
    # fraction-based MP: fractions must be >= 0 and sum to 1; sets divide the batch
    fr = np.array([0.5, 0.4], np.float64)
    assert lib.sc_assign_fraction(None, 4, 2, 0, fr.ctypes.data, 2, None, None, None, None) == L.SC_ERR_ARG
    assert "sum" in L.sc_last_error()
    fr = np.array([1.5, -0.5], np.float64)
    assert lib.sc_assign_fraction(None, 4, 2, 0, fr.ctypes.data, 2, None, None, None, None) == L.SC_ERR_ARG
    fr = np.array([0.5, 0.5], np.float64)
    assert lib.sc_assign_fraction(None, 4, 4, 3, fr.ctypes.data, 2, None, None, None, None) == L.SC_ERR_ARG
    # seed-bank variants: shift below 2^sc_prec, antithetic 0 or 1
    assert lib.sc_build_table_variant(8, lad.ctypes.data, 3, None, 0, 0, 0, 256, 0, ctypes.byref(h)) == L.SC_ERR_ARG
    assert lib.sc_build_table_variant(8, lad.ctypes.data, 3, None, 0, 0, 0, 3, 2, ctypes.byref(h)) == L.SC_ERR_ARG
    # descriptor enums: scales, mode, workspace size
    for bad in (dict(scales=2), dict(mode=2), dict(workspace_bytes=-1),
                dict(workspace=8, workspace_bytes=1 << 20)):
        d = L.ScMatmulDesc(4, 4, 8, 1, 0, 0, 0.0)
        for k, v in bad.items():
            setattr(d, k, v)
        t = vp(1)  # never dereferenced: the descriptor fails first
        assert lib.sc_matmul(ctypes.byref(d), None, None, None, None, None, None, None, t, None, None, None, None) == L.SC_ERR_ARG, bad


def test_no_cpu_fallback_when_library_missing(monkeypatch, tmp_path):
    monkeypatch.setattr(L, "_lib", None)
    monkeypatch.setattr(L, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        L.load()


def test_table_construction_self_check_every_length():
    """sc_build_table checks, before any device call, that every chunk table
    of the tensor-core B operand reproduces the folded rows P_L[b, .] of every
    level; a failure returns SC_ERR_TABLE.  Without a GPU the call then stops
    at the device (SC_ERR_CUDA); with one it succeeds."""
    import ctypes

    import numpy as np

    from mixed_precision_vit_b200 import _lib as L
    lib = L.load()
    for Lv in range(1, 257):
        for shift, anti in ((0, 0), (37, 1), (200, 0)):
            lad = np.array([Lv], np.int32)
            out = ctypes.c_void_p()
            rc = lib.sc_build_table_variant(8, lad.ctypes.data, 1, None, 0, 0, 0, shift, anti,
                                            ctypes.byref(out))
            assert rc in (L.SC_OK, L.SC_ERR_CUDA), (Lv, shift, anti, lib.sc_last_error())
            if rc == L.SC_OK:
                lib.sc_table_destroy(out)

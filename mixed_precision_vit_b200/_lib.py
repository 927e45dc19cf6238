"""ctypes binding of the C ABI declared in ``include/sc.h``.

Argument marshalling only: every step of the SC matmul runs in the CUDA
library ``libsc_b200.so``.  If the library is missing this module raises on
import of any entry point; there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsc_b200.so")

SC_OK, SC_ERR_ARG, SC_ERR_UNSUPPORTED, SC_ERR_TABLE, SC_ERR_NONFINITE, SC_ERR_CUDA = 0, 1, 2, 3, 4, 5
SC_DEV_NONFINITE, SC_DEV_LEVEL_RANGE, SC_DEV_WAIT_LIMIT = 0x1, 0x2, 0x4
SC_STAT_AMAX, SC_STAT_ROWMAX = 0, 1
SC_OP_LINEAR, SC_OP_QK, SC_OP_AV = 0, 1, 2
SC_ENGINE_AUTO, SC_ENGINE_GATHER, SC_ENGINE_TC = 0, 1, 2
SC_SCALES_ROW, SC_SCALES_BAND = 0, 1
SC_MODE_BIPOLAR, SC_MODE_UNIPOLAR = 0, 1
SC_ORDER_NATURAL, SC_ORDER_GRAY = 0, 1
SC_MAX_PREC, SC_MAX_RUNGS, SC_MAX_BANDS = 8, 8, 64

# every symbol include/sc.h declares
EXPORTS = ("sc_last_error", "sc_version", "sc_kband_tilt", "sc_build_table", "sc_table_destroy",
           "sc_build_table_variant", "sc_build_table_seq", "sc_table_info", "sc_quantize", "sc_quantize_chunked",
           "sc_assign_rows", "sc_assign_fraction", "sc_matmul", "sc_matmul_engine", "sc_matmul_workspace_bytes",
           "sc_matmul_static_ws", "sc_matmul_launches", "sc_prepare_b", "sc_prepare_b_bytes",
           "sc_bprep_destroy", "sc_selftest_wait_limit")
SC_STATIC_WS_BYTES = 64 << 20


class ScMatmulDesc(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int64), ("N", ctypes.c_int64), ("D", ctypes.c_int64),
                ("batch", ctypes.c_int64), ("op", ctypes.c_int32), ("engine", ctypes.c_int32),
                ("q_dec", ctypes.c_double), ("scales", ctypes.c_int32),
                ("mode", ctypes.c_int32), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_int64), ("b_prep", ctypes.c_void_p)]


class ScError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[{code}] {msg}")
        self.code = code


_lib = None
_lock = threading.Lock()


def load():
    """Load ``libsc_b200.so`` (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"CUDA library not built: {LIB_PATH} (run __graft_entry__.build())")
        lib = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, f64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.sc_last_error.restype = ctypes.c_char_p
        lib.sc_last_error.argtypes = []
        lib.sc_version.restype = ctypes.c_char_p
        lib.sc_version.argtypes = []
        lib.sc_kband_tilt.argtypes = [vp, i32, i32, f64, i32, vp]
        lib.sc_build_table.argtypes = [i32, vp, i32, vp, i32, i64, i64, ctypes.POINTER(vp)]
        lib.sc_table_destroy.argtypes = [vp]
        lib.sc_build_table_variant.argtypes = [i32, vp, i32, vp, i32, i64, i64, ctypes.c_uint32, i32,
                                               ctypes.POINTER(vp)]
        lib.sc_build_table_seq.argtypes = [i32, vp, i32, vp, i32, i64, i64, i32, vp, i32,
                                           ctypes.POINTER(vp)]
        lib.sc_table_info.argtypes = [vp, vp, vp, vp, vp, vp]
        lib.sc_quantize.argtypes = [vp, i64, i64, i64, i64, i64, i32, i32, i32, vp, vp, vp, vp, vp]
        lib.sc_quantize_chunked.argtypes = [vp, i64, i64, i64, i64, i64, i64, i32, i32, vp, vp, vp,
                                            vp, vp]
        lib.sc_assign_rows.argtypes = [vp, i64, i64, vp, i32, vp, vp, vp, vp]
        lib.sc_assign_fraction.argtypes = [vp, i64, i64, i64, vp, i32, vp, vp, vp, vp]
        lib.sc_matmul.argtypes = [ctypes.POINTER(ScMatmulDesc), vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                  vp, vp, vp]
        lib.sc_matmul_engine.argtypes = [ctypes.POINTER(ScMatmulDesc), vp]
        lib.sc_matmul_static_ws.argtypes = [ctypes.POINTER(ScMatmulDesc), vp, vp, vp, vp, vp, vp, vp,
                                            vp, vp, vp, vp, vp]
        lib.sc_matmul_launches.argtypes = [ctypes.POINTER(ScMatmulDesc), vp]
        lib.sc_matmul_workspace_bytes.argtypes = [ctypes.POINTER(ScMatmulDesc), vp]
        lib.sc_matmul_workspace_bytes.restype = ctypes.c_int64
        lib.sc_prepare_b.argtypes = [ctypes.POINTER(ScMatmulDesc), vp, vp, ctypes.POINTER(vp), vp]
        lib.sc_prepare_b_bytes.argtypes = [ctypes.POINTER(ScMatmulDesc), vp]
        lib.sc_prepare_b_bytes.restype = ctypes.c_int64
        lib.sc_bprep_destroy.argtypes = [vp]
        lib.sc_selftest_wait_limit.argtypes = [vp, i64, vp]
        for name in EXPORTS:
            getattr(lib, name).restype = getattr(lib, name).restype or ctypes.c_int
        _lib = lib
        return lib


def _check(code: int):
    if code != SC_OK:
        raise ScError(code, load().sc_last_error().decode())


def _ptr(x):
    """Raw address of a torch tensor / numpy array / int / None."""
    if x is None:
        return None
    if isinstance(x, int):
        return ctypes.c_void_p(x)
    if hasattr(x, "data_ptr"):
        return ctypes.c_void_p(x.data_ptr())
    if hasattr(x, "ctypes"):
        return ctypes.c_void_p(x.ctypes.data)
    raise TypeError(type(x))


def _stream(stream):
    if stream is None:
        return None
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def sc_version() -> str:
    return load().sc_version().decode()


def sc_last_error() -> str:
    return load().sc_last_error().decode()


def sc_kband_tilt(ladder_ptr, n_rungs, n_bands, tilt, ceiling, out_ptr):
    _check(load().sc_kband_tilt(_ptr(ladder_ptr), n_rungs, n_bands, float(tilt), ceiling,
                                _ptr(out_ptr)))


def sc_build_table(sc_prec, ladder_ptr, n_rungs, band_len_ptr, n_bands, chunk_d, contraction_d):
    out = ctypes.c_void_p()
    _check(load().sc_build_table(sc_prec, _ptr(ladder_ptr), n_rungs, _ptr(band_len_ptr), n_bands,
                                 chunk_d, contraction_d, ctypes.byref(out)))
    return out.value


def sc_build_table_variant(sc_prec, ladder_ptr, n_rungs, band_len_ptr, n_bands, chunk_d,
                           contraction_d, b_shift, b_antithetic):
    out = ctypes.c_void_p()
    _check(load().sc_build_table_variant(sc_prec, _ptr(ladder_ptr), n_rungs, _ptr(band_len_ptr),
                                         n_bands, chunk_d, contraction_d, int(b_shift),
                                         int(b_antithetic), ctypes.byref(out)))
    return out.value


def sc_build_table_seq(sc_prec, ladder_ptr, n_rungs, band_len_ptr, n_bands, chunk_d,
                       contraction_d, order, pool_ptr, n_pool):
    out = ctypes.c_void_p()
    _check(load().sc_build_table_seq(sc_prec, _ptr(ladder_ptr), n_rungs, _ptr(band_len_ptr),
                                     n_bands, chunk_d, contraction_d, int(order), _ptr(pool_ptr),
                                     int(n_pool), ctypes.byref(out)))
    return out.value


def sc_table_destroy(table):
    _check(load().sc_table_destroy(ctypes.c_void_p(table) if table else None))


def sc_table_info(table):
    vals = [ctypes.c_int(), ctypes.c_int(), ctypes.c_int(), ctypes.c_int64(), ctypes.c_int64()]
    _check(load().sc_table_info(ctypes.c_void_p(table), *[ctypes.byref(v) for v in vals]))
    return tuple(v.value for v in vals)


def sc_quantize(x, rows, cols, ld, batch, batch_stride, axis, sc_prec, stat_mode, levels, scales,
                stat, dev_status, stream=None):
    _check(load().sc_quantize(_ptr(x), rows, cols, ld, batch, batch_stride, axis, sc_prec,
                              stat_mode, _ptr(levels), _ptr(scales), _ptr(stat), _ptr(dev_status),
                              _stream(stream)))


def sc_quantize_chunked(x, rows, cols, ld, batch, batch_stride, chunk, sc_prec, stat_mode, levels,
                        scales, stat, dev_status, stream=None):
    _check(load().sc_quantize_chunked(_ptr(x), rows, cols, ld, batch, batch_stride, chunk, sc_prec,
                                      stat_mode, _ptr(levels), _ptr(scales), _ptr(stat),
                                      _ptr(dev_status), _stream(stream)))


def sc_assign_rows(stat, rows, batch, tau_ptr, n_rungs, rung, perm, rung_offsets, stream=None):
    _check(load().sc_assign_rows(_ptr(stat), rows, batch, _ptr(tau_ptr), n_rungs, _ptr(rung),
                                 _ptr(perm), _ptr(rung_offsets), _stream(stream)))


def sc_assign_fraction(stat, rows, batch, set_size, fractions_ptr, n_rungs, rung, perm,
                       rung_offsets, stream=None):
    _check(load().sc_assign_fraction(_ptr(stat), rows, batch, set_size, _ptr(fractions_ptr),
                                     n_rungs, _ptr(rung), _ptr(perm), _ptr(rung_offsets),
                                     _stream(stream)))


def sc_matmul(desc: ScMatmulDesc, a_lv, a_s, b_lv, b_s, rung, perm, rung_offsets, table, out,
              counts, dev_status, stream=None):
    _check(load().sc_matmul(ctypes.byref(desc), _ptr(a_lv), _ptr(a_s), _ptr(b_lv), _ptr(b_s),
                            _ptr(rung), _ptr(perm), _ptr(rung_offsets),
                            ctypes.c_void_p(table) if table else None, _ptr(out), _ptr(counts),
                            _ptr(dev_status), _stream(stream)))


def sc_matmul_static_ws(desc: ScMatmulDesc, a_lv, a_s, b_lv, b_s, rung, perm, rung_offsets, table,
                        out, counts, dev_status, stream=None):
    _check(load().sc_matmul_static_ws(ctypes.byref(desc), _ptr(a_lv), _ptr(a_s), _ptr(b_lv),
                                      _ptr(b_s), _ptr(rung), _ptr(perm), _ptr(rung_offsets),
                                      ctypes.c_void_p(table) if table else None, _ptr(out),
                                      _ptr(counts), _ptr(dev_status), _stream(stream)))


def sc_matmul_engine(desc: ScMatmulDesc, table) -> int:
    e = load().sc_matmul_engine(ctypes.byref(desc), ctypes.c_void_p(table) if table else None)
    if e < 0:
        _check(-e)
    return e


def sc_matmul_workspace_bytes(desc: ScMatmulDesc, table) -> int:
    n = load().sc_matmul_workspace_bytes(ctypes.byref(desc), ctypes.c_void_p(table) if table else None)
    if n < 0:
        _check(int(-n))
    return int(n)


def sc_matmul_launches(desc: ScMatmulDesc, table) -> int:
    n = load().sc_matmul_launches(ctypes.byref(desc), ctypes.c_void_p(table) if table else None)
    if n < 0:
        _check(-n)
    return n


def sc_prepare_b(desc: ScMatmulDesc, b_lv, table, stream=None):
    out = ctypes.c_void_p()
    _check(load().sc_prepare_b(ctypes.byref(desc), _ptr(b_lv), ctypes.c_void_p(table) if table else None,
                               ctypes.byref(out), _stream(stream)))
    return out.value


def sc_prepare_b_bytes(desc: ScMatmulDesc, table) -> int:
    n = load().sc_prepare_b_bytes(ctypes.byref(desc), ctypes.c_void_p(table) if table else None)
    if n < 0:
        _check(int(-n))
    return int(n)


def sc_bprep_destroy(prep):
    _check(load().sc_bprep_destroy(ctypes.c_void_p(prep) if prep else None))


def sc_selftest_wait_limit(dev_status, limit_cycles, stream=None):
    _check(load().sc_selftest_wait_limit(_ptr(dev_status), int(limit_cycles), _stream(stream)))

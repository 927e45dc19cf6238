"""CPU oracle for the stochastic-computing (SC) bipolar XNOR matmul.

TEST INFRASTRUCTURE ONLY: this package is imported by the test-suite, by the
smoke check and by the CPU-baseline leg of the benchmark, never by the
product path.  It shares no code with the CUDA library; its arithmetic lives
in ``sc_oracle.c`` (plain C, OpenMP over outputs, every bitstream simulated bit
by bit) and this module only marshals numpy arrays into it.

Each function cites the passage it follows; see ``sc_oracle.c`` for the
readings taken where the pages leave a step open.

Parity status: every function here is pinned by the ``-m "not gpu"`` tests
(closed forms of the Sobol prefix counts, brute force over all level pairs,
full-period and zero invariants, the linear cost identity, hand-derived
decode examples, exhaustive apportionment for the tilt).  The exact Sobol
sequence of the pages' own kernel is not printed on the pages, so agreement
with that kernel's bit pattern is not claimed.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sc_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
_lock = threading.Lock()
_lib = None

OK, ERR_ARG, ERR_TABLE, ERR_NONFINITE = 0, 1, 3, 4


def build(force: bool = False) -> str:
    """Compile ``sc_oracle.c`` with gcc (IEEE fp32, no fast-math, OpenMP)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", "-Wall", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        i32, i64, f64, vp = ctypes.c_int, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        lib.orc_sobol_r.argtypes = [i32, vp]
        lib.orc_indicator.argtypes = [i32, vp]
        lib.orc_quantize.argtypes = [vp, i64, i64, i64, i32, i32, vp, vp]
        lib.orc_row_stat.argtypes = [vp, i64, i64, i64, i32, vp]
        lib.orc_assign_rungs.argtypes = [vp, i64, i64, vp, i32, vp]
        lib.orc_assign_fraction.argtypes = [vp, i64, i64, i64, vp, i32, vp]
        lib.orc_cbsg_count.argtypes = [i32, i32, i32, i32]
        lib.orc_cbsg_count.restype = i64
        lib.orc_cbsg_streams.argtypes = [i32, i32, i32, i32, vp, vp]
        lib.orc_cbsg_table.argtypes = [i32, i32, vp]
        lib.orc_matmul.argtypes = [i32, f64, i64, i64, i64, i64, vp, vp, vp, vp, vp, vp, i32,
                                   vp, i32, i64, i64, vp, vp, vp, vp, i32, i32, i32,
                                   ctypes.c_uint32, i32, i32, vp, i32]
        lib.orc_matmul_memo.argtypes = lib.orc_matmul.argtypes
        lib.orc_sobol_r_variant.argtypes = [i32, ctypes.c_uint32, i32, vp]
        lib.orc_sobol_r_gray.argtypes = [i32, vp]
        lib.orc_indicator_points.argtypes = [i32, vp, vp]
        lib.orc_indicator_variant.argtypes = [i32, ctypes.c_uint32, i32, vp]
        lib.orc_and_count.argtypes = [i32, i32, i32, i32, vp]
        lib.orc_and_count.restype = ctypes.c_int64
        lib.orc_quantize_chunked.argtypes = [vp, i64, i64, i64, i64, i32, vp, vp]
        lib.orc_kband_tilt.argtypes = [vp, i32, i32, f64, i32, vp]
        lib.orc_max_threads.argtypes = []
        _lib = lib
        return lib


def _p(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


class OracleError(RuntimeError):
    def __init__(self, code, what):
        super().__init__(f"oracle {what} returned {code}")
        self.code = code


def _check(code, what):
    if code != OK:
        raise OracleError(code, what)


def max_threads() -> int:
    return int(_load().orc_max_threads())


# -- Sobol-8 and the cumulative indicator table [Precision As You Need, key design 1]

def sobol_r(sc_prec: int = 8) -> np.ndarray:
    """r_l = u_l * 2^p + 1, l = 0..2^p-1, from the first-dimension direction numbers."""
    r = np.zeros(1 << sc_prec, dtype=np.int32)
    _check(_load().orc_sobol_r(sc_prec, _p(r)), "sobol_r")
    return r


def sobol_r_gray(sc_prec: int = 8) -> np.ndarray:
    """The first dimension's thresholds in Gray-code order: point l is the
    XOR of the direction numbers over the set bits of l XOR (l >> 1)."""
    r = np.zeros(1 << sc_prec, dtype=np.int32)
    _check(_load().orc_sobol_r_gray(sc_prec, _p(r)), "sobol_r_gray")
    return r


def indicator_points(u, sc_prec: int = 8) -> np.ndarray:
    """K[b, l] = 1[u_l + 1 <= b] of one sequence of integer points u (a
    permutation of [0, 2^p), else OracleError ERR_TABLE)."""
    q = 1 << sc_prec
    u = _c(u, np.int32)
    k = np.zeros((q + 1, q), dtype=np.uint8)
    _check(_load().orc_indicator_points(sc_prec, _p(u), _p(k)), "indicator_points")
    return k


def indicator(sc_prec: int = 8) -> np.ndarray:
    """K[b, l] = 1[r_l <= b], levels b = 0..2^p, positions l < 2^p."""
    q = 1 << sc_prec
    k = np.zeros((q + 1, q), dtype=np.uint8)
    _check(_load().orc_indicator(sc_prec, _p(k)), "indicator")
    return k


# -- Quantisation [scmp_vit README, "Why it works"]

def quantize(x: np.ndarray, axis: int = 0, sc_prec: int = 8, allow_nonfinite=False):
    """Symmetric quantisation of a 2-D fp32 matrix to levels x_int + 2^(p-1).

    axis 0: one scale per row, levels [rows, cols]; axis 1: one scale per
    column, levels transposed to [cols, rows].  Returns (levels, scales)."""
    x = _c(x, np.float32)
    rows, cols = x.shape
    n_vec, length = (rows, cols) if axis == 0 else (cols, rows)
    lv = np.zeros((n_vec, length), dtype=np.uint8)
    sc = np.zeros(n_vec, dtype=np.float32)
    code = _load().orc_quantize(_p(x), rows, cols, cols, axis, sc_prec, _p(lv), _p(sc))
    if not (allow_nonfinite and code == ERR_NONFINITE):
        _check(code, "quantize")
    return lv, sc


def quantize_chunked(x: np.ndarray, chunk: int, sc_prec: int = 8, allow_nonfinite=False):
    """Per-(row, chunk) symmetric quantisation of a 2-D fp32 matrix [K-band
    pull request, "Summary": bands of whole quantisation chunks].  Returns
    (levels [rows, cols], scales [rows, cols // chunk])."""
    x = _c(x, np.float32)
    rows, cols = x.shape
    lv = np.zeros((rows, cols), dtype=np.uint8)
    sc = np.zeros((rows, cols // chunk), dtype=np.float32)
    code = _load().orc_quantize_chunked(_p(x), rows, cols, cols, int(chunk), sc_prec, _p(lv), _p(sc))
    if not (allow_nonfinite and code == ERR_NONFINITE):
        _check(code, "quantize_chunked")
    return lv, sc


def quantize_batched(x: np.ndarray, axis: int = 0, sc_prec: int = 8):
    """quantize() applied to every [rows, cols] matrix of a [batch, rows, cols] array."""
    out = [quantize(m, axis, sc_prec) for m in np.asarray(x, dtype=np.float32)]
    return np.stack([o[0] for o in out]), np.stack([o[1] for o in out])


# -- Row statistic and rungs [Precision As You Need, key design 2]

STAT_AMAX, STAT_ROWMAX = 0, 1


def row_stat(x: np.ndarray, mode: int = STAT_AMAX) -> np.ndarray:
    x = _c(x, np.float32)
    rows, cols = x.shape
    st = np.zeros(rows, dtype=np.float32)
    _check(_load().orc_row_stat(_p(x), rows, cols, cols, mode, _p(st)), "row_stat")
    return st


def assign_rungs(stat: np.ndarray, tau, n_rungs: int) -> np.ndarray:
    """stat [batch, rows] (or [rows]) -> rung index per row."""
    st = _c(stat, np.float32)
    batch, rows = (1, st.shape[0]) if st.ndim == 1 else st.shape
    t = _c(np.asarray(tau if n_rungs > 1 else [0.0], dtype=np.float32), np.float32)
    rung = np.zeros(st.shape, dtype=np.int32)
    _check(_load().orc_assign_rungs(_p(st), rows, batch, _p(t), n_rungs, _p(rung)), "assign_rungs")
    return rung


def assign_fraction(stat: np.ndarray, fractions, set_size: int = 0) -> np.ndarray:
    """Fraction-based fixed MP ["scmp_vit" README, MP flags].  stat [batch, rows]
    (or [rows]); fractions[k] = fraction of units on rung k (ascending length).
    set_size 0: rows are ranked within each batch entry; set_size > 0: batch
    entries (heads) are ranked by their max statistic within sets of set_size."""
    st = _c(stat, np.float32)
    batch, rows = (1, st.shape[0]) if st.ndim == 1 else st.shape
    fr = _c(np.asarray(fractions, dtype=np.float64), np.float64)
    rung = np.zeros(st.shape, dtype=np.int32)
    _check(_load().orc_assign_fraction(_p(st), rows, batch, set_size, _p(fr), len(fr), _p(rung)),
           "assign_fraction")
    return rung


# -- C-BSG bipolar XNOR count [Precision As You Need, key design 1]

def cbsg_count(a: int, b: int, L: int, sc_prec: int = 8) -> int:
    c = int(_load().orc_cbsg_count(sc_prec, a, b, L))
    if c < 0:
        raise OracleError(ERR_ARG, "cbsg_count")
    return c


def sobol_r_variant(shift: int = 0, antithetic: bool = False, sc_prec: int = 8) -> np.ndarray:
    """Seed-bank variant of the Sobol thresholds ["scmp_vit" README, Sobol-seed
    bank]: r'_l = (u_l XOR shift) + 1, or 2^p - (u_l XOR shift) if antithetic."""
    r = np.zeros(1 << sc_prec, dtype=np.int32)
    _check(_load().orc_sobol_r_variant(sc_prec, shift, 1 if antithetic else 0, _p(r)), "sobol_r_variant")
    return r


def indicator_variant(shift: int = 0, antithetic: bool = False, sc_prec: int = 8) -> np.ndarray:
    q = 1 << sc_prec
    K = np.zeros((q + 1, q), dtype=np.uint8)
    _check(_load().orc_indicator_variant(sc_prec, shift, 1 if antithetic else 0, _p(K)),
           "indicator_variant")
    return K


def and_count(a: int, b: int, L: int, sc_prec: int = 8) -> int:
    """Signed unipolar AND count of bipolar level codes a, b at length L."""
    out = ctypes.c_int64(0)
    _check(int(_load().orc_and_count(sc_prec, a, b, L, ctypes.byref(out))), "and_count")
    return int(out.value)


def cbsg_table(L: int, sc_prec: int = 8) -> np.ndarray:
    """Bit-by-bit counts for all level pairs (a, b) in [0, 2^p]^2 at length L."""
    q = 1 << sc_prec
    t = np.zeros((q + 1, q + 1), dtype=np.int32)
    _check(_load().orc_cbsg_table(sc_prec, L, _p(t)), "cbsg_table")
    return t


def cbsg_streams(a: int, b: int, L: int, sc_prec: int = 8):
    za = np.zeros(max(L, 1), dtype=np.uint8)
    zb = np.zeros(max(L, 1), dtype=np.uint8)
    _check(_load().orc_cbsg_streams(sc_prec, a, b, L, _p(za), _p(zb)), "cbsg_streams")
    return za[:L], zb[:L]


def matmul(a_lv, a_s, b_lv, b_s, rung, ladder, *, sc_prec=8, q_dec=None,
           band_len=None, chunk_d=0, sel=None, n_threads=0, band_scales=False, unipolar=False,
           b_shift=0, b_antithetic=False, memo=False, gray=False, pool=None):
    """Bit-by-bit SC matmul with decode [Precision As You Need, key designs 1, 3;
    K-band pull request, "How the banding works"].

    a_lv [batch, M, D] uint8, a_s [batch, M], b_lv [batch, N, D] uint8,
    b_s [batch, N] (with band_scales: a_s [batch, M, n_bands] and b_s
    [batch, N, n_bands], one scale per band), rung [batch, M]; ladder
    [n_rungs]; band_len
    [n_bands, n_rungs] or None.  sel: None (all outputs) or int64 [n, 3] of
    (g, i, j).  Returns (counts [n, n_bands_eff] int32 — or [batch, M, N,
    n_bands_eff] when sel is None —, out fp32 of matching shape, xnor steps).
    unipolar: sign-magnitude AND streams with one enable-gated counter
    (counts are signed; the decode is q^2 s^A s^B sum_bands count_b / L_b).
    b_shift, b_antithetic: seed-bank variant of B's sequence (A keeps the default).
    gray: the first Sobol dimension in Gray-code order (both operands).
    pool: None, or int32 [n_pool, 2^p] integer points, one Sobol sequence per
    row; contraction index d streams both operands from row d mod n_pool.
    memo: take each (a, b, L) count from a table of the bit-by-bit counts of
    every level pair at that length (the same simulation, done once per pair)
    instead of simulating it again for every (i, j, d): identical results,
    pinned by the tests, fast enough for full-size problems."""
    a_lv = _c(a_lv, np.uint8)
    b_lv = _c(b_lv, np.uint8)
    if a_lv.ndim == 2:
        a_lv, b_lv = a_lv[None], b_lv[None]
        a_s, b_s, rung = np.asarray(a_s)[None], np.asarray(b_s)[None], np.asarray(rung)[None]
    batch, M, D = a_lv.shape
    N = b_lv.shape[1]
    a_s = _c(a_s, np.float32)
    b_s = _c(b_s, np.float32)
    rung = _c(rung, np.int32)
    lad = _c(ladder, np.int32)
    q_dec = float(1 << (sc_prec - 1)) if q_dec is None else float(q_dec)
    if band_len is not None:
        bl = _c(band_len, np.int32)
        n_bands = bl.shape[0]
    else:
        bl, n_bands = None, 0
    nb = max(n_bands, 1)
    if sel is None:
        n_sel, selp = batch * M * N, None
    else:
        sel = _c(sel, np.int64).reshape(-1, 3)
        n_sel, selp = sel.shape[0], sel
    counts = np.zeros((n_sel, nb), dtype=np.int32)
    out = np.zeros(n_sel, dtype=np.float32)
    steps = ctypes.c_int64(0)
    pl = None if pool is None else _c(pool, np.int32).reshape(-1, 1 << sc_prec)
    fn = _load().orc_matmul_memo if memo else _load().orc_matmul
    code = fn(sc_prec, q_dec, batch, M, N, D, _p(a_lv), _p(a_s), _p(b_lv), _p(b_s),
                              _p(rung), _p(lad), len(lad), _p(bl), n_bands, int(chunk_d),
                              n_sel, _p(selp), _p(counts), _p(out), ctypes.byref(steps),
                              int(n_threads), 1 if band_scales else 0, 1 if unipolar else 0,
                              int(b_shift), 1 if b_antithetic else 0, 1 if gray else 0, _p(pl),
                              0 if pl is None else pl.shape[0])
    _check(code, "matmul")
    if sel is None:
        counts = counts.reshape(batch, M, N, nb)
        out = out.reshape(batch, M, N)
    return counts, out, int(steps.value)


# -- K-band tilt [K-band pull request, "Tooling" and "Guards"]

def kband_tilt(ladder, n_bands: int, tilt: float, ceiling: int) -> np.ndarray:
    lad = _c(ladder, np.int32)
    out = np.zeros((n_bands, len(lad)), dtype=np.int32)
    _check(_load().orc_kband_tilt(_p(lad), len(lad), n_bands, float(tilt), int(ceiling), _p(out)),
           "kband_tilt")
    return out

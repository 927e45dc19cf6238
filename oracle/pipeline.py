"""The oracle applied to a whole workload: quantise both operands, row
statistic, rungs, band table, then the bit-by-bit matmul (all outputs, or a
selected subset).  TEST INFRASTRUCTURE ONLY (see the package docstring).

Steps in the pages' order: quantise ("scmp_vit" README, "Why it works"), row
statistic and thresholds ("Precision As You Need", key design 2) or fixed
fractions of rows / heads per length ("scmp_vit" README, MP flags), C-BSG
streams and XNOR counts with early termination (key designs 1 and 3), K-band
lengths and the summed decode ("feat(mp) ... K-band", "How the banding works",
"Tooling").
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import (assign_fraction, assign_rungs, kband_tilt, matmul, quantize, quantize_chunked,
               row_stat)


@dataclass
class OracleState:
    a_lv: np.ndarray      # [batch, M, D]
    a_s: np.ndarray       # [batch, M] (with band scales [batch, M, n_bands])
    stat: np.ndarray      # [batch, M]
    b_lv: np.ndarray      # [batch, N, D]
    b_s: np.ndarray       # [batch, N] (with band scales [batch, N, n_bands])
    rung: np.ndarray      # [batch, M]
    ladder: np.ndarray
    band_len: np.ndarray | None
    chunk_d: int
    band_scales: bool = False


def prepare(w) -> OracleState:
    """Everything before the count: levels, scales, statistic, rungs, bands."""
    a = w.a.numpy()
    b = w.b.numpy()
    a_lv, a_s, st, b_lv, b_s = [], [], [], [], []
    chunked = getattr(w, "band_scales", False)
    for g in range(w.batch):
        if chunked:  # one quantisation chunk per band, rows of A and of B ([N, D])
            lv, s = quantize_chunked(a[g], w.chunk_d, sc_prec=w.sc_prec)
        else:
            lv, s = quantize(a[g], axis=0, sc_prec=w.sc_prec)
        a_lv.append(lv)
        a_s.append(s)
        st.append(row_stat(a[g], w.stat_mode))
        if chunked:
            lv, s = quantize_chunked(b[g], w.chunk_d, sc_prec=w.sc_prec)
        else:
            lv, s = quantize(b[g], axis=w.b_axis, sc_prec=w.sc_prec)
        b_lv.append(lv)
        b_s.append(s)
    stat = np.stack(st)
    n_rungs = len(w.ladder)
    fractions = getattr(w, "fractions", ())
    if fractions:  # fraction-based fixed MP ("scmp_vit" README, MP flags)
        rung = assign_fraction(stat, fractions, getattr(w, "frac_set", 0))
    else:
        rung = assign_rungs(stat, np.asarray(w.tau, np.float32), n_rungs)
    band_len = None
    if w.n_bands:
        band_len = kband_tilt(np.asarray(w.ladder, np.int32), w.n_bands, w.tilt, 1 << w.sc_prec)
    return OracleState(np.stack(a_lv), np.stack(a_s), stat, np.stack(b_lv), np.stack(b_s), rung,
                       np.asarray(w.ladder, np.int32), band_len, w.chunk_d, chunked)


def run(w, st: OracleState | None = None, sel=None, n_threads=0, memo=False):
    """Counts / outputs of the whole workload (sel None) or of selected
    (g, i, j) triples.  Returns (state, counts, out, xnor_steps).  memo: the
    count of each (a, b, L) from a table of bit-by-bit counts (see
    oracle.matmul)."""
    st = prepare(w) if st is None else st
    counts, out, steps = matmul(st.a_lv, st.a_s, st.b_lv, st.b_s, st.rung, st.ladder,
                                sc_prec=w.sc_prec, band_len=st.band_len, chunk_d=st.chunk_d,
                                sel=sel, n_threads=n_threads, band_scales=st.band_scales,
                                unipolar=getattr(w, "unipolar", False),
                                b_shift=getattr(w, "b_shift", 0),
                                b_antithetic=getattr(w, "b_antithetic", False), memo=memo,
                                gray=getattr(w, "gray", False), pool=getattr(w, "pool", None))
    return st, counts, out, steps

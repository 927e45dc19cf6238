"""Torch-facing helpers over the C ABI: device buffers, tables and the full
SC matmul step (quantise A, quantise B, assign rows, count + decode).

Every operation is one call into ``libsc_b200.so``; torch provides device
memory and streams only.  On a machine without CUDA these helpers raise.
"""
from __future__ import annotations

import numpy as np
import torch

from . import _lib as L
from .workloads import Workload


def _require_cuda(t: torch.Tensor, what: str):
    if not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")


def kband_tilt(ladder, n_bands: int, tilt: float, ceiling: int) -> np.ndarray:
    lad = np.ascontiguousarray(ladder, dtype=np.int32)
    out = np.zeros((n_bands, len(lad)), dtype=np.int32)
    L.sc_kband_tilt(lad, len(lad), n_bands, tilt, ceiling, out)
    return out


class ScTable:
    """Device-resident stream tables (built once per layer).

    order: SC_ORDER_NATURAL / SC_ORDER_GRAY for the built-in Sobol sequence;
    pool: None or int32 [n_pool, 2^sc_prec] integer points, one sequence per
    row, contraction index d using row d mod n_pool (see sc_build_table_seq)."""

    def __init__(self, ladder, sc_prec: int = 8, band_len=None, chunk_d: int = 0,
                 contraction_d: int = 0, b_shift: int = 0, b_antithetic: bool = False,
                 order: int = L.SC_ORDER_NATURAL, pool=None):
        self.ladder = np.ascontiguousarray(ladder, dtype=np.int32)
        self.sc_prec = sc_prec
        self.band_len = None if band_len is None else np.ascontiguousarray(band_len, dtype=np.int32)
        n_bands = 0 if self.band_len is None else self.band_len.shape[0]
        if pool is not None or order != L.SC_ORDER_NATURAL:
            if b_shift or b_antithetic:
                raise ValueError("seed-bank variants and other sequences do not combine")
            pl = None if pool is None else np.ascontiguousarray(pool, dtype=np.int32)
            self.handle = L.sc_build_table_seq(sc_prec, self.ladder, len(self.ladder),
                                               self.band_len, n_bands, chunk_d, contraction_d,
                                               order, pl, 0 if pl is None else pl.shape[0])
        else:
            self.handle = L.sc_build_table_variant(sc_prec, self.ladder, len(self.ladder),
                                                   self.band_len, n_bands, chunk_d, contraction_d,
                                                   b_shift, 1 if b_antithetic else 0)
        self.n_bands = n_bands
        self.chunk_d = chunk_d

    _cache = {}

    @classmethod
    def for_width(cls, ladder, D: int, sc_prec: int = 8, band_len=None, chunk_d: int = 0,
                  n_pool: int = 0):
        """The table of a per-index Sobol pool for contraction width D, built
        once and shared by every caller of the same (ladder, D, sc_prec, bands,
        pool size) -- the pages' per-(D, sc_prec) pool cache: every op of one
        width (e.g. the block's per-head QK and a head-aligned compensator)
        streams from the same sequences.  The pool is the first 2^sc_prec
        points of Sobol dimensions 1..n_pool (n_pool = D by default)."""
        from .workloads import sobol_pool
        n = n_pool or D
        bl = None if band_len is None else np.ascontiguousarray(band_len, dtype=np.int32)
        key = (tuple(int(v) for v in ladder), int(D), int(sc_prec), None if bl is None else bl.tobytes(),
               int(chunk_d), int(n))
        t = cls._cache.get(key)
        if t is None or not t.handle:
            t = cls(ladder, sc_prec, bl, chunk_d, D if bl is not None else 0,
                    pool=sobol_pool(n, sc_prec))
            cls._cache[key] = t
        return t

    def info(self):
        return L.sc_table_info(self.handle)

    def close(self):
        if self.handle:
            L.sc_table_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def quantize(x: torch.Tensor, axis: int, sc_prec: int = 8, stat_mode: int = L.SC_STAT_AMAX,
             want_stat: bool = False, dev_status=None, stream=None, out=None):
    """x [batch, rows, cols] fp32 CUDA -> (levels, scales, stat)."""
    _require_cuda(x, "x")
    if x.dim() == 2:
        x = x.unsqueeze(0)
    batch, rows, cols = x.shape
    if out is None:
        nv, ln = (rows, cols) if axis == 0 else (cols, rows)
        lv = torch.empty(batch, nv, ln, dtype=torch.uint8, device=x.device)
        sc = torch.empty(batch, nv, dtype=torch.float32, device=x.device)
        st = torch.empty(batch, rows, dtype=torch.float32, device=x.device) if want_stat else None
    else:
        lv, sc, st = out
    L.sc_quantize(x, rows, cols, cols, batch, rows * cols, axis, sc_prec, stat_mode, lv, sc, st,
                  dev_status, stream)
    return lv, sc, st


def quantize_chunked(x: torch.Tensor, chunk: int, sc_prec: int = 8, stat_mode: int = L.SC_STAT_AMAX,
                     want_stat: bool = False, dev_status=None, stream=None):
    """x [batch, rows, cols] fp32 CUDA -> (levels [batch, rows, cols],
    scales [batch, rows, cols // chunk], stat [batch, rows] or None)."""
    _require_cuda(x, "x")
    if x.dim() == 2:
        x = x.unsqueeze(0)
    batch, rows, cols = x.shape
    if chunk < 1 or cols % chunk:
        raise ValueError(f"chunk {chunk} must divide cols {cols}")
    lv = torch.empty(batch, rows, cols, dtype=torch.uint8, device=x.device)
    sc = torch.empty(batch, rows, cols // chunk, dtype=torch.float32, device=x.device)
    st = torch.empty(batch, rows, dtype=torch.float32, device=x.device) if want_stat else None
    L.sc_quantize_chunked(x, rows, cols, cols, batch, rows * cols, chunk, sc_prec, stat_mode, lv, sc,
                          st, dev_status, stream)
    return lv, sc, st


def assign_rows(stat: torch.Tensor, tau, n_rungs: int, stream=None, out=None):
    """stat [batch, rows] -> (rung [batch, rows], perm [batch, rows], offsets [batch, n_rungs+1])."""
    _require_cuda(stat, "stat")
    batch, rows = stat.shape
    t = np.ascontiguousarray(tau if n_rungs > 1 else [0.0], dtype=np.float32)
    if out is None:
        rung = torch.empty(batch, rows, dtype=torch.int32, device=stat.device)
        perm = torch.empty(batch, rows, dtype=torch.int32, device=stat.device)
        offs = torch.empty(batch, n_rungs + 1, dtype=torch.int32, device=stat.device)
    else:
        rung, perm, offs = out
    L.sc_assign_rows(stat, rows, batch, t, n_rungs, rung, perm, offs, stream)
    return rung, perm, offs


def assign_fraction(stat: torch.Tensor, fractions, set_size: int = 0, stream=None):
    """Fraction-based fixed MP: stat [batch, rows] -> (rung, perm, offsets);
    fractions[k] is the share of units on rung k (ascending length)."""
    _require_cuda(stat, "stat")
    batch, rows = stat.shape
    fr = np.ascontiguousarray(fractions, dtype=np.float64)
    n_rungs = len(fr)
    rung = torch.empty(batch, rows, dtype=torch.int32, device=stat.device)
    perm = torch.empty(batch, rows, dtype=torch.int32, device=stat.device)
    offs = torch.empty(batch, n_rungs + 1, dtype=torch.int32, device=stat.device)
    L.sc_assign_fraction(stat, rows, batch, set_size, fr, n_rungs, rung, perm, offs, stream)
    return rung, perm, offs


def matmul(a_lv, a_s, b_lv, b_s, rung, perm, offs, table: ScTable, *, op=L.SC_OP_LINEAR,
           engine=L.SC_ENGINE_AUTO, q_dec=0.0, want_counts=False, dev_status=None, stream=None,
           out=None, counts=None, scales=L.SC_SCALES_ROW, workspace=None,
           mode=L.SC_MODE_BIPOLAR):
    """Levels [batch, M, D] x [batch, N, D] -> fp32 [batch, M, N] (and int32 counts).
    scales=SC_SCALES_BAND: a_s [batch, M, n_bands], b_s [batch, N, n_bands].
    workspace: optional device tensor the call may use as scratch."""
    batch, M, D = a_lv.shape
    N = b_lv.shape[1]
    dev = a_lv.device
    if out is None:
        out = torch.empty(batch, M, N, dtype=torch.float32, device=dev)
    if want_counts and counts is None:
        nb = max(table.n_bands, 1)
        counts = torch.empty(batch, nb, M, N, dtype=torch.int32, device=dev)
    desc = L.ScMatmulDesc(M, N, D, batch, op, engine, q_dec, scales, mode,
                          None if workspace is None else workspace.data_ptr(),
                          0 if workspace is None else workspace.numel() * workspace.element_size())
    L.sc_matmul(desc, a_lv, a_s, b_lv, b_s, rung, perm, offs, table.handle, out, counts,
                dev_status, stream)
    return out, counts


class ScStep:
    """All device buffers of one workload, and the full hot-path step:
    quantise A (+ row statistic), quantise B, assign rows (rung-sorted order),
    SC count + decode.  Four C-ABI calls on one stream, no host sync."""

    def __init__(self, w: Workload, device="cuda", engine=L.SC_ENGINE_AUTO, want_counts=False,
                 use_workspace=True, prepare_b=False):
        self.w = w
        self.device = torch.device(device)
        self.engine = engine
        self.n_rungs = len(w.ladder)
        band_len = None
        if w.n_bands:
            band_len = kband_tilt(w.ladder, w.n_bands, w.tilt, 1 << w.sc_prec)
        self.band_len = band_len
        self.table = ScTable(w.ladder, w.sc_prec, band_len, w.chunk_d, w.D if w.n_bands else 0,
                             w.b_shift, w.b_antithetic,
                             L.SC_ORDER_GRAY if w.gray else L.SC_ORDER_NATURAL, w.pool)
        self.a = w.a.to(self.device).contiguous()
        self.b = w.b.to(self.device).contiguous()
        B, M, D, N = w.batch, w.M, w.D, w.N
        dv = self.device
        if w.band_scales and (not w.n_bands or w.b_axis != 0):
            raise ValueError("per-band scales need K-bands and B given as [N, D]")
        ns = (w.n_bands,) if w.band_scales else ()  # one scale per (row, band)
        self.a_lv = torch.empty(B, M, D, dtype=torch.uint8, device=dv)
        self.a_s = torch.empty(B, M, *ns, dtype=torch.float32, device=dv)
        self.stat = torch.empty(B, M, dtype=torch.float32, device=dv)
        self.b_lv = torch.empty(B, N, D, dtype=torch.uint8, device=dv)
        self.b_s = torch.empty(B, N, *ns, dtype=torch.float32, device=dv)
        self.rung = torch.empty(B, M, dtype=torch.int32, device=dv)
        self.perm = torch.empty(B, M, dtype=torch.int32, device=dv)
        self.offs = torch.empty(B, self.n_rungs + 1, dtype=torch.int32, device=dv)
        self.out = torch.empty(B, M, N, dtype=torch.float32, device=dv)
        self.counts = (torch.empty(B, max(w.n_bands, 1), M, N, dtype=torch.int32, device=dv)
                       if want_counts else None)
        self.dev_status = torch.zeros(1, dtype=torch.int32, device=dv)
        self.tau = np.ascontiguousarray(w.tau if self.n_rungs > 1 else [0.0], dtype=np.float32)
        self.fractions = (np.ascontiguousarray(w.fractions, dtype=np.float64) if w.fractions
                          else None)
        self.desc = L.ScMatmulDesc(M, N, D, B, w.op, engine, 0.0,
                                   L.SC_SCALES_BAND if w.band_scales else L.SC_SCALES_ROW,
                                   L.SC_MODE_UNIPOLAR if w.unipolar else L.SC_MODE_BIPOLAR)
        # scratch for the fp64 band sums of the wide-tile band kernel
        self.workspace = None
        nbytes = L.sc_matmul_workspace_bytes(self.desc, self.table.handle) if use_workspace else 0
        if nbytes > 0:
            self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=dv)
            self.desc.workspace = self.workspace.data_ptr()
            self.desc.workspace_bytes = nbytes
        # a static second operand (a layer's weight): quantised and prepared
        # once here, as at layer load; run() then quantises A only
        self.b_prep = None
        self.prep_ms = 0.0
        if prepare_b:
            ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ev0.record()
            self._quantize_b(self.b, None)
            self.b_prep = L.sc_prepare_b(self.desc, self.b_lv, self.table.handle)
            ev1.record()
            torch.cuda.synchronize()
            self.prep_ms = ev0.elapsed_time(ev1)
            self.desc.b_prep = self.b_prep

    def _quantize_b(self, b, stream):
        w = self.w
        B, D, N = w.batch, w.D, w.N
        if w.band_scales:
            L.sc_quantize_chunked(b, N, D, D, B, N * D, w.chunk_d, w.sc_prec, L.SC_STAT_AMAX,
                                  self.b_lv, self.b_s, None, self.dev_status, stream)
        elif w.b_axis == 0:
            L.sc_quantize(b, N, D, D, B, N * D, 0, w.sc_prec, L.SC_STAT_AMAX, self.b_lv,
                          self.b_s, None, self.dev_status, stream)
        else:
            L.sc_quantize(b, D, N, N, B, D * N, 1, w.sc_prec, L.SC_STAT_AMAX, self.b_lv,
                          self.b_s, None, self.dev_status, stream)

    def run(self, stream=None, a=None, b=None, events=None, out=None):
        """One pass of the hot path.  a / b: optional replacement inputs of the
        same shape (device tensors; b is ignored when the second operand was
        prepared once).  events: optional (start, end) CUDA events recorded on
        `stream` around the count + decode call."""
        w = self.w
        a = self.a if a is None else a
        b = self.b if b is None else b
        B, M, D, N = w.batch, w.M, w.D, w.N
        if w.band_scales:
            # one scale per (row, band): the bands are the quantisation chunks
            L.sc_quantize_chunked(a, M, D, D, B, M * D, w.chunk_d, w.sc_prec, w.stat_mode,
                                  self.a_lv, self.a_s, self.stat, self.dev_status, stream)
        else:
            L.sc_quantize(a, M, D, D, B, M * D, 0, w.sc_prec, w.stat_mode, self.a_lv, self.a_s,
                          self.stat, self.dev_status, stream)
        if self.b_prep is None:
            self._quantize_b(b, stream)
        if self.fractions is not None:  # fraction-based fixed MP
            L.sc_assign_fraction(self.stat, M, B, w.frac_set, self.fractions, self.n_rungs,
                                 self.rung, self.perm, self.offs, stream)
        else:
            L.sc_assign_rows(self.stat, M, B, self.tau, self.n_rungs, self.rung, self.perm,
                             self.offs, stream)
        if events is not None:
            events[0].record(stream)
        out = self.out if out is None else out
        L.sc_matmul(self.desc, self.a_lv, self.a_s, self.b_lv, self.b_s, self.rung, self.perm,
                    self.offs, self.table.handle, out, self.counts, self.dev_status, stream)
        if events is not None:
            events[1].record(stream)
        return out

    def engine_used(self) -> str:
        e = L.sc_matmul_engine(self.desc, self.table.handle)
        return {L.SC_ENGINE_GATHER: "gather", L.SC_ENGINE_TC: "tc"}[e]

    def row_lengths(self) -> np.ndarray:
        """Stream length L_i of every row (after run()), [batch, M]."""
        lad = np.asarray(self.w.ladder, dtype=np.int64)
        return lad[self.rung.cpu().numpy()]

    def bitops(self) -> int:
        """sum_i L_i * N * D for the last run (iso-compute: bands do not change it)."""
        return int(self.row_lengths().sum()) * self.w.N * self.w.D

    def launches(self) -> int:
        """Kernels one run() launches: two quantisations, the row assignment
        (two kernels with fractions: rank, then the rung-sorted order) and
        those of sc_matmul (none for an empty call)."""
        w = self.w
        n = (1 if w.batch * w.M * w.D else 0)
        n += 1 if w.batch * w.N * w.D and self.b_prep is None else 0
        n += (2 if self.fractions is not None else 1) if w.batch and w.M else 0
        return n + L.sc_matmul_launches(self.desc, self.table.handle)

    def fold_macs(self) -> int:
        """Algorithmic int8 MACs of the exact contraction for the last run:
        sum over bands and rows of K(L) * N * (band width), K(L) = ceil(L / 2)
        (bipolar: the folded window) or L (unipolar: the L stream positions)."""
        rung = self.rung.cpu().numpy()
        w = self.w
        per = (lambda L: L) if w.unipolar else (lambda L: (L + 1) // 2)
        if self.band_len is None:
            fold = per(np.asarray(w.ladder, dtype=np.int64))
            return int(fold[rung].sum()) * w.N * w.D
        fold = per(self.band_len.astype(np.int64))             # [n_bands, n_rungs]
        return int(fold[:, rung].sum()) * w.N * w.chunk_d

    def close(self):
        if self.b_prep:
            L.sc_bprep_destroy(self.b_prep)
            self.b_prep = None
            self.desc.b_prep = None
        self.table.close()


class HostPipeline:
    """A step over a sequence of host (pinned) inputs with host outputs, the
    copies overlapped with the compute: the upload of step k + 1 and the
    download of step k - 1 run while step k computes (one stream each,
    inputs and outputs double-buffered, ordered by events).  Every step still
    uploads its own inputs and downloads its own output.

    step: a ScStep (its second operand may be prepared, then only A is
    uploaded).  run(a_host, b_host, out_host, steps): a_host / b_host pinned
    CPU tensors of the step's input shapes (the same inputs every step, as a
    benchmark would), out_host a pinned CPU tensor of the output's shape."""

    def __init__(self, step: "ScStep"):
        self.step = step
        dev = step.device
        self.s_in = torch.cuda.Stream(device=dev)
        self.s_cmp = torch.cuda.Stream(device=dev)
        self.s_out = torch.cuda.Stream(device=dev)
        self.a = [torch.empty_like(step.a) for _ in range(2)]
        self.b = [torch.empty_like(step.b) for _ in range(2)] if step.b_prep is None else None
        self.o = [torch.empty_like(step.out) for _ in range(2)]

    def bytes_per_step(self):
        h2d = self.step.a.numel() * 4 + (self.step.b.numel() * 4 if self.b is not None else 0)
        return h2d, self.step.out.numel() * 4

    def run(self, a_host, b_host, out_host, steps: int):
        """Enqueue `steps` steps; returns (start, end) events bracketing them
        (start on the upload stream, end on the download stream)."""
        E = lambda: torch.cuda.Event(enable_timing=False)
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        in_ready = [E(), E()]
        done = [None, None]       # compute of the step that last used slot s
        out_free = [None, None]   # download of the step that last used slot s
        start.record(self.s_in)
        for k in range(steps):
            s = k % 2
            with torch.cuda.stream(self.s_in):
                if done[s] is not None:
                    self.s_in.wait_event(done[s])        # inputs of step k - 2 consumed
                self.a[s].copy_(a_host, non_blocking=True)
                if self.b is not None:
                    self.b[s].copy_(b_host, non_blocking=True)
                in_ready[s].record(self.s_in)
            with torch.cuda.stream(self.s_cmp):
                self.s_cmp.wait_event(in_ready[s])
                if out_free[s] is not None:
                    self.s_cmp.wait_event(out_free[s])   # output of step k - 2 downloaded
                self.step.run(stream=self.s_cmp, a=self.a[s],
                              b=None if self.b is None else self.b[s], out=self.o[s])
                done[s] = E()
                done[s].record(self.s_cmp)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(done[s])
                out_host.copy_(self.o[s], non_blocking=True)
                out_free[s] = E()
                out_free[s].record(self.s_out)
        # the last download ends the run; it waits for every earlier step
        self.s_out.wait_stream(self.s_in)
        self.s_out.wait_stream(self.s_cmp)
        end.record(self.s_out)
        return start, end

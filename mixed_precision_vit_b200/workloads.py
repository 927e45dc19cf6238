"""Seeded synthetic inputs for the SC matmul workloads.

This module only draws random tensors of the shapes, distributions and
structure of the ViT-L/14 operators the pages evaluate (DINOv2 ViT-L/14:
257 tokens, d = 1024, 16 heads of 64, MLP 4096).  It holds none of the SC
method's arithmetic: no quantisation, no statistic, no bitstream.  Both the
CUDA path and the CPU oracle consume exactly the tensors returned here.

Everything is drawn on the CPU with ``torch.Generator`` so that the same seed
gives the same bytes on any machine; the caller moves tensors to the GPU.

Workloads (M x N x D per matrix, groups):
  single : A [64x64], B [64x64] ~ N(0,1), seed 0; uniform L = 64.
  qk     : Q, K [256 x 257 x 64] ~ N(0,1); in every (batch, head) matrix and
           every tensor, round(0.02 * 257) = 5 rows picked by a seeded
           permutation are scaled by 8 (outlier rows); ladder keyed on
           ||Q_i||_inf; seed 1.
  av     : A = softmax(N(0, 2^2) logits) [256 x 257 x 257], V [256 x 257 x 64]
           ~ N(0,1); ladder keyed on max_j A_ij; seed 2.
  fc1    : X [4112 x 1024] Student-t(nu = 4), W [4096 x 1024] ~ N(0, 0.02^2),
           out = X W^T; ladder keyed on ||X_i||_inf; seed 3.
  fc2    : X [4112 x 4096] = GELU(N(0,1)) (erf form), W [1024 x 4096]
           ~ N(0, 0.02^2); contraction split in 16 bands of 256 with a linear
           tilt of the ladder; seed 4.
  fc2_bs : fc2 with one quantisation scale per (row, band of 256) instead of
           per row (same tensors, seed 4).
  qk_mp, av_mp, fc1_mp : the qk / av / fc1 tensors with fraction-based fixed
           MP instead of thresholds: lengths {256, 128, 64, 32} on 15 %,
           57.5 %, 22.5 %, 5 % of the units (the 8-bit "p7 mp" row of the
           scmp_vit config matrix); units are heads within each image of 16
           heads for qk, rows for av and fc1.
  qk_uni : the qk tensors in the unipolar AND mode (sign-magnitude streams).
  qk_gray: the qk tensors with the Sobol sequence in Gray-code order.
  qk_pool, fc2_pool : the qk / fc2 tensors with a per-index Sobol pool of the
           contraction width (64 / 4096 sequences: sobol_pool).
"""
from __future__ import annotations

import functools
from dataclasses import dataclass, field

import numpy as np
import torch

LADDER = (64, 96, 128, 192, 256)
TAU = (0.8, 0.6, 0.4, 0.2)
SC_PREC = 8

STAT_AMAX = 0      # g_i = max_j |x_ij|
STAT_ROWMAX = 1    # g_i = max_j x_ij

OP_LINEAR, OP_QK, OP_AV = 0, 1, 2


@dataclass
class Workload:
    name: str
    a: torch.Tensor          # row operand, fp32 [batch, M, D]
    b: torch.Tensor          # fp32 [batch, N, D] if b_axis == 0 else [batch, D, N]
    b_axis: int              # 0: B given as [N, D] (one scale per row); 1: [D, N] (per column)
    stat_mode: int
    ladder: tuple
    tau: tuple
    op: int = OP_LINEAR
    n_bands: int = 0
    chunk_d: int = 0
    tilt: float = 0.0
    sc_prec: int = SC_PREC
    meta: dict = field(default_factory=dict)
    band_scales: bool = False  # one quantisation scale per (row, band) instead of per row
    # fraction-based fixed MP: fraction of units per rung (ascending length)
    # instead of thresholds; frac_set 0 ranks rows within each group, > 0
    # ranks whole groups (heads) within sets of frac_set consecutive groups
    fractions: tuple = ()
    frac_set: int = 0
    unipolar: bool = False     # sign-magnitude AND streams instead of bipolar XNOR
    # seed-bank variant of the second operand's Sobol sequence (digital
    # shift of the integer points, antithetic 1 - u); the first keeps the default
    b_shift: int = 0
    b_antithetic: bool = False
    gray: bool = False         # the Sobol sequence in Gray-code order
    pool: np.ndarray = None    # int32 [n_pool, 2^sc_prec] points: index d uses row d mod n_pool

    @property
    def batch(self) -> int:
        return self.a.shape[0]

    @property
    def M(self) -> int:
        return self.a.shape[1]

    @property
    def D(self) -> int:
        return self.a.shape[2]

    @property
    def N(self) -> int:
        return self.b.shape[1] if self.b_axis == 0 else self.b.shape[2]


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _student_t(shape, nu: int, g: torch.Generator) -> torch.Tensor:
    # t = Z / sqrt(chi2_nu / nu), chi2_nu as a sum of nu squared normals
    z = torch.randn(shape, generator=g, dtype=torch.float64)
    chi2 = torch.zeros(shape, dtype=torch.float64)
    for _ in range(nu):
        chi2 += torch.randn(shape, generator=g, dtype=torch.float64) ** 2
    return (z / torch.sqrt(chi2 / nu)).to(torch.float32)


def _gelu_erf(x: torch.Tensor) -> torch.Tensor:
    xd = x.to(torch.float64)
    return (0.5 * xd * (1.0 + torch.erf(xd / 2.0 ** 0.5))).to(torch.float32)


def _with_outlier_rows(x: torch.Tensor, frac: float, factor: float, g: torch.Generator):
    batch, rows, _ = x.shape
    n_out = int(round(frac * rows))
    picks = []
    for bidx in range(batch):
        idx = torch.randperm(rows, generator=g)[:n_out]
        x[bidx, idx] *= factor
        picks.append(idx)
    return x, torch.stack(picks) if picks else torch.zeros(0, n_out, dtype=torch.long)


def single(seed: int = 0, M: int = 64, N: int = 64, D: int = 64) -> Workload:
    g = _gen(seed)
    a = torch.randn(1, M, D, generator=g)
    b = torch.randn(1, D, N, generator=g)
    return Workload("single", a, b, 1, STAT_AMAX, (64,), (), op=OP_LINEAR)


def qk(seed: int = 1, groups: int = 256, T: int = 257, dh: int = 64,
       outlier_frac: float = 0.02, outlier_scale: float = 8.0) -> Workload:
    g = _gen(seed)
    q = torch.randn(groups, T, dh, generator=g)
    k = torch.randn(groups, T, dh, generator=g)
    q, q_out = _with_outlier_rows(q, outlier_frac, outlier_scale, g)
    k, k_out = _with_outlier_rows(k, outlier_frac, outlier_scale, g)
    return Workload("qk", q, k, 0, STAT_AMAX, LADDER, TAU, op=OP_QK,
                    meta={"q_outliers": q_out, "k_outliers": k_out})


def av(seed: int = 2, groups: int = 256, T: int = 257, dh: int = 64,
       logit_std: float = 2.0) -> Workload:
    g = _gen(seed)
    logits = torch.randn(groups, T, T, generator=g, dtype=torch.float64) * logit_std
    attn = torch.softmax(logits, dim=-1).to(torch.float32)
    v = torch.randn(groups, T, dh, generator=g)
    return Workload("av", attn, v, 1, STAT_ROWMAX, LADDER, TAU, op=OP_AV)


def fc1(seed: int = 3, tokens: int = 16 * 257, d_in: int = 1024, d_out: int = 4096,
        w_std: float = 0.02) -> Workload:
    g = _gen(seed)
    x = _student_t((1, tokens, d_in), 4, g)
    w = torch.randn(1, d_out, d_in, generator=g) * w_std
    return Workload("fc1", x, w, 0, STAT_AMAX, LADDER, TAU, op=OP_LINEAR)


def fc2(seed: int = 4, tokens: int = 16 * 257, d_in: int = 4096, d_out: int = 1024,
        w_std: float = 0.02, n_bands: int = 16, tilt: float = 0.25,
        band_scales: bool = False) -> Workload:
    g = _gen(seed)
    x = _gelu_erf(torch.randn(1, tokens, d_in, generator=g))
    w = torch.randn(1, d_out, d_in, generator=g) * w_std
    if d_in % n_bands:
        raise ValueError("d_in must be a multiple of n_bands")
    return Workload("fc2_bs" if band_scales else "fc2", x, w, 0, STAT_AMAX, LADDER, TAU,
                    op=OP_LINEAR, n_bands=n_bands, chunk_d=d_in // n_bands, tilt=tilt,
                    band_scales=band_scales)


def fc2_bs(seed: int = 4, **kw) -> Workload:
    return fc2(seed=seed, band_scales=True, **kw)


# fraction-based fixed MP: lengths ascending with their share of the units
MP_LADDER = (32, 64, 128, 256)
MP_FRACTIONS = (0.05, 0.225, 0.575, 0.15)
HEADS = 16


def _with_fractions(w: Workload, name: str, frac_set: int) -> Workload:
    w.name = name
    w.ladder = MP_LADDER
    w.tau = ()
    w.fractions = MP_FRACTIONS
    w.frac_set = frac_set
    return w


def qk_mp(seed: int = 1, **kw) -> Workload:
    w = qk(seed=seed, **kw)
    return _with_fractions(w, "qk_mp", HEADS if w.batch % HEADS == 0 else w.batch)


def av_mp(seed: int = 2, **kw) -> Workload:
    return _with_fractions(av(seed=seed, **kw), "av_mp", 0)


def fc1_mp(seed: int = 3, **kw) -> Workload:
    return _with_fractions(fc1(seed=seed, **kw), "fc1_mp", 0)


def qk_uni(seed: int = 1, **kw) -> Workload:
    w = qk(seed=seed, **kw)
    w.name = "qk_uni"
    w.unipolar = True
    return w


BUILDERS = {"single": single, "qk": qk, "av": av, "fc1": fc1, "fc2": fc2, "fc2_bs": fc2_bs,
            "qk_mp": qk_mp, "av_mp": av_mp, "fc1_mp": fc1_mp, "qk_uni": qk_uni}


def make(name: str, **kw) -> Workload:
    return BUILDERS[name](**kw)


def qk_gray(seed: int = 1, **kw) -> Workload:
    w = qk(seed=seed, **kw)
    w.name = "qk_gray"
    w.gray = True
    return w


@functools.lru_cache(maxsize=16)
def _sobol_pool_cached(n_dims: int, sc_prec: int) -> bytes:
    eng = torch.quasirandom.SobolEngine(dimension=n_dims, scramble=False)
    pts = eng.draw(1 << sc_prec, dtype=torch.float64) * (1 << sc_prec)
    u = torch.round(pts).to(torch.int32).T.contiguous()
    return u.numpy().tobytes()


def sobol_pool(n_dims: int, sc_prec: int = 8) -> np.ndarray:
    """The random source of a per-index Sobol pool: the first 2^sc_prec points
    of dimensions 1..n_dims of an unscrambled Sobol generator (torch's
    SobolEngine, which emits them in Gray-code order), as integers
    u = x * 2^sc_prec in [0, 2^sc_prec), int32 [n_dims, 2^sc_prec].  Drawn once
    per (n_dims, sc_prec) and shared.  Holds none of the SC arithmetic: the
    thresholds, tables and counts are computed from these points by the
    library and by the oracle, each on its own."""
    u = np.frombuffer(_sobol_pool_cached(int(n_dims), int(sc_prec)), dtype=np.int32)
    return u.reshape(n_dims, 1 << sc_prec).copy()


def qk_pool(seed: int = 1, **kw) -> Workload:
    w = qk(seed=seed, **kw)
    w.name = "qk_pool"
    w.pool = sobol_pool(w.D, w.sc_prec)
    return w


def fc2_pool(seed: int = 4, **kw) -> Workload:
    w = fc2(seed=seed, **kw)
    w.name = "fc2_pool"
    w.pool = sobol_pool(w.D, w.sc_prec)
    return w


BUILDERS.update(qk_gray=qk_gray, qk_pool=qk_pool, fc2_pool=fc2_pool)

BASE_SEED = {"single": 0, "qk": 1, "av": 2, "fc1": 3, "fc2": 4, "fc2_bs": 4, "qk_mp": 1, "av_mp": 2,
             "fc1_mp": 3, "qk_uni": 1, "qk_gray": 1, "qk_pool": 1, "fc2_pool": 4}


def shard(name: str, rank: int, **kw) -> Workload:
    """The workload one rank of a data-parallel job runs (weak scaling: every
    rank has a whole problem of its own).  Attention workloads: the rank's own
    batch of independent (batch, head) groups, drawn with seed
    base + 1000 * rank.  Linear workloads: the rank's own batch of tokens (its
    own X, drawn the same way) against the weight of rank 0, which every rank
    holds (replicated W).  Rank 0's shard is the workload itself."""
    base = BASE_SEED[name]
    w = make(name, seed=base + 1000 * rank, **kw)
    if rank and w.op == OP_LINEAR:
        w.b = make(name, seed=base, **kw).b
    return w

"""GPU parity of fraction-based fixed mixed precision: per-row and per-head
rung assignment through the C ABI against the CPU oracle, and the whole step
(quantise, assign by fractions, count + decode) on both count engines.

Bar: rungs, the rung-sorted order and the offsets bit-identical; counts
bit-identical; fp32 outputs within 1e-6 relative error.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import pipeline
from mixed_precision_vit_b200 import _lib as L
from mixed_precision_vit_b200 import workloads as W

pytestmark = pytest.mark.gpu

REL_TOL = 1e-6
ENGINES = [L.SC_ENGINE_GATHER, L.SC_ENGINE_TC]
P7 = W.MP_FRACTIONS                                    # 5 / 22.5 / 57.5 / 15 %


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mixed_precision_vit_b200 import build
    build.build()
    oracle.build()
    L.load()


def _check_order(rung, perm, offs, n_rungs):
    for g in range(rung.shape[0]):
        assert np.array_equal(perm[g], np.argsort(rung[g], kind="stable"))
        hist = np.bincount(rung[g], minlength=n_rungs)
        assert np.array_equal(offs[g], np.concatenate([[0], np.cumsum(hist)]))


# (batch, rows, set_size, fractions, statistic recipe)
CASES = [
    (3, 257, 0, P7, "normal"),
    (1, 4112, 0, P7, "normal"),
    (2, 5000, 0, (0.25, 0.25, 0.25, 0.25), "ties"),       # many equal statistics
    (2, 300, 0, (1 / 3, 1 / 3, 1 / 3), "nan"),            # NaN and -inf ranked last
    (1, 1, 0, (0.5, 0.5), "normal"),
    (32, 257, 16, P7, "normal"),                          # 2 images x 16 heads
    (48, 7, 16, (1 / 3, 1 / 3, 1 / 3), "ties"),
    (5, 40, 5, (0.0, 1.0), "normal"),
    (4, 64, 0, (1.0,), "normal"),
]


@pytest.mark.parametrize("k", range(len(CASES)))
def test_assign_fraction_matches_oracle(k):
    from mixed_precision_vit_b200.sc import assign_fraction
    batch, rows, set_size, fr, kind = CASES[k]
    rng = np.random.default_rng(100 + k)
    if kind == "ties":
        stat = rng.integers(0, 6, (batch, rows)).astype(np.float32)
    else:
        stat = np.abs(rng.standard_normal((batch, rows))).astype(np.float32)
    if kind == "nan":
        stat[:, ::7] = np.nan
        stat[:, 3::11] = -np.inf
    rung, perm, offs = assign_fraction(torch.from_numpy(stat).cuda(), fr, set_size)
    torch.cuda.synchronize()
    want = oracle.assign_fraction(stat, fr, set_size)
    got = rung.cpu().numpy()
    assert np.array_equal(got, want)
    _check_order(got, perm.cpu().numpy(), offs.cpu().numpy(), len(fr))


def test_assign_fraction_rejects_bad_arguments():
    from mixed_precision_vit_b200.sc import assign_fraction
    stat = torch.ones(4, 8, device="cuda")
    for fr, ss in [((0.5, 0.4), 0), ((1.5, -0.5), 0), ((0.5, 0.5), 3)]:
        with pytest.raises(L.ScError) as e:
            assign_fraction(stat, fr, ss)
        assert e.value.code == L.SC_ERR_ARG


SMALL = {
    "qk_mp": lambda: W.qk_mp(groups=32),
    "av_mp": lambda: W.av_mp(groups=3),
    "fc1_mp": lambda: W.fc1_mp(tokens=300, d_in=160, d_out=200),
}


@pytest.mark.parametrize("engine", ENGINES)
@pytest.mark.parametrize("name", list(SMALL))
def test_fraction_mp_step_parity(name, engine):
    from mixed_precision_vit_b200.sc import ScStep
    w = SMALL[name]()
    s = ScStep(w, engine=engine, want_counts=True)
    s.run()
    torch.cuda.synchronize()
    st, counts, out, steps = pipeline.run(w)
    assert np.array_equal(s.stat.cpu().numpy(), st.stat)
    assert np.array_equal(s.rung.cpu().numpy(), st.rung)
    _check_order(st.rung, s.perm.cpu().numpy(), s.offs.cpu().numpy(), len(w.ladder))
    assert np.array_equal(s.counts.cpu().numpy(), np.moveaxis(counts, -1, 1))
    got = s.out.cpu().numpy().astype(np.float64)
    want = np.asarray(out, np.float64)
    zero = want == 0
    assert np.all(got[zero] == 0)
    rel = np.abs(got[~zero] - want[~zero]) / np.abs(want[~zero])
    assert rel.size == 0 or rel.max() <= REL_TOL, f"{name}: max rel err {rel.max():.3e}"
    assert steps == s.bitops()
    assert s.dev_status.item() == 0
    s.close()


def test_fraction_mp_full_size_qk_rungs_and_sampled_outputs():
    """qk_mp at full size (256 heads in 16 images): every rung exact, sampled
    outputs against the oracle."""
    from mixed_precision_vit_b200.sc import ScStep
    w = W.qk_mp()
    s = ScStep(w, want_counts=True)
    s.run()
    torch.cuda.synchronize()
    st = pipeline.prepare(w)
    assert np.array_equal(s.rung.cpu().numpy(), st.rung)
    # per image: the head counts per length follow the fractions
    heads = st.rung[:, 0].reshape(-1, 16)
    assert np.all(np.bincount(heads[0], minlength=4) == np.bincount(heads[-1], minlength=4))
    rng = np.random.default_rng(13)
    sel = np.array([(rng.integers(w.batch), rng.integers(w.M), rng.integers(w.N))
                    for _ in range(800)], np.int64)
    _, counts, out, _ = pipeline.run(w, st, sel=sel)
    g, i, j = sel.T
    assert np.array_equal(s.counts.cpu().numpy()[g, :, i, j], counts)
    got = s.out.cpu().numpy()[g, i, j].astype(np.float64)
    want = np.asarray(out, np.float64)
    nz = want != 0
    assert np.all(got[~nz] == 0)
    assert np.max(np.abs(got[nz] - want[nz]) / np.abs(want[nz])) <= REL_TOL
    s.close()

"""GPU parity of the other Sobol sequences ("scmp_vit" README: the Sobol pool
of a (contraction width, precision) pair, _CFG_CACHE[(D, sc_prec)], shared by
every op of that width): the first dimension in Gray-code order, and a
per-index pool in which contraction index d streams both operands from
sequence d mod n_pool.  Every count bit-identical to the oracle, every output
within 1e-6 relative error.
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


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mixed_precision_vit_b200 import build
    build.build()
    oracle.build()
    L.load()


def _check(s, counts, out, where):
    got_c = s.counts.cpu().numpy()
    want_c = np.moveaxis(counts, -1, 1)
    n_bad = int(np.count_nonzero(got_c != want_c))
    assert n_bad == 0, f"{where}: {n_bad} of {want_c.size} counts differ"
    got = s.out.cpu().numpy().astype(np.float64)
    want = out.astype(np.float64)
    zero = want == 0
    assert np.all(got[zero] == 0), where
    rel = np.abs(got[~zero] - want[~zero]) / np.abs(want[~zero])
    assert rel.size == 0 or rel.max() <= REL_TOL, f"{where}: max rel err {rel.max():.3e}"


def _run(w, engine):
    from mixed_precision_vit_b200.sc import ScStep
    s = ScStep(w, engine=engine, want_counts=True)
    s.run()
    torch.cuda.synchronize()
    assert s.dev_status.item() == 0
    return s


SMALL = {
    "qk_gray": lambda: W.qk_gray(groups=3),
    "fc2_gray": lambda: _gray(W.fc2(tokens=150, d_in=16 * 24, d_out=130)),
    "qk_pool": lambda: W.qk_pool(groups=3),
    "fc2_pool": lambda: W.fc2_pool(tokens=150, d_in=16 * 24, d_out=130),
    "fc1_pool_unipolar": lambda: _unipolar(W.fc1(tokens=90, d_in=160, d_out=70), pool=True),
}


def _gray(w):
    w.name += "_gray"
    w.gray = True
    return w


def _unipolar(w, pool=False):
    w.unipolar = True
    if pool:
        w.pool = W.sobol_pool(w.D, w.sc_prec)
    return w


@pytest.mark.parametrize("engine", [L.SC_ENGINE_GATHER, L.SC_ENGINE_TC])
@pytest.mark.parametrize("name", list(SMALL))
def test_small_every_output(name, engine):
    w = SMALL[name]()
    if engine == L.SC_ENGINE_TC and w.pool is not None:
        from mixed_precision_vit_b200.sc import ScStep
        with pytest.raises(L.ScError) as e:   # refused when the step resolves its engine
            s = ScStep(w, engine=engine, want_counts=True)
            s.run()
        assert e.value.code == L.SC_ERR_UNSUPPORTED
        return
    s = _run(w, engine)
    _, counts, out, steps = pipeline.run(w)
    _check(s, counts, out, name)
    assert steps == s.bitops()
    s.close()


def test_gray_differs_from_natural():
    """Same inputs, the two orders: different counts at 96 / 192, so the
    option reaches the kernels."""
    from mixed_precision_vit_b200.sc import ScStep
    a = _run(W.qk(groups=2), L.SC_ENGINE_TC)
    b = _run(W.qk_gray(groups=2), L.SC_ENGINE_TC)
    rung = a.rung.cpu().numpy()
    assert np.any((rung == 1) | (rung == 3))
    assert not torch.equal(a.counts, b.counts)
    a.close()
    b.close()


@pytest.mark.parametrize("name", ["qk_gray", "qk_pool"])
def test_full_size_every_output(name):
    w = W.make(name)
    s = _run(w, L.SC_ENGINE_AUTO)
    assert s.engine_used() == ("gather" if w.pool is not None else "tc")
    _, counts, out, steps = pipeline.run(w, memo=True)
    _check(s, counts, out, name)
    assert steps == s.bitops()
    s.close()


def test_full_size_fc2_pool_sampled():
    """fc2 with a pool of 4096 sequences (one per contraction index): the
    oracle's memo would need a table per (sequence, length), so the outputs
    are sampled (every row of the longer rungs at random columns, random
    outputs, the corners) and computed bit by bit."""
    w = W.make("fc2_pool")
    s = _run(w, L.SC_ENGINE_AUTO)
    st = pipeline.prepare(w)
    rng = np.random.default_rng(41)
    sel = [(0, i, rng.integers(w.N)) for i in np.nonzero(st.rung[0] >= 3)[0][::16]]
    sel += [(0, rng.integers(w.M), rng.integers(w.N)) for _ in range(800)]
    sel += [(0, i, j) for i in (0, w.M - 1) for j in (0, w.N - 1)]
    sel = np.array(sel, np.int64)
    _, counts, out, _ = pipeline.run(w, st, sel=sel)
    g, i, j = sel.T
    assert np.array_equal(s.counts.cpu().numpy()[g, :, i, j], counts)
    got = s.out.cpu().numpy()[g, i, j].astype(np.float64)
    nz = out != 0
    assert np.all(got[~nz] == 0)
    assert np.max(np.abs(got[nz] - out[nz]) / np.abs(out[nz])) <= REL_TOL
    s.close()


def test_pool_table_cache_is_keyed_by_width():
    """ScTable.for_width: one table per (ladder, D, sc_prec, bands, pool
    size), shared by every caller of that width."""
    from mixed_precision_vit_b200.sc import ScTable
    t1 = ScTable.for_width(W.LADDER, 64)
    t2 = ScTable.for_width(W.LADDER, 64)
    t3 = ScTable.for_width(W.LADDER, 128)
    assert t1 is t2 and t1 is not t3
    assert t1.handle and t3.handle


def test_pool_must_be_permutations():
    from mixed_precision_vit_b200.sc import ScTable
    pool = W.sobol_pool(4, 8)
    pool[2, 5] = pool[2, 6]
    with pytest.raises(L.ScError) as e:
        ScTable(W.LADDER, pool=pool)
    assert e.value.code == L.SC_ERR_TABLE
    with pytest.raises(L.ScError) as e:
        ScTable(W.LADDER, pool=W.sobol_pool(4, 8), order=L.SC_ORDER_GRAY)
    assert e.value.code == L.SC_ERR_ARG

"""GPU parity of the unipolar AND mode (sign-magnitude streams, one
enable-gated counter) on both engines -- the tensor cores (the signed
thermometer of n = C[2|x_a|][L] ones against sgn_b K[2|x_b|, .] over the L
stream positions, an exact int8 contraction) and the CUDA cores -- through
the C ABI, against the CPU oracle on the same seeded inputs.

Bar: signed counts bit-identical; fp32 outputs within 1e-6 relative error.
"""
import dataclasses

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


def _check_outputs(got, want, where=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    zero = want == 0
    assert np.all(got[zero] == 0), f"{where}: nonzero where oracle is exactly 0"
    rel = np.abs(got[~zero] - want[~zero]) / np.abs(want[~zero])
    assert rel.size == 0 or rel.max() <= REL_TOL, f"{where}: max rel err {rel.max():.3e}"


def _uni(w):
    return dataclasses.replace(w, unipolar=True)


CASES = {
    "qk": lambda: W.qk_uni(groups=3),
    "av": lambda: _uni(W.av(groups=2)),
    "fc1": lambda: _uni(W.fc1(tokens=300, d_in=160, d_out=200)),
    "fc2_bands": lambda: _uni(W.fc2(tokens=150, d_in=16 * 24, d_out=130)),
    "fc2_band_scales": lambda: _uni(W.fc2_bs(tokens=150, d_in=16 * 24, d_out=130)),
    "qk_mp": lambda: _uni(W.qk_mp(groups=16)),
}


@pytest.mark.parametrize("engine", [L.SC_ENGINE_GATHER, L.SC_ENGINE_TC])
@pytest.mark.parametrize("name", list(CASES))
def test_unipolar_parity(name, engine):
    from mixed_precision_vit_b200.sc import ScStep
    w = CASES[name]()
    s = ScStep(w, engine=engine, want_counts=True)
    assert s.engine_used() == ("gather" if engine == L.SC_ENGINE_GATHER else "tc")
    s.run()
    torch.cuda.synchronize()
    st, counts, out, steps = pipeline.run(w)
    assert np.array_equal(s.rung.cpu().numpy(), st.rung)
    assert np.array_equal(s.counts.cpu().numpy(), np.moveaxis(counts, -1, 1))
    _check_outputs(s.out.cpu().numpy(), out, name)
    assert steps == s.bitops()
    assert s.dev_status.item() == 0
    s.close()


def test_unipolar_counts_are_signed_and_differ_from_bipolar():
    from mixed_precision_vit_b200.sc import ScStep
    w = W.qk(groups=2)
    outs = []
    for uni in (False, True):
        s = ScStep(dataclasses.replace(w, unipolar=uni), engine=L.SC_ENGINE_GATHER,
                   want_counts=True)
        s.run()
        torch.cuda.synchronize()
        outs.append((s.counts.cpu().numpy(), s.out.cpu().numpy()))
        s.close()
    assert (outs[1][0] < 0).any() and not (outs[0][0] < 0).any()
    assert not np.array_equal(outs[0][1], outs[1][1])


def test_unipolar_tensor_memory_band_sums():
    """fc2 bands in the unipolar mode without a workspace: the band kernel
    that keeps its fp64 sums in tensor memory."""
    from mixed_precision_vit_b200.sc import ScStep
    w = _uni(W.fc2(tokens=300, d_in=16 * 24, d_out=200))
    s = ScStep(w, engine=L.SC_ENGINE_TC, want_counts=True, use_workspace=False)
    assert s.workspace is None
    s.run()
    torch.cuda.synchronize()
    _, counts, out, _ = pipeline.run(w)
    assert np.array_equal(s.counts.cpu().numpy(), np.moveaxis(counts, -1, 1))
    _check_outputs(s.out.cpu().numpy(), out, "fc2 unipolar tmem sums")
    s.close()


@pytest.mark.parametrize("L_", [1, 15, 16, 17, 33, 100, 255, 256])
def test_unipolar_lengths_on_tensor_cores(L_):
    """Single-length ladders across the chunk counts 1..16 of the unipolar
    operands (round16(L) contraction bytes per index), with a ragged D."""
    from mixed_precision_vit_b200.sc import ScStep
    w = _uni(W.fc1(tokens=200, d_in=37, d_out=45, seed=7))
    w = dataclasses.replace(w, ladder=(L_,), tau=())
    s = ScStep(w, engine=L.SC_ENGINE_TC, want_counts=True)
    s.run()
    torch.cuda.synchronize()
    _, counts, out, _ = pipeline.run(w)
    assert np.array_equal(s.counts.cpu().numpy(), np.moveaxis(counts, -1, 1))
    _check_outputs(s.out.cpu().numpy(), out, f"unipolar L={L_}")
    assert s.dev_status.item() == 0
    s.close()


def test_unipolar_full_size_qk_sampled():
    from mixed_precision_vit_b200.sc import ScStep
    w = W.qk_uni()
    s = ScStep(w, want_counts=True)
    s.run()
    torch.cuda.synchronize()
    st = pipeline.prepare(w)
    rng = np.random.default_rng(15)
    sel = np.array([(rng.integers(w.batch), rng.integers(w.M), rng.integers(w.N))
                    for _ in range(1000)], np.int64)
    _, counts, out, _ = pipeline.run(w, st, sel=sel)
    g, i, j = sel.T
    assert np.array_equal(s.counts.cpu().numpy()[g, :, i, j], counts)
    _check_outputs(s.out.cpu().numpy()[g, i, j], out, "qk_uni full size")
    s.close()

"""GPU parity of the Sobol seed-bank variants of the second operand's
sequence (digital shift, antithetic) on every engine: the tensor-core kernel
with its leftover-row kernel, the band kernels and the CUDA-core engine
(bipolar and unipolar), through the C ABI, against the CPU oracle.

Bar: counts bit-identical; fp32 outputs within 1e-6 relative error.
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
VARIANTS = [(0, True), (91, False), (200, True)]
ENGINES = [L.SC_ENGINE_GATHER, L.SC_ENGINE_TC]


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


BASES = {
    "qk": lambda: W.qk(groups=3),
    "av": lambda: W.av(groups=2),
    "fc2_bands": lambda: W.fc2(tokens=150, d_in=16 * 24, d_out=130),
    "qk_unipolar": lambda: W.qk_uni(groups=3),
}


@pytest.mark.parametrize("variant", VARIANTS, ids=lambda v: f"shift{v[0]}_anti{int(v[1])}")
@pytest.mark.parametrize("engine", ENGINES)
@pytest.mark.parametrize("name", list(BASES))
def test_seed_bank_variant_parity(name, engine, variant):
    from mixed_precision_vit_b200.sc import ScStep
    base = BASES[name]()
    if base.unipolar and engine == L.SC_ENGINE_TC:
        pytest.skip("the unipolar mode runs on the CUDA-core engine")
    w = dataclasses.replace(base, b_shift=variant[0], b_antithetic=variant[1])
    s = ScStep(w, engine=engine, want_counts=True)
    s.run()
    torch.cuda.synchronize()
    st, counts, out, _ = pipeline.run(w)
    assert np.array_equal(s.counts.cpu().numpy(), np.moveaxis(counts, -1, 1))
    _check_outputs(s.out.cpu().numpy(), out, f"{name} {variant}")
    assert s.dev_status.item() == 0
    s.close()


def test_default_variant_is_the_plain_table_and_variants_differ():
    from mixed_precision_vit_b200.sc import ScStep
    base = W.qk(groups=2)
    res = []
    for v in [(0, False), (0, True)]:
        s = ScStep(dataclasses.replace(base, b_shift=v[0], b_antithetic=v[1]), want_counts=True)
        s.run()
        torch.cuda.synchronize()
        res.append(s.counts.cpu().numpy())
        s.close()
    plain = ScStep(base, want_counts=True)
    plain.run()
    torch.cuda.synchronize()
    assert np.array_equal(res[0], plain.counts.cpu().numpy())
    assert not np.array_equal(res[1], res[0])
    plain.close()


def test_variant_arguments_are_checked():
    with pytest.raises(L.ScError) as e:
        L.sc_build_table_variant(8, np.array([64], np.int32), 1, None, 0, 0, 0, 256, 0)
    assert e.value.code == L.SC_ERR_ARG
    with pytest.raises(L.ScError) as e:
        L.sc_build_table_variant(8, np.array([64], np.int32), 1, None, 0, 0, 0, 0, 2)
    assert e.value.code == L.SC_ERR_ARG

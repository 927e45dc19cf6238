"""GPU parity of per-(row, band) quantisation scales with K-bands: chunked
quantisation and the band-scale decode of both count engines, through the C
ABI, against the CPU oracle on the same seeded inputs.

Bar: levels, scales, statistics and counts bit-identical; fp32 outputs within
1e-6 relative error element by element.
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
LADDER = (64, 96, 128, 192, 256)
TAU = (0.8, 0.6, 0.4, 0.2)


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


# (rows, cols, chunk): register path with 1, 2, 4 and 8 float4 per lane,
# and the scalar path (chunk not a multiple of 4)
QC_SHAPES = [(37, 96, 32), (65, 512, 256), (9, 1536, 512), (5, 2048, 1024), (40, 45, 15), (3, 7, 7)]


@pytest.mark.parametrize("stat_mode", [L.SC_STAT_AMAX, L.SC_STAT_ROWMAX])
@pytest.mark.parametrize("shape", QC_SHAPES)
def test_quantize_chunked_matches_oracle(shape, stat_mode):
    from mixed_precision_vit_b200.sc import quantize_chunked
    rows, cols, chunk = shape
    g = torch.Generator().manual_seed(rows * cols + chunk)
    x = torch.randn(2, rows, cols, generator=g)
    x[:, :, : cols // 3] *= 9.0                                   # chunks of different range
    x[0, 1 % rows, :] = 0.0                                       # an all-zero row
    lv, sc, st = quantize_chunked(x.cuda(), chunk, stat_mode=stat_mode, want_stat=True)
    lv0, sc0, _ = quantize_chunked(x.cuda(), chunk)                # no statistic: packed path
    for b in range(2):
        want_lv, want_sc = oracle.quantize_chunked(x[b].numpy(), chunk)
        assert np.array_equal(lv[b].cpu().numpy(), want_lv)
        assert np.array_equal(sc[b].cpu().numpy(), want_sc)
        assert np.array_equal(lv0[b].cpu().numpy(), want_lv)
        assert np.array_equal(sc0[b].cpu().numpy(), want_sc)
        xb = x[b].numpy()
        want_st = np.abs(xb).max(axis=1) if stat_mode == L.SC_STAT_AMAX else xb.max(axis=1)
        assert np.array_equal(st[b].cpu().numpy(), want_st.astype(np.float32))


def _band_workload(M, N, n_bands, chunk_d, tilt, batch=1, seed=0, ladder=LADDER, tau=TAU):
    g = torch.Generator().manual_seed(seed)
    D = n_bands * chunk_d
    a = torch.randn(batch, M, D, generator=g)
    b = torch.randn(batch, N, D, generator=g) * 0.05
    # bands of very different range, so that per-band scales matter
    ramp = torch.logspace(-1, 1, n_bands).repeat_interleave(chunk_d)
    a = a * ramp
    return W.Workload("band_scales", a, b, 0, W.STAT_AMAX, tuple(ladder), tuple(tau),
                      n_bands=n_bands, chunk_d=chunk_d, tilt=tilt, band_scales=True)


BS_CASES = [
    dict(M=300, N=100, n_bands=5, chunk_d=7, tilt=0.3),            # odd band width, ragged tiles
    dict(M=600, N=230, n_bands=4, chunk_d=16, tilt=-0.2, batch=2), # row tiles + leftovers, 3 col tiles
    dict(M=150, N=130, n_bands=16, chunk_d=24, tilt=0.25),         # fc2-like band layout, small
    dict(M=64, N=33, n_bands=1, chunk_d=48, tilt=0.0, ladder=(100,), tau=()),
]


@pytest.mark.parametrize("ws", [True, False], ids=["workspace_sums", "tmem_sums"])
@pytest.mark.parametrize("engine", ENGINES)
@pytest.mark.parametrize("k", range(len(BS_CASES)))
def test_band_scales_parity(k, engine, ws):
    from mixed_precision_vit_b200.sc import ScStep
    if engine == L.SC_ENGINE_GATHER and not ws:
        pytest.skip("the gather engine takes no workspace")
    w = _band_workload(**BS_CASES[k], seed=k)
    s = ScStep(w, engine=engine, want_counts=True, use_workspace=ws)
    s.run()
    torch.cuda.synchronize()
    st, counts, out, _ = pipeline.run(w)
    assert np.array_equal(s.a_lv.cpu().numpy(), st.a_lv)
    assert np.array_equal(s.a_s.cpu().numpy(), st.a_s)
    assert np.array_equal(s.stat.cpu().numpy(), st.stat)
    assert np.array_equal(s.b_lv.cpu().numpy(), st.b_lv)
    assert np.array_equal(s.b_s.cpu().numpy(), st.b_s)
    assert np.array_equal(s.rung.cpu().numpy(), st.rung)
    assert np.array_equal(s.counts.cpu().numpy(), np.moveaxis(counts, -1, 1))
    _check_outputs(s.out.cpu().numpy(), out, f"band_scales{k}")
    assert s.dev_status.item() == 0
    s.close()


def test_band_scales_full_size_fc2_sampled():
    """The ViT-L fc2 workload (16 bands of 256) with per-band scales, on the
    default engine, at sampled outputs."""
    from mixed_precision_vit_b200.sc import ScStep
    base = W.fc2()
    w = W.Workload("fc2_band_scales", base.a, base.b, 0, base.stat_mode, base.ladder, base.tau,
                   op=base.op, n_bands=base.n_bands, chunk_d=base.chunk_d, tilt=base.tilt,
                   band_scales=True)
    s = ScStep(w, want_counts=True)
    s.run()
    torch.cuda.synchronize()
    st = pipeline.prepare(w)
    assert np.array_equal(s.a_lv.cpu().numpy(), st.a_lv)
    assert np.array_equal(s.a_s.cpu().numpy(), st.a_s)
    assert np.array_equal(s.b_s.cpu().numpy(), st.b_s)
    assert np.array_equal(s.rung.cpu().numpy(), st.rung)
    rng = np.random.default_rng(12)
    M, N = w.M, w.N
    sel = [(0, i, rng.integers(N)) for i in np.nonzero(st.rung[0] > 0)[0][:64]]
    sel += [(0, rng.integers(M), rng.integers(N)) for _ in range(600)]
    sel += [(0, i, j) for i in (0, M - 1) for j in (0, N - 1)]
    sel = np.array(sel, np.int64)
    _, counts, out, _ = pipeline.run(w, st, sel=sel)
    g, i, j = sel.T
    assert np.array_equal(s.counts.cpu().numpy()[g, :, i, j], counts)
    _check_outputs(s.out.cpu().numpy()[g, i, j], out, "fc2_band_scales")
    s.close()


def test_band_scales_guards():
    from mixed_precision_vit_b200.sc import ScTable, matmul
    dev = torch.device("cuda")
    a_lv = torch.full((1, 4, 8), 128, dtype=torch.uint8, device=dev)
    b_lv = torch.full((1, 3, 8), 128, dtype=torch.uint8, device=dev)
    rung = torch.zeros(1, 4, dtype=torch.int32, device=dev)
    perm = torch.arange(4, dtype=torch.int32, device=dev).view(1, 4)
    offs = torch.tensor([[0, 4]], dtype=torch.int32, device=dev)
    out = torch.full((1, 4, 3), 7.0, device=dev)
    plain = ScTable([64])
    with pytest.raises(L.ScError) as e:      # per-band scales without bands
        matmul(a_lv, torch.ones(1, 4, 1, device=dev), b_lv, torch.ones(1, 3, 1, device=dev), rung,
               perm, offs, plain, out=out, scales=L.SC_SCALES_BAND)
    assert e.value.code == L.SC_ERR_ARG
    banded = ScTable([64], band_len=np.array([[64], [64]], np.int32), chunk_d=4, contraction_d=8)
    with pytest.raises(L.ScError) as e:      # unknown scale mode
        matmul(a_lv, torch.ones(1, 4, 2, device=dev), b_lv, torch.ones(1, 3, 2, device=dev), rung,
               perm, offs, banded, out=out, scales=2)
    assert e.value.code == L.SC_ERR_ARG
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)             # nothing written on an error
    plain.close()
    banded.close()

"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
same seeded inputs.

Bar (from the target): integer counts bit-identical, levels / scales / rungs
bit-identical, fp32 outputs within 1e-6 relative error element by element.
The perm (rung-sorted order) is the stable sort of the rungs, which is unique.
These tests run reduced sizes (several tiles and ragged tails) and edge
cases; every output of the full-size workloads is compared in
test_gpu_full_size_parity.py.
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


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mixed_precision_vit_b200 import build
    build.build()
    oracle.build()
    L.load()


def _engine_ok(step_cls, w, engine, use_workspace=True):
    from mixed_precision_vit_b200.sc import ScStep
    s = ScStep(w, engine=engine, want_counts=True, use_workspace=use_workspace)
    try:
        s.run()
    except L.ScError as e:
        s.close()
        if e.code == L.SC_ERR_UNSUPPORTED:
            pytest.skip(f"engine {engine} unsupported here: {e}")
        raise
    torch.cuda.synchronize()
    return s


def _check_outputs(got, want, where=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    zero = want == 0
    assert np.all(got[zero] == 0), f"{where}: nonzero where oracle is exactly 0"
    rel = np.abs(got[~zero] - want[~zero]) / np.abs(want[~zero])
    assert rel.size == 0 or rel.max() <= REL_TOL, f"{where}: max rel err {rel.max():.3e}"


def _check_prepare(s, st):
    assert np.array_equal(s.a_lv.cpu().numpy(), st.a_lv)
    assert np.array_equal(s.a_s.cpu().numpy(), st.a_s)
    assert np.array_equal(s.stat.cpu().numpy(), st.stat)
    assert np.array_equal(s.b_lv.cpu().numpy(), st.b_lv)
    assert np.array_equal(s.b_s.cpu().numpy(), st.b_s)
    rung = s.rung.cpu().numpy()
    assert np.array_equal(rung, st.rung)
    perm = s.perm.cpu().numpy()
    offs = s.offs.cpu().numpy()
    n_r = len(st.ladder)
    for g in range(rung.shape[0]):
        assert np.array_equal(perm[g], np.argsort(rung[g], kind="stable"))
        hist = np.bincount(rung[g], minlength=n_r)
        assert np.array_equal(offs[g], np.concatenate([[0], np.cumsum(hist)]))


SMALL = {
    "single": lambda: W.single(),
    "qk": lambda: W.qk(groups=3),
    "av": lambda: W.av(groups=2),
    "fc1": lambda: W.fc1(tokens=300, d_in=160, d_out=200),
    "fc2": lambda: W.fc2(tokens=150, d_in=16 * 24, d_out=130),
}


@pytest.mark.parametrize("engine", ENGINES)
@pytest.mark.parametrize("name", list(SMALL))
def test_full_parity_small(name, engine):
    w = SMALL[name]()
    s = _engine_ok(None, w, engine)
    st, counts, out, steps = pipeline.run(w)
    _check_prepare(s, st)
    got_c = s.counts.cpu().numpy()                       # [batch, nb, M, N]
    assert np.array_equal(got_c, np.moveaxis(counts, -1, 1))
    _check_outputs(s.out.cpu().numpy(), out, name)
    assert steps == s.bitops()
    assert s.dev_status.item() == 0
    s.close()


@pytest.mark.parametrize("engine", ENGINES)
def test_groups_beyond_one_launch_window(engine):
    """600 groups: more (group, rung) units than one tensor-core launch takes
    (2048 / 5 rungs = 409 groups), so the engine runs two windows of both
    kernels; every output against the oracle."""
    w = W.qk(groups=600, T=33, dh=16)
    s = _engine_ok(None, w, engine)
    if engine == L.SC_ENGINE_TC:
        assert L.sc_matmul_launches(s.desc, s.table.handle) == 4
    st, counts, out, _ = pipeline.run(w)
    _check_prepare(s, st)
    assert np.array_equal(s.counts.cpu().numpy(), np.moveaxis(counts, -1, 1))
    _check_outputs(s.out.cpu().numpy(), out, "600 groups")
    s.close()


def test_band_segments_follow_the_workspace_and_are_deterministic():
    """The band kernel's segment count follows the workspace size (the
    preferred size, two slices, one slice, less than one slice: the
    tensor-memory kernel); every size matches the oracle, and each is
    bit-identical when run again."""
    from mixed_precision_vit_b200.sc import ScStep
    w = W.fc2(tokens=300, d_in=16 * 24, d_out=330)
    s = ScStep(w, engine=L.SC_ENGINE_TC, want_counts=True)
    pref = L.sc_matmul_workspace_bytes(s.desc, s.table.handle)
    slice_b = -(-(300 * 330 * 8) // 256) * 256
    st, counts, out, _ = pipeline.run(w)
    for nbytes in (pref, pref - slice_b, 2 * slice_b + (pref - (pref // slice_b) * slice_b),
                   slice_b + (pref - (pref // slice_b) * slice_b), slice_b - 8):
        ws = torch.empty(max(nbytes, 8), dtype=torch.uint8, device="cuda")
        s.desc.workspace = ws.data_ptr()
        s.desc.workspace_bytes = nbytes
        got = []
        for _ in range(2):
            s.out.fill_(7.0)
            s.run()
            torch.cuda.synchronize()
            got.append(s.out.cpu().numpy().copy())
        assert np.array_equal(got[0], got[1]), nbytes
        assert np.array_equal(s.counts.cpu().numpy(), np.moveaxis(counts, -1, 1))
        _check_outputs(got[0], out, f"workspace {nbytes}")
    s.close()


def test_workspace_bytes():
    from mixed_precision_vit_b200.sc import ScStep
    fc2 = W.fc2(tokens=150, d_in=16 * 24, d_out=130)
    s = ScStep(fc2, engine=L.SC_ENGINE_TC)
    nbytes = L.sc_matmul_workspace_bytes(s.desc, s.table.handle)
    assert nbytes >= 150 * 130 * 8                  # at least one slice of fp64 band sums
    s.desc.engine = L.SC_ENGINE_GATHER
    assert L.sc_matmul_workspace_bytes(s.desc, s.table.handle) == 0
    s.close()
    q = ScStep(W.qk(groups=2), engine=L.SC_ENGINE_TC)
    assert L.sc_matmul_workspace_bytes(q.desc, q.table.handle) == 0 and q.workspace is None
    q.close()
    # rows of 257 levels: room for both operands' levels in 272-byte rows
    a = ScStep(W.av(groups=2), engine=L.SC_ENGINE_TC)
    r256 = lambda x: (x + 255) // 256 * 256
    assert L.sc_matmul_workspace_bytes(a.desc, a.table.handle) == r256(2 * 257 * 272) + r256(2 * 64 * 272)
    a.close()


# Level rows whose length is not a multiple of 16 bytes: with a workspace the
# call copies both operands' levels into 16-byte rows first (two more
# launches) and the kernels read them aligned; without one they read the
# caller's rows.  Both paths give the oracle's counts.
PADDED = {
    "av": lambda: W.av(groups=2),
    "qk_d37": lambda: _with_width(W.qk(groups=2), 37),
    "fc1_d37": lambda: W.fc1(tokens=77, d_in=37, d_out=130, seed=9),
    "fc2_d24x17": lambda: W.fc2(tokens=150, d_in=24 * 17, d_out=130, n_bands=17),
}


def _with_width(w, D):
    assert w.b_axis == 0
    w.a = w.a[..., :D].contiguous()
    w.b = w.b[..., :D].contiguous()
    return w


@pytest.mark.parametrize("name", list(PADDED))
def test_padded_level_rows(name):
    from mixed_precision_vit_b200.sc import ScStep
    w = PADDED[name]()
    assert w.D % 16 != 0
    st, counts, out, steps = pipeline.run(w)
    want_c = np.moveaxis(counts, -1, 1)
    got = {}
    for ws in (True, False):
        s = _engine_ok(None, w, L.SC_ENGINE_TC, use_workspace=ws)
        base = L.sc_matmul_launches(s.desc, s.table.handle)
        got[ws] = s.counts.cpu().numpy()
        assert np.array_equal(got[ws], want_c), (name, ws)
        _check_outputs(s.out.cpu().numpy(), out, f"{name} workspace={ws}")
        assert s.dev_status.item() == 0
        if ws:
            s.desc.workspace, s.desc.workspace_bytes = 0, 0
            assert L.sc_matmul_launches(s.desc, s.table.handle) == base - 2
        s.close()


def _custom(M, N, D, ladder, tau=(), batch=1, seed=0, zero_rows=(), stat_mode=0, b_axis=0):
    g = torch.Generator().manual_seed(seed)
    a = torch.randn(batch, M, D, generator=g)
    b = torch.randn(batch, N, D, generator=g) if b_axis == 0 else torch.randn(batch, D, N, generator=g)
    for r in zero_rows:
        a[:, r] = 0.0
    return W.Workload("edge", a, b, b_axis, stat_mode, tuple(ladder), tuple(tau))


EDGES = [
    dict(M=1, N=1, D=1, ladder=(64,)),
    dict(M=5, N=3, D=1, ladder=(1,)),
    dict(M=7, N=9, D=3, ladder=(1, 2, 3, 255, 256), tau=(0.9, 0.7, 0.5, 0.3)),
    dict(M=129, N=257, D=65, ladder=(256,)),
    dict(M=130, N=17, D=33, ladder=(64, 96, 128, 192, 256), tau=(0.8, 0.6, 0.4, 0.2), zero_rows=(0, 5)),
    dict(M=33, N=40, D=300, ladder=(97, 131), tau=(0.5,), b_axis=1),
    dict(M=257, N=257, D=64, ladder=(64, 96, 128, 192, 256), tau=(0.8, 0.6, 0.4, 0.2), batch=2),
    # N <= 64: the one-CTA (M = 128) tensor-core kernel; rungs crossing 128-row
    # tiles, a ragged D, an N below one 32-column block
    dict(M=300, N=64, D=257, ladder=(64, 96, 128, 192, 256), tau=(0.7, 0.5, 0.3, 0.1), batch=3),
    dict(M=140, N=50, D=19, ladder=(32, 200), tau=(0.4,), batch=2, b_axis=1),
]


@pytest.mark.parametrize("engine", ENGINES)
@pytest.mark.parametrize("k", range(len(EDGES)))
def test_edge_shapes(k, engine):
    w = _custom(**EDGES[k])
    s = _engine_ok(None, w, engine)
    st, counts, out, _ = pipeline.run(w)
    _check_prepare(s, st)
    assert np.array_equal(s.counts.cpu().numpy(), np.moveaxis(counts, -1, 1))
    _check_outputs(s.out.cpu().numpy(), out, f"edge{k}")
    s.close()


BAND_EDGES = [
    # band width not a multiple of 16, one band per 7 indices, ragged row tiles
    dict(M=300, N=100, D=35, n_bands=5, chunk_d=7, tilt=0.3, ladder=(64, 96, 128, 192, 256),
         tau=(0.8, 0.6, 0.4, 0.2)),
    # two row tiles on the bottom rung, leftover rows on the others, 3 column tiles
    dict(M=600, N=230, D=64, n_bands=4, chunk_d=16, tilt=-0.2, ladder=(64, 96, 128, 192, 256),
         tau=(0.8, 0.6, 0.4, 0.2), batch=2),
    # single band, single rung
    dict(M=64, N=33, D=48, n_bands=1, chunk_d=48, tilt=0.0, ladder=(100,), tau=()),
]


@pytest.mark.parametrize("ws", [True, False], ids=["workspace_sums", "tmem_sums"])
@pytest.mark.parametrize("engine", ENGINES)
@pytest.mark.parametrize("k", range(len(BAND_EDGES)))
def test_band_edges(k, engine, ws):
    """Bands on both engines; on the tensor cores with the fp64 band sums in
    the workspace (wide tiles) and in tensor memory (no workspace)."""
    if engine == L.SC_ENGINE_GATHER and not ws:
        pytest.skip("the gather engine takes no workspace")
    e = dict(BAND_EDGES[k])
    nb, cd, tilt = e.pop("n_bands"), e.pop("chunk_d"), e.pop("tilt")
    base = _custom(**e)
    w = W.Workload("band_edge", base.a, base.b, 0, 0, base.ladder, base.tau,
                   n_bands=nb, chunk_d=cd, tilt=tilt)
    s = _engine_ok(None, w, engine, use_workspace=ws)
    if engine == L.SC_ENGINE_TC:
        assert (s.workspace is not None) == ws
    st, counts, out, _ = pipeline.run(w)
    _check_prepare(s, st)
    assert np.array_equal(s.counts.cpu().numpy(), np.moveaxis(counts, -1, 1))
    _check_outputs(s.out.cpu().numpy(), out, f"band_edge{k}")
    s.close()


def test_bands_tilt_zero_equals_parent_and_tilt_differs():
    from mixed_precision_vit_b200.sc import ScStep
    base = W.fc2(tokens=64, d_in=16 * 16, d_out=96)
    parent = W.Workload("p", base.a, base.b, 0, 0, base.ladder, base.tau)
    flat = W.Workload("t0", base.a, base.b, 0, 0, base.ladder, base.tau, n_bands=16, chunk_d=16, tilt=0.0)
    outs = []
    for w in (parent, flat, base):
        s = ScStep(w, want_counts=True)
        s.run()
        torch.cuda.synchronize()
        outs.append((s.counts.cpu().numpy(), s.out.cpu().numpy()))
        s.close()
    assert np.array_equal(outs[1][0].sum(axis=1), outs[0][0][:, 0])
    rel0 = np.linalg.norm(outs[1][1] - outs[0][1]) / np.linalg.norm(outs[0][1])
    rel1 = np.linalg.norm(outs[2][1] - outs[0][1]) / np.linalg.norm(outs[0][1])
    assert rel0 < 1e-5 and rel1 > 1e-4


def test_empty_inputs_launch_nothing():
    from mixed_precision_vit_b200.sc import ScTable
    t = ScTable([64])
    out = torch.full((1, 0, 4), 7.0, device="cuda")
    z = torch.zeros(1, 0, 8, dtype=torch.uint8, device="cuda")
    d = L.ScMatmulDesc(0, 4, 8, 1, 0, 0, 0.0)
    L.sc_matmul(d, z, z, z, z, z, z, z, t.handle, out, None, None)
    t.close()


def test_guards_reject_without_writing():
    from mixed_precision_vit_b200.sc import ScTable, kband_tilt
    lad = [64, 96, 128, 192, 256]
    bl = kband_tilt(lad, 4, 0.25, 256)
    t = ScTable(lad, 8, bl, 16, 64)
    x = torch.full((1, 8, 8), 3.0, device="cuda")
    lv = torch.full((1, 8, 64), 128, dtype=torch.uint8, device="cuda")
    sc = torch.ones(1, 8, device="cuda")
    rg = torch.zeros(1, 8, dtype=torch.int32, device="cuda")
    offs = torch.tensor([[0, 8, 8, 8, 8, 8]], dtype=torch.int32, device="cuda")
    for op, D, code in [(L.SC_OP_QK, 64, L.SC_ERR_TABLE), (L.SC_OP_AV, 64, L.SC_ERR_TABLE),
                        (L.SC_OP_LINEAR, 32, L.SC_ERR_TABLE)]:
        d = L.ScMatmulDesc(8, 8, D, 1, op, 0, 0.0)
        with pytest.raises(L.ScError) as e:
            L.sc_matmul(d, lv, sc, lv, sc, rg, rg, offs, t.handle, x, None, None)
        assert e.value.code == code
    torch.cuda.synchronize()
    assert torch.all(x == 3.0)
    t.close()


def test_nonfinite_input_sets_device_status():
    from mixed_precision_vit_b200.sc import ScStep
    w = _custom(M=8, N=8, D=16, ladder=(64,))
    w.a[0, 3, 5] = float("nan")
    s = ScStep(w)
    s.run()
    torch.cuda.synchronize()
    assert s.dev_status.item() & L.SC_DEV_NONFINITE
    s.close()


def test_deterministic_two_runs():
    from mixed_precision_vit_b200.sc import ScStep
    s = ScStep(W.qk(groups=8), want_counts=True)
    s.run()
    o1, c1 = s.out.clone(), s.counts.clone()
    s.run()
    torch.cuda.synchronize()
    assert torch.equal(o1, s.out) and torch.equal(c1, s.counts)
    s.close()


def test_launch_count_matches_engine():
    """sc_matmul_launches: one gather kernel, or the tensor-core kernel plus
    the leftover-row kernel per window of groups; a step adds the two
    quantisations and the row assignment."""
    from mixed_precision_vit_b200.sc import ScStep
    w = SMALL["qk"]()
    for engine, n_mm in ((L.SC_ENGINE_GATHER, 1), (L.SC_ENGINE_TC, 2)):
        s = ScStep(w, engine=engine)
        assert L.sc_matmul_launches(s.desc, s.table.handle) == n_mm
        assert s.launches() == 3 + n_mm
        s.close()
    d = L.ScMatmulDesc(0, 4, 8, 1, 0, 0, 0.0)
    from mixed_precision_vit_b200.sc import ScTable
    t = ScTable([64])
    assert L.sc_matmul_launches(d, t.handle) == 0
    t.close()


PREP = {
    "fc1": lambda: W.fc1(tokens=300, d_in=160, d_out=200),
    "fc1_ragged": lambda: W.fc1(tokens=77, d_in=37, d_out=130, seed=9),
    "fc2": lambda: W.fc2(tokens=150, d_in=16 * 24, d_out=330),
    "fc2_bs": lambda: W.fc2_bs(tokens=150, d_in=16 * 24, d_out=130),
    "fc1_uni": lambda: _unipolar(W.fc1(tokens=300, d_in=160, d_out=200)),
    "fc2_uni": lambda: _unipolar(W.fc2(tokens=150, d_in=16 * 24, d_out=130)),
    "qk": lambda: W.qk(groups=3),
}


def _unipolar(w):
    w.unipolar = True
    return w


@pytest.mark.parametrize("name", list(PREP))
def test_prepared_second_operand(name):
    """sc_prepare_b: the B stages written once in the kernel's shared-memory
    layout and copied by the tensor-core kernel give the oracle's counts and
    outputs, on every wide-tile layout (no bands, bands with workspace sums,
    per-band scales, the unipolar mode, a batch of groups), two runs in a row."""
    from mixed_precision_vit_b200.sc import ScStep
    w = PREP[name]()
    s = ScStep(w, engine=L.SC_ENGINE_TC, want_counts=True, prepare_b=True)
    assert s.b_prep
    st, counts, out, _ = pipeline.run(w)
    for _ in range(2):
        s.out.fill_(7.0)
        s.run()
        torch.cuda.synchronize()
        _check_prepare(s, st)
        assert np.array_equal(s.counts.cpu().numpy(), np.moveaxis(counts, -1, 1))
        _check_outputs(s.out.cpu().numpy(), out, f"prepared {name}")
        assert s.dev_status.item() == 0
    s.close()


def test_prepared_operand_rejections():
    """Problems that run another kernel cannot be prepared, and a prepared
    operand is refused by a problem or table it was not made for."""
    from mixed_precision_vit_b200.sc import ScStep
    for w, kw in ((W.av(groups=2), {}),                                   # N <= 64: one-CTA kernel
                  (W.fc2(tokens=150, d_in=16 * 24, d_out=130), dict(use_workspace=False))):
        with pytest.raises(L.ScError) as e:
            ScStep(w, engine=L.SC_ENGINE_TC, prepare_b=True, **kw)
        assert e.value.code == L.SC_ERR_UNSUPPORTED
    a = ScStep(W.fc1(tokens=100, d_in=64, d_out=130), engine=L.SC_ENGINE_TC, prepare_b=True)
    b = ScStep(W.fc1(tokens=100, d_in=64, d_out=200), engine=L.SC_ENGINE_TC)
    b.desc.b_prep = a.b_prep                       # made for N = 130, used with N = 200
    with pytest.raises(L.ScError) as e:
        b.run()
    assert e.value.code == L.SC_ERR_ARG
    b.desc.b_prep = None
    a.close()
    b.close()


def test_bounded_wait_reports_its_expiry():
    """The pipeline barriers' bounded wait, alone, on a barrier nothing
    arrives at with a limit of about a millisecond: the kernel returns, the
    status word carries SC_DEV_WAIT_LIMIT, and the context still runs work."""
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.sc_selftest_wait_limit(status, 2_000_000)
    torch.cuda.synchronize()
    assert status.item() & L.SC_DEV_WAIT_LIMIT
    with pytest.raises(L.ScError):
        L.sc_selftest_wait_limit(status, 0)
    x = torch.ones(8, device="cuda")
    assert float((x * 2).sum()) == 16.0


@pytest.mark.parametrize("prep", [False, True])
def test_host_pipeline_matches_the_step(prep):
    """HostPipeline (uploads, compute and downloads of neighbouring steps
    overlapped on three streams) returns exactly the output of a plain step,
    with and without a prepared second operand."""
    from mixed_precision_vit_b200.sc import HostPipeline, ScStep
    w = W.fc1(tokens=300, d_in=160, d_out=200)
    s = ScStep(w, engine=L.SC_ENGINE_TC, prepare_b=prep)
    s.run()
    torch.cuda.synchronize()
    want = s.out.cpu()
    out_h = torch.full(tuple(s.out.shape), 7.0).pin_memory()
    pipe = HostPipeline(s)
    st, en = pipe.run(w.a.pin_memory(), w.b.pin_memory(), out_h, 5)
    torch.cuda.synchronize()
    assert torch.equal(out_h, want)
    assert st.elapsed_time(en) > 0
    h2d, d2h = pipe.bytes_per_step()
    assert h2d == w.a.numel() * 4 + (0 if prep else w.b.numel() * 4) and d2h == want.numel() * 4
    s.close()


# Per-row quantisation of long rows: every kernel width class (rows that fit
# a warp's registers, four-wide rows of up to 512, one block per row of
# 513..8192 floats, and the scalar two-pass kernel beyond), batched, with
# both row statistics, against the oracle bit for bit.
@pytest.mark.parametrize("cols", [260, 512, 516, 1024, 2052, 4096, 8192, 8196])
def test_quantize_rows_every_width(cols):
    from mixed_precision_vit_b200.sc import quantize
    g = torch.Generator().manual_seed(cols)
    x = torch.randn(3, 37, cols, generator=g) * torch.rand(3, 37, 1, generator=g) * 5
    x[1, 4] = 0.0                                   # a zero row
    x[2, 7, cols // 3] = 1e4                         # an outlier
    for mode in (L.SC_STAT_AMAX, L.SC_STAT_ROWMAX):
        lv, sc, st = quantize(x.cuda(), axis=0, stat_mode=mode, want_stat=True)
        torch.cuda.synchronize()
        for b in range(3):
            want_lv, want_sc = oracle.quantize(x[b].numpy(), axis=0)
            assert np.array_equal(lv[b].cpu().numpy(), want_lv), (cols, mode, b)
            assert np.array_equal(sc[b].cpu().numpy(), want_sc), (cols, mode, b)
            assert np.array_equal(st[b].cpu().numpy(), oracle.row_stat(x[b].numpy(), mode)), (cols, mode, b)


# Per-column quantisation (transposed levels): columns short enough for the
# register kernel (rows <= 320) and longer ones, ragged column blocks.
@pytest.mark.parametrize("rows,cols", [(1, 5), (7, 64), (257, 64), (320, 33), (321, 64), (600, 100)])
def test_quantize_cols_every_height(rows, cols):
    from mixed_precision_vit_b200.sc import quantize
    g = torch.Generator().manual_seed(rows * 1000 + cols)
    x = torch.randn(3, rows, cols, generator=g) * torch.rand(3, 1, cols, generator=g) * 4
    x[0, :, cols // 2] = 0.0                         # a zero column
    lv, sc, _ = quantize(x.cuda(), axis=1)
    torch.cuda.synchronize()
    for b in range(3):
        want_lv, want_sc = oracle.quantize(x[b].numpy(), axis=1)
        assert np.array_equal(lv[b].cpu().numpy(), want_lv), (rows, cols, b)
        assert np.array_equal(sc[b].cpu().numpy(), want_sc), (rows, cols, b)

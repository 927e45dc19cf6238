"""GPU tests of sc_matmul_static_ws, the entry point that uses the library's
static scratch buffer in place of a caller workspace, for callers that cannot
allocate device memory themselves (code inside a framework that owns every
device allocation, or a process that must not grow after start-up).  Kept in
its own file, collected last, because the buffer is shared by every call on
the device and keeps the last call's contents.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import pipeline
from mixed_precision_vit_b200 import _lib as L
from mixed_precision_vit_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mixed_precision_vit_b200 import build
    build.build()
    oracle.build()
    L.load()


def _run_static(s, out, counts):
    d = L.ScMatmulDesc(s.desc.M, s.desc.N, s.desc.D, s.desc.batch, s.desc.op, s.desc.engine,
                       s.desc.q_dec, s.desc.scales, 0, None, 0)
    L.sc_matmul_static_ws(d, s.a_lv, s.a_s, s.b_lv, s.b_s, s.rung, s.perm, s.offs, s.table.handle,
                          out, counts, s.dev_status)


# fc2 / fc2_bs: band sums in the buffer; av and fc2_odd (widths 257 and 408,
# not multiples of 16): the levels copied into 16-byte rows there too
@pytest.mark.parametrize("name", ["fc2", "fc2_bs", "qk", "av", "fc2_odd"])
def test_static_scratch_equals_caller_workspace_and_oracle(name):
    from mixed_precision_vit_b200.sc import ScStep
    w = {"fc2": lambda: W.fc2(tokens=150, d_in=16 * 24, d_out=130),
         "fc2_bs": lambda: W.fc2_bs(tokens=150, d_in=16 * 24, d_out=130),
         "qk": lambda: W.qk(groups=3),
         "av": lambda: W.av(groups=2),
         "fc2_odd": lambda: W.fc2(tokens=150, d_in=24 * 17, d_out=130, n_bands=17)}[name]()
    s = ScStep(w, engine=L.SC_ENGINE_TC, want_counts=True)
    s.run()
    # two calls in a row: the second finds the first one's leftovers in the
    # shared buffer and must give the same result
    for _ in range(2):
        out = torch.full_like(s.out, 7.0)
        counts = torch.full_like(s.counts, -1)
        _run_static(s, out, counts)
        torch.cuda.synchronize()
        assert torch.equal(out, s.out) and torch.equal(counts, s.counts)
    _, want_c, want_o, _ = pipeline.run(w)
    assert np.array_equal(counts.cpu().numpy(), np.moveaxis(want_c, -1, 1))
    got = out.cpu().numpy().astype(np.float64)
    nz = want_o != 0
    assert np.all(got[~nz] == 0)
    assert np.max(np.abs(got[nz] - want_o[nz]) / np.abs(want_o[nz])) <= 1e-6
    s.close()


def test_static_scratch_rejects_oversize_and_a_named_workspace():
    from mixed_precision_vit_b200.sc import ScTable
    dev = torch.device("cuda")
    M, N, D = 4112, 4096, 32                  # 4112 x 4096 x 8 B of sums > 64 MiB
    assert M * N * 8 > L.SC_STATIC_WS_BYTES
    table = ScTable([64], band_len=np.array([[64], [64]], np.int32), chunk_d=16, contraction_d=D)
    a_lv = torch.full((1, M, D), 128, dtype=torch.uint8, device=dev)
    b_lv = torch.full((1, N, D), 128, dtype=torch.uint8, device=dev)
    a_s = torch.ones(1, M, device=dev)
    b_s = torch.ones(1, N, device=dev)
    rung = torch.zeros(1, M, dtype=torch.int32, device=dev)
    perm = torch.arange(M, dtype=torch.int32, device=dev).view(1, M)
    offs = torch.tensor([[0, M]], dtype=torch.int32, device=dev)
    out = torch.full((1, M, N), 7.0, device=dev)
    d = L.ScMatmulDesc(M, N, D, 1, L.SC_OP_LINEAR, L.SC_ENGINE_TC, 0.0, 0, 0, None, 0)
    with pytest.raises(L.ScError) as e:
        L.sc_matmul_static_ws(d, a_lv, a_s, b_lv, b_s, rung, perm, offs, table.handle, out, None,
                              None)
    assert e.value.code == L.SC_ERR_UNSUPPORTED
    ws = torch.empty(16, dtype=torch.uint8, device=dev)
    d2 = L.ScMatmulDesc(8, 8, D, 1, L.SC_OP_LINEAR, L.SC_ENGINE_TC, 0.0, 0, 0, ws.data_ptr(), 16)
    with pytest.raises(L.ScError) as e:
        L.sc_matmul_static_ws(d2, a_lv, a_s, b_lv, b_s, rung, perm, offs, table.handle, out, None,
                              None)
    assert e.value.code == L.SC_ERR_ARG
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)               # nothing enqueued on a rejected call
    table.close()

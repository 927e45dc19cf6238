"""The N>1 bench path on CPU: two gloo ranks, each with its own batch of
independent groups; times reduce by max, work by sum; no data-path
collective.  Also checks that the per-rank inputs differ and the oracle
results of the ranks are independent of each other."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    from mixed_precision_vit_b200 import workloads as W
    w = W.qk(seed=bench.rank_seed("qk", rank), groups=2, T=17, dh=8)
    bits = 1000 * (rank + 1)
    t = 10.0 + rank
    res = bench.combine_ranks(t, 2 * t, 0.5 * t, bits, torch.device("cpu"))
    q.put((rank, res, float(w.a.sum())))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    for _, res, _ in out:
        assert res == (11.0, 22.0, 5.5, 3000.0)
    assert out[0][2] != out[1][2]           # each rank draws its own groups


def test_single_process_combine_is_identity():
    import bench
    assert bench.combine_ranks(1.0, 2.0, 3.0, 7, torch.device("cpu")) == (1.0, 2.0, 3.0, 7.0)

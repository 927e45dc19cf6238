"""The N>1 path on CPU: two gloo ranks.

Data parallelism here is weak scaling with no data-path collective: every
rank runs a whole problem of its own (its own (batch, head) groups for the
attention workloads; its own token batch against the replicated weight for
the linear layers), and only the timings (max) and the work (sum) are
reduced.  These tests run each rank's shard through the oracle and check that
the shards partition the job as claimed: for attention, the union of the two
ranks' results is, group by group, the single-process result of the
concatenated groups (nothing couples groups); for a linear layer, the ranks
hold the same weight and different tokens, and each rank's result is the
single-process result of its own tokens.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

SMALL = {"qk": dict(groups=2, T=17, dh=8), "fc2": dict(tokens=20, d_in=16 * 4, d_out=12)}


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
    import oracle
    from oracle import pipeline
    from mixed_precision_vit_b200 import workloads as W
    oracle.build()
    res = {}
    for name, kw in SMALL.items():
        w = W.shard(name, rank, **kw)
        _, counts, out, steps = pipeline.run(w, n_threads=1)
        res[name] = (w.a.numpy(), w.b.numpy(), counts, out, steps)
    # the bench's reduction: times by max, work by sum over ranks
    bits = sum(r[4] for r in res.values())
    t = 10.0 + rank
    red = bench.combine_ranks(t, 2 * t, 0.5 * t, bits, torch.device("cpu"))
    gathered = [None] * world
    dist.all_gather_object(gathered, res)
    q.put((rank, red, bits, gathered if rank == 0 else None))
    dist.barrier()
    dist.destroy_process_group()


@pytest.fixture(scope="module")
def two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort(key=lambda x: x[0])
    return out


def test_reduction_is_max_time_and_summed_work(two_ranks):
    bits = [r[2] for r in two_ranks]
    for _, red, _, _ in two_ranks:
        assert red == (11.0, 22.0, 5.5, float(sum(bits)))


def test_attention_shards_union_is_the_single_process_result(two_ranks):
    import dataclasses

    from oracle import pipeline
    from mixed_precision_vit_b200 import workloads as W
    shards = two_ranks[0][3]
    a = np.concatenate([s["qk"][0] for s in shards])
    b = np.concatenate([s["qk"][1] for s in shards])
    assert not np.array_equal(shards[0]["qk"][0], shards[1]["qk"][0])   # own groups per rank
    w = dataclasses.replace(W.qk(**SMALL["qk"]), a=torch.from_numpy(a), b=torch.from_numpy(b))
    _, counts, out, steps = pipeline.run(w)
    assert np.array_equal(counts, np.concatenate([s["qk"][2] for s in shards]))
    assert np.array_equal(out, np.concatenate([s["qk"][3] for s in shards]))
    assert steps == sum(s["qk"][4] for s in shards)


def test_linear_shards_share_the_weight_and_keep_their_tokens(two_ranks):
    import dataclasses

    from oracle import pipeline
    from mixed_precision_vit_b200 import workloads as W
    shards = two_ranks[0][3]
    w0 = W.fc2(**SMALL["fc2"])
    assert np.array_equal(shards[0]["fc2"][1], shards[1]["fc2"][1])      # replicated W
    assert np.array_equal(shards[0]["fc2"][1], w0.b.numpy())
    assert not np.array_equal(shards[0]["fc2"][0], shards[1]["fc2"][0])  # own tokens
    for s in shards:
        w = dataclasses.replace(w0, a=torch.from_numpy(s["fc2"][0]))
        _, counts, out, _ = pipeline.run(w)
        assert np.array_equal(counts, s["fc2"][2])
        assert np.array_equal(out, s["fc2"][3])


def test_single_process_combine_is_identity():
    import bench
    assert bench.combine_ranks(1.0, 2.0, 3.0, 7, torch.device("cpu")) == (1.0, 2.0, 3.0, 7.0)

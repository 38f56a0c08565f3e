"""The multi-process path of the benchmark, on CPU with gloo and two ranks.

Self-attention over (b, h) pairs has no cross-pair term, so the path shards
without a data-path collective: every rank runs its own independent call
(weak scaling, each rank with its own seeded batch element) and the only
collectives are the barrier and the max-over-ranks of the timings.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist

    import bench
    import synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # max over ranks of a per-rank time
        got = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        # per-rank workloads differ only by seed
        w = bench.rank_workload(synth.WORKLOADS["tiny"], rank)
        q, _, _ = synth.qkv_numpy(w)
        digest = torch.tensor([float(q[0, 0, :4, :4].astype("int64").sum())], dtype=torch.float64)
        allq = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(allq, digest)
        dist.barrier()
        out[rank] = (got, w.seed, [float(x.item()) for x in allq])
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_gloo_max_and_independent_shards():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
        assert p.exitcode == 0
    assert out[0][0] == out[1][0] == 15.0
    assert (out[0][1], out[1][1]) == (0, 1)
    digests = out[0][2]
    assert digests == out[1][2] and digests[0] != digests[1]


def test_single_rank_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5

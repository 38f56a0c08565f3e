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


def _ulysses_rank(rank, world, port, result_q):
    import os

    import numpy as np
    import torch
    import torch.distributed as dist

    import synth
    from _util import attention_per_head_ref, attention_seqpar_ref, ulysses_ref_permute
    from video_dit_quantized_b200 import sage
    from video_dit_quantized_b200.ulysses import UlyssesAttention

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = synth.Workload("uly", 1, 4, 96, 16, seed=3)
        full = [torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) for a in synth.qkv_numpy(w)]
        # [B, H, N, d] -> the sequence-parallel layout [B, N, H, d], this rank's token slice
        Nl = w.N // world
        mine = [t.permute(0, 2, 1, 3)[:, rank * Nl:(rank + 1) * Nl].contiguous() for t in full]

        def a2a(out, inp):
            return dist.all_to_all_single(out, inp, async_op=True)

        ua = UlyssesAttention(w.B, Nl, w.H, w.d, world, mode=sage.MODE_BF16, device="cpu",
                              permute=ulysses_ref_permute, attention=attention_seqpar_ref, a2a=a2a)
        ua.send("q", mine[0])          # q goes out before k and v exist, as a DiT block would issue it
        ua.send("k", mine[1])
        ua.send("v", mine[2])
        out = ua.attend()
        ref = attention_per_head_ref(*full, sage.MODE_BF16, torch.empty_like(full[0]))
        want = ref.permute(0, 2, 1, 3)[:, rank * Nl:(rank + 1) * Nl]
        result_q.put((rank, bool(torch.equal(out.view(torch.int16), want.contiguous().view(torch.int16)))))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_ulysses_exchange_gloo_ranks(world):
    """Two or four CPU ranks run the Ulysses exchange around a per-head reference attention; each
    rank's output slice equals single-process attention on the whole sequence, bit for bit."""
    import multiprocessing as mp
    import socket

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_ulysses_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    results = dict(q.get(timeout=5) for _ in range(world))
    assert results == {r: True for r in range(world)}


def test_ulysses_host_checks():
    """UlyssesAttention refuses what the exchange cannot do, on the host (no GPU, no process group)."""
    import torch

    from _util import attention_per_head_ref, attention_seqpar_ref, ulysses_ref_permute
    from video_dit_quantized_b200 import sage
    from video_dit_quantized_b200.ulysses import UlyssesAttention

    with pytest.raises(ValueError):
        UlyssesAttention(1, 8, 6, 16, 4, device="cpu", permute=ulysses_ref_permute,
                         attention=attention_seqpar_ref, a2a=lambda o, i: None)        # 6 heads over 4 ranks
    sent = []

    def a2a(out, inp):
        sent.append(inp.shape)
        out.copy_(inp)
        return None

    ua = UlyssesAttention(1, 8, 4, 16, 1, mode=sage.MODE_BF16, device="cpu", permute=ulysses_ref_permute,
                          attention=attention_seqpar_ref, a2a=a2a)
    x = torch.randn(1, 8, 4, 16).to(torch.bfloat16)
    with pytest.raises(ValueError):
        ua.send("q", torch.randn(1, 8, 2, 16).to(torch.bfloat16))                    # wrong shape
    with pytest.raises(ValueError):
        ua.send("x", x)
    ua.send("q", x)
    with pytest.raises(RuntimeError):
        ua.attend()                                                                  # k and v not sent
    ua.send("k", x)
    ua.send("v", x)
    out = ua.attend()
    ref = attention_per_head_ref(*(x.permute(0, 2, 1, 3),) * 3, sage.MODE_BF16,
                                 torch.empty(1, 4, 8, 16, dtype=torch.bfloat16))
    assert torch.equal(out.view(torch.int16), ref.permute(0, 2, 1, 3).contiguous().view(torch.int16))
    assert sent == []                      # one rank: the exchange is the identity and no collective runs

"""Multi-rank host logic on CPU: two gloo ranks (127.0.0.1).

The data path shards with no exchange, so what needs checking across ranks is
the bookkeeping: the round-robin sharding of independent units covers every
unit exactly once, and the timing reduction takes the maximum over ranks."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from w4a4_post_quantization_dual_b200 import dist
    r, w, _ = dist.init("gloo", timeout_s=60)
    try:
        mine = dist.shard(224, r, w)                  # the 224-weight sweep
        gathered = [None] * w
        torch.distributed.all_gather_object(gathered, mine)
        times = dist.max_over_ranks([1.0 + r, 5.0 - r])
        dist.barrier()
        q.put((r, gathered, times))
    finally:
        dist.finalize()


def test_two_gloo_ranks_shard_and_reduce():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, gathered, times in results:
        units = sorted(u for part in gathered for u in part)
        assert units == list(range(224))                     # complete, no duplicates
        assert set(gathered[0]).isdisjoint(gathered[1])
        assert times == [2.0, 5.0]                           # max over ranks, element-wise


def test_single_rank_defaults():
    from w4a4_post_quantization_dual_b200 import dist
    assert dist.shard(5, 0, 1) == [0, 1, 2, 3, 4]
    assert dist.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]

"""Multi-rank host logic on CPU: two gloo ranks (127.0.0.1).

The data path shards with no exchange, so what needs checking across ranks is
the bookkeeping: the round-robin sharding of independent units covers every
unit exactly once, the timing reduction takes the maximum over ranks, and the
whole-model sweep driver partitions the 224 linears of a Llama-3.1-8B-shaped
model over the ranks and gathers every weight's result exactly once."""
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


def _sweep_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from w4a4_post_quantization_dual_b200 import dist, sweep
    r, w, _ = dist.init("gloo", timeout_s=60)
    try:
        lin = sweep.llama8b_linears()
        # a stand-in for the GPU solve: the weight's index and shape, tagged
        # with the rank that handled it
        local = sweep.run(lin, make_weight=lambda i: (i, lin[i][1], lin[i][2]),
                          solve=lambda ws: [{"index": i, "shape": [m, n], "rank": r}
                                            for i, m, n in ws], rank=r, world=w)
        merged = sweep.gather(local, r, w)
        q.put((r, sorted(local), merged))
    finally:
        dist.finalize()


def test_sweep_partitions_and_gathers_over_two_gloo_ranks():
    from w4a4_post_quantization_dual_b200 import sweep
    lin = sweep.llama8b_linears()
    assert len(lin) == 224 and len({n for n, _, _ in lin}) == 224
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sweep_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    locals_ = {r: names for r, names, _ in results}
    assert set(locals_[0]).isdisjoint(locals_[1])
    assert len(locals_[0]) == len(locals_[1]) == 112
    for r, _, merged in results:
        assert sorted(merged) == sorted(n for n, _, _ in lin)
        for i, (name, m, n) in enumerate(lin):
            assert merged[name] == {"index": i, "shape": [m, n], "rank": i % 2}


def test_single_rank_defaults():
    from w4a4_post_quantization_dual_b200 import dist
    assert dist.shard(5, 0, 1) == [0, 1, 2, 3, 4]
    assert dist.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]

"""Multi-rank host logic on CPU (gloo, world size 2): sharding of independent
layers across ranks and the max-over-ranks timing reduction used by bench.py."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from w4a16_gemm_wq_b200 import dist as wqdist
from w4a16_gemm_wq_b200 import synth


def test_shard_range_covers_exactly_once():
    for n in (0, 1, 7, 12, 504):
        for world in (1, 2, 3, 8):
            seen = []
            for r in range(world):
                rg = wqdist.shard_range(n, world, r)
                seen.extend(rg)
                assert len(rg) in (n // world, n // world + 1)
            assert seen == list(range(n))
    with pytest.raises(ValueError):
        wqdist.shard_range(4, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, lr = wqdist.dist_env()
        assert (w, r, lr) == (world, rank, rank)
        # config-5 style sharding of the 504 Linears: disjoint, complete
        n = synth.N_LAYERS * synth.LINEARS_PER_LAYER
        mine = list(wqdist.shard_range(n, world, rank))
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        flat = sorted(i for part in gathered for i in part)
        # timing reduction: every rank reports its own time, the job time is the max
        t = wqdist.max_over_ranks([1.0 + rank, 5.0 - rank])
        b = wqdist.sum_over_ranks([len(mine)])
        dist.barrier()
        q.put((rank, flat == list(range(n)), t, b))
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_sharding_and_max_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, complete, t, b in res:
        assert complete
        assert t == [2.0, 5.0]
        assert b == [504.0]

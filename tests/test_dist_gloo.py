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


def _worker_paths(rank, world, port, q):
    # The two shardings of the path, on the oracle (CPU) with a gloo group:
    #  (i) independent matrices quantized on their ranks: the union of the ranks'
    #      packs is the single-process list of packs, and the byte totals add up;
    #  (ii) one Linear split along N: each rank's pack of its rows is those rows of the
    #      full pack, and the all-gathered N-split product is the full product.
    import hashlib

    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle
    from w4a16_gemm_wq_b200 import PackedInt4

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        shapes = [(64 + 8 * i, 256 if i % 3 else 512) for i in range(11)]  # 11 small matrices (N, K)

        def pack_digest(i):
            N, K = shapes[i]
            W = synth.weight(N, K, seed=900 + i)
            p = oracle.quantize_int4(W, 64)
            h = hashlib.sha256(p["qweight"].tobytes() + p["scales"].tobytes() + p["zeros"].tobytes()).hexdigest()
            return h, p["qweight"].nbytes + p["scales"].nbytes + p["zeros"].nbytes

        mine = {i: pack_digest(i) for i in wqdist.shard_range(len(shapes), world, rank)}
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        union = {k: v for part in gathered for k, v in part.items()}
        total = wqdist.sum_over_ranks([sum(b for _, b in mine.values())])[0]
        ok_i = union == {i: pack_digest(i) for i in range(len(shapes))} and total == sum(
            b for _, b in union.values())

        N, K, M = 201, 256, 5
        W = synth.weight(N, K, seed=31)
        X = synth.activations(M, K, seed=32)
        full = oracle.quantize_int4(W, 64)
        rows = wqdist.shard_range(N, world, rank)
        part = oracle.quantize_int4(W[rows.start:rows.stop], 64)
        as_t = lambda a: torch.from_numpy(a.view(np.int32).copy())
        fullp = PackedInt4(as_t(full["qweight"]), torch.from_numpy(full["scales"].view(np.int16).copy()),
                           as_t(full["zeros"]), N, K, 64, 1)
        sh = wqdist.shard_rows(fullp, rows)
        ok_rows = (np.array_equal(part["qweight"], sh.qweight.numpy().view(np.uint32))
                   and np.array_equal(part["scales"], sh.scales.numpy().view(np.uint16))
                   and np.array_equal(part["zeros"], sh.zeros.numpy().view(np.uint32)) and sh.N == len(rows))
        local = lambda x: torch.from_numpy(oracle.linear(x, oracle.dequant_int4(part)))
        Y = wqdist.column_parallel_linear(X, local, N, world, rank)
        ok_y = np.array_equal(Y.numpy(), oracle.linear(X, oracle.dequant_int4(full)))
        dist.barrier()
        q.put((rank, ok_i, ok_rows, ok_y))
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_sharded_quantize_and_column_parallel_linear():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_paths, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok_i, ok_rows, ok_y in res:
        assert ok_i, f"rank {rank}: sharded packs differ from the single-process packs"
        assert ok_rows, f"rank {rank}: row shard of the pack differs from the pack of the rows"
        assert ok_y, f"rank {rank}: gathered N-split product differs from the full product"

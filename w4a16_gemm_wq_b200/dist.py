"""Host-side helpers for running the library on several GPUs (one process per GPU).

Two shardings of the path:
  * independent problems -- the layers of a decode sweep, or the matrices of a
    model being quantized -- split across ranks, each rank running its own
    share with no data-path collective; what crosses ranks is timing (barrier +
    max over ranks) and bookkeeping (byte totals);
  * one quantized Linear split along its N output channels (column parallel):
    rank r holds rows shard_range(N, world, r) of the packed weight, X is
    replicated, and one all-gather assembles Y [M, N] (NCCL over NVLink on
    GPUs; the library's kernels only ever read this GPU's memory).
"""
from __future__ import annotations

import os


def dist_env() -> tuple[int, int, int]:
    """(world_size, rank, local_rank) from the torchrun environment (1, 0, 0 without it)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def shard_range(n_units: int, world: int, rank: int) -> range:
    """Contiguous, balanced share of n_units for `rank` (sizes differ by at most one)."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(n_units, world)
    lo = rank * base + min(rank, extra)
    return range(lo, lo + base + (1 if rank < extra else 0))


def max_over_ranks(values, device="cpu"):
    """Element-wise max of a list of floats over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def sum_over_ranks(values, device="cpu"):
    """Element-wise sum of a list of numbers over all ranks."""
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return t.tolist()


def shard_rows(pack, rows: range):
    """The rows [rows.start, rows.stop) of a packed weight (PackedInt4 / PackedNVFP4):
    rows are quantized independently, so this is the pack of those rows of W.  The
    NVFP4 per-tensor scale stays the whole tensor's."""
    import dataclasses

    from w4a16_gemm_wq_b200 import PackedInt4

    sl = slice(rows.start, rows.stop)
    n = rows.stop - rows.start
    if isinstance(pack, PackedInt4):
        return dataclasses.replace(pack, qweight=pack.qweight[sl].contiguous(), scales=pack.scales[sl].contiguous(),
                                   zeros=None if pack.zeros is None else pack.zeros[sl].contiguous(), N=n)
    return dataclasses.replace(pack, codes=pack.codes[sl].contiguous(), bscale=pack.bscale[sl].contiguous(), N=n)


def column_parallel_linear(X, local_linear, N: int, world: int, rank: int, group=None):
    """Y = X W^T with W's N output channels split over the ranks (rank r holds rows
    shard_range(N, world, r) of the packed weight): this rank computes its columns with
    local_linear(X) -> [M, n_r], and one all-gather over the process group assembles the
    full Y [M, N] on every rank.  X is replicated.  Shards of unequal size travel padded
    to the largest one."""
    import torch
    import torch.distributed as dist

    sizes = [len(shard_range(N, world, r)) for r in range(world)]
    y = local_linear(X)
    M = y.shape[0]
    if y.shape != (M, sizes[rank]):
        raise ValueError(f"local_linear returned {tuple(y.shape)}, expected ({M}, {sizes[rank]})")
    nmax = max(sizes)
    if sizes[rank] != nmax:
        y = torch.nn.functional.pad(y, (0, nmax - sizes[rank]))
    parts = [torch.empty((M, nmax), dtype=y.dtype, device=y.device) for _ in range(world)]
    dist.all_gather(parts, y.contiguous(), group=group)
    return torch.cat([p[:, :sizes[r]] for r, p in enumerate(parts)], dim=1)

"""Row sharding across processes (one process per GPU).

Cross-entropy rows are independent: the loss, lse and gradient of row i depend
on row i alone (Ineshin, "A fused linear cross-entropy forward kernel for
Apple GPUs", section 1 computes each row's log-sum-exp by itself). A
data-parallel batch is therefore split into contiguous blocks of rows, one
block per rank, and the kernels run on each block with no exchange of data.

The one quantity that crosses ranks is the denominator of a mean over the
global batch: with ignore_index, the number of counted rows differs between
blocks, so every rank needs the global count to scale its upstream gradient
(g = 1 / count). That is one all-reduce of a single integer per batch, made
when the batch is formed, before any kernel runs.

These helpers are host logic over ``torch.distributed``; they run on any
backend (NCCL on GPUs, gloo on CPU) and never touch the logits.
"""
from __future__ import annotations

import datetime
import os
from dataclasses import dataclass
from typing import Optional, Tuple


@dataclass(frozen=True)
class Rank:
    """This process's place in the job, as the launcher's environment gives it."""
    rank: int
    world: int
    local: int
    group: Optional[object]  # torch.distributed when world > 1, else None
    device: object           # torch.device the collectives' tensors live on


def shard_bounds(n: int, rank: int, world: int) -> Tuple[int, int]:
    """Rows [start, stop) of rank `rank` when n rows are split into `world`
    contiguous blocks whose sizes differ by at most one (the first n % world
    blocks take the extra row). Blocks are disjoint and cover [0, n)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world {world}")
    if n < 0:
        raise ValueError(f"negative row count {n}")
    q, r = divmod(n, world)
    start = rank * q + min(rank, r)
    return start, start + q + (1 if rank < r else 0)


def init_from_env(backend: str = "nccl", timeout_s: float = 120.0) -> Rank:
    """Joins the process group the launcher (torchrun) describes in RANK,
    WORLD_SIZE, LOCAL_RANK and MASTER_ADDR/PORT. A single process (no
    WORLD_SIZE, or 1) gets no group. With NCCL the process binds its GPU
    before the group is created; the short timeout turns a rank that never
    arrives into an error instead of a wait without end."""
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if backend == "nccl":
        device = torch.device("cuda", local)
        torch.cuda.set_device(local)
    else:
        device = torch.device("cpu")
    if world == 1:
        return Rank(rank, 1, local, None, device)
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if backend == "nccl":
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)
    return Rank(dist.get_rank(), dist.get_world_size(), local, dist, device)


def barrier(rk: Rank) -> None:
    if rk.group is not None:
        rk.group.barrier()


def _all_reduce(rk: Rank, value, dtype, op: str):
    import torch
    t = torch.tensor([value], dtype=dtype, device=rk.device)
    if rk.group is not None:
        rk.group.all_reduce(t, op=getattr(rk.group.ReduceOp, op))
    return t.item()


def max_over_ranks(rk: Rank, x: float) -> float:
    """The largest of every rank's x (a job is as slow as its slowest rank)."""
    import torch
    return float(_all_reduce(rk, float(x), torch.float64, "MAX"))


def global_count(rk: Rank, local_count: int) -> int:
    """Sum of every rank's count (exact, int64)."""
    import torch
    return int(_all_reduce(rk, int(local_count), torch.int64, "SUM"))


def counted_rows(targets, ignore_index: int = -100) -> int:
    """Rows whose target is not ignore_index (they enter a mean)."""
    return int((targets != ignore_index).sum())


def mean_grad_scale(rk: Rank, targets, ignore_index: int = -100) -> float:
    """Upstream gradient of a mean over the global batch: 1 / (rows counted on
    all ranks), or 0 when no row anywhere is counted (the mean of nothing
    contributes no gradient)."""
    n = global_count(rk, counted_rows(targets, ignore_index))
    return 1.0 / n if n > 0 else 0.0

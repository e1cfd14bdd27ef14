"""Row sharding across ranks, on CPU: world-size-2 gloo process groups.

The kernels run per rank on a block of rows with no exchange of data; what
the ranks share is host logic (the block bounds, the global count behind a
mean, the barrier and max-over-ranks timing). These tests run that logic
in two real processes and check, with the float64 oracle as the per-rank
compute, that the sharded job gives the single-process answer."""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from softmax_cross_entropy_lse_b200 import sharding
from softmax_cross_entropy_lse_b200 import workloads as wl

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank: int, world: int, port: int) -> None:
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})


def _run(fn, *args, world=WORLD):
    mp.start_processes(fn, args=(world, _free_port()) + args, nprocs=world, join=True,
                       start_method="spawn")


# -- pure host logic ---------------------------------------------------------------------------
@pytest.mark.parametrize("n", [0, 1, 2, 3, 7, 1000, 1001, (1 << 27) + (1 << 20)])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_shard_bounds_partition(n, world):
    spans = [sharding.shard_bounds(n, r, world) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == n
    for (a, b), (c, _) in zip(spans, spans[1:]):
        assert b == c  # contiguous, disjoint
    sizes = [b - a for a, b in spans]
    assert min(sizes) >= 0 and max(sizes) - min(sizes) <= 1


def test_shard_bounds_rejects():
    for bad in [(10, 2, 2), (10, -1, 2), (10, 0, 0), (-1, 0, 1)]:
        with pytest.raises(ValueError):
            sharding.shard_bounds(*bad)


def test_single_process_has_no_group(monkeypatch):
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    rk = sharding.init_from_env("gloo")
    assert rk.group is None and rk.world == 1
    assert sharding.max_over_ranks(rk, 2.5) == 2.5
    assert sharding.global_count(rk, 7) == 7
    sharding.barrier(rk)


# -- two ranks over gloo ----------------------------------------------------------------------------
def _sharded_mean(rank, world, port, N, V, eps):
    import oracle
    _env(rank, world, port)
    rk = sharding.init_from_env("gloo", timeout_s=30)
    try:
        # the global batch (every rank draws the same seeded rows) and this rank's block
        z, z32, y = wl.rows(N, V, "f32", seed=11, ignore_frac=0.3)
        a, b = sharding.shard_bounds(N, rk.rank, rk.world)
        zl, yl = z32[a:b].astype(np.float64), y[a:b]
        g = sharding.mean_grad_scale(rk, yl)
        orc = oracle.get()
        loss, _, _ = orc.ce_forward(zl, yl, eps)
        dz = orc.ce_backward(zl, yl, g, eps)
        parts = [None] * rk.world
        rk.group.all_gather_object(parts, (a, b, loss.sum() * g, dz))
        t_max = sharding.max_over_ranks(rk, float(rk.rank + 1))
        assert t_max == float(rk.world)
        sharding.barrier(rk)
        if rk.rank == 0:
            full_loss, _, _ = orc.ce_forward(z32.astype(np.float64), y, eps)
            n_counted = int((y != -100).sum())
            g_full = 1.0 / n_counted
            assert abs(g - g_full) <= 1e-15 * g_full
            mean_sharded = sum(p[2] for p in parts)
            assert abs(mean_sharded - full_loss.sum() / n_counted) <= 1e-12 * abs(mean_sharded)
            full_dz = orc.ce_backward(z32.astype(np.float64), y, g_full, eps)
            got = np.concatenate([p[3] for p in sorted(parts, key=lambda p: p[0])])
            assert [p[0] for p in sorted(parts, key=lambda p: p[0])][0] == 0
            np.testing.assert_array_equal(got, full_dz)
    finally:
        rk.group.destroy_process_group()


@pytest.mark.parametrize("N,V,eps", [(101, 37, 0.0), (64, 300, 0.1)])
def test_two_ranks_mean_equals_single_process(N, V, eps):
    """Odd row counts give blocks of different sizes; 30% of rows ignored."""
    _run(_sharded_mean, N, V, eps)


def _all_ignored(rank, world, port):
    _env(rank, world, port)
    rk = sharding.init_from_env("gloo", timeout_s=30)
    try:
        y = np.full(5, -100, np.int32) if rk.rank == 0 else np.array([1, -100, 2], np.int32)
        assert sharding.global_count(rk, sharding.counted_rows(y)) == 2
        assert sharding.mean_grad_scale(rk, y) == 0.5
        none = np.full(3, -100, np.int32)
        assert sharding.mean_grad_scale(rk, none) == 0.0
    finally:
        rk.group.destroy_process_group()


def test_two_ranks_count_with_fully_ignored_block():
    _run(_all_ignored)


def _one_rank_leaves(rank, world, port):
    _env(rank, world, port)
    rk = sharding.init_from_env("gloo", timeout_s=5)
    sharding.barrier(rk)
    if rk.rank == 1:
        os._exit(0)  # leaves between steps, nothing in flight
    with pytest.raises(Exception):
        sharding.max_over_ranks(rk, 1.0)  # the next collective fails instead of waiting
    rk.group.destroy_process_group()


def test_rank_that_leaves_ends_the_next_collective_with_an_error():
    _run(_one_rank_leaves)

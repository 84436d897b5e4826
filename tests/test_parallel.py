"""Multi-rank host logic on CPU (gloo, world size 2): batch sharding covers
every (batch, head) chain exactly once, and the timing reductions take the
slowest rank."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from selective_state_space_exp_b200.parallel import max_over_ranks, shard_range, sum_over_ranks


@pytest.mark.parametrize("n,world", [(8, 2), (7, 2), (1, 2), (64, 8), (5, 3)])
def test_shard_range_partitions(n, world):
    seen = []
    for r in range(world):
        a, b = shard_range(n, world, r)
        assert 0 <= a <= b <= n
        seen.extend(range(a, b))
    assert seen == list(range(n))


def test_shard_range_rejects_bad_rank():
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        a, b = shard_range(8, world, rank)
        local_chains = (b - a) * 64
        t = 1.0 + rank  # this rank's step time
        out[rank] = torch.tensor([max_over_ranks(t), sum_over_ranks(local_chains)])
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_gloo_two_ranks():
    world = 2
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        mx, total = out[r].tolist()
        assert mx == 2.0          # the slowest rank
        assert total == 8 * 64    # every chain exactly once


def test_single_process_reductions_are_identity():
    assert max_over_ranks(3.5) == 3.5 and sum_over_ranks(2.0) == 2.0

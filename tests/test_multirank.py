"""The multi-GPU plumbing of bench.py on CPU: two gloo ranks shard the batch by sequence with no
exchange, and the step time is the max over ranks while token counts sum."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, lr = bench.dist_env()
        lo, hi = bench.shard_sequences(10, r, w)
        mx = bench.max_over_ranks(float(rank + 1) * 1.5)
        sm = bench.sum_over_ranks(float(hi - lo))
        bench.barrier()
        out[rank] = torch.tensor([lo, hi, mx, sm, r, w, lr], dtype=torch.float64)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_reduce():
    world = 2
    out = torch.zeros((world, 7), dtype=torch.float64).share_memory_()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    (lo0, hi0, mx0, sm0, r0, w0, _), (lo1, hi1, mx1, sm1, r1, w1, _) = out.tolist()
    assert (lo0, hi0, lo1, hi1) == (0, 5, 5, 10)          # contiguous, disjoint, covering
    assert mx0 == mx1 == 3.0                              # slowest rank's time
    assert sm0 == sm1 == 10.0                             # all ranks' sequences counted
    assert (r0, r1, w0, w1) == (0, 1, 2, 2)


@pytest.mark.parametrize("B,world", [(8, 1), (8, 3), (3, 4), (1000, 8)])
def test_shard_sequences_partition(B, world):
    ranges = [bench.shard_sequences(B, r, world) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == B
    assert all(ranges[i][1] == ranges[i + 1][0] for i in range(world - 1))
    sizes = [hi - lo for lo, hi in ranges]
    assert max(sizes) - min(sizes) <= 1


def test_single_process_reductions_are_identity():
    assert bench.max_over_ranks(2.5) == 2.5 and bench.sum_over_ranks(4.0) == 4.0

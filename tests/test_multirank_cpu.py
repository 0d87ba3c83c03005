"""The N>1 path of bench.py on CPU: two gloo ranks, independent problems
(distinct seeds) and the max-over-ranks reduction of timings."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_local_b200.dist_timing import max_over_ranks, rank_seed


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = max_over_ranks([1.0 + rank, 10.0 - 3 * rank, 0.5 * rank])
        seeds = [None] * world
        dist.all_gather_object(seeds, rank_seed(2000, rank))
        q.put((rank, got, seeds))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_to_the_slowest():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for _, got, seeds in res:
        assert got == [2.0, 10.0, 0.5]
        assert len(set(seeds)) == world


def test_single_process_is_identity():
    assert max_over_ranks([3.5, 1.25]) == [3.5, 1.25]

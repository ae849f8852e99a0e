"""Multi-rank host logic of bench.py on CPU with gloo (world size 2): each rank
draws its own batch and the step time is the max over ranks."""
import os
import socket

import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    import torch.distributed as dist
    r, w, _ = bench.rank_env()
    bench.init_dist(w, "gloo")
    got = bench.max_over_ranks(10.0 + 5.0 * r, w)
    bench.barrier(w)
    seeds = [None] * w
    dist.all_gather_object(seeds, bench.rank_seed(1004, r))
    out[r] = (got, tuple(seeds))
    dist.destroy_process_group()


def test_two_ranks_max_time_and_distinct_batches():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    assert out[0][0] == out[1][0] == 15.0
    assert out[0][1] == out[1][1]
    assert len(set(out[0][1])) == world


def test_single_rank_helpers_need_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)
    assert bench.rank_seed(1004, 0) == 1004

"""Host logic of the multi-rank benchmark on CPU (gloo, world size 2).

The decode linear does not shard in this build (one GPU per the workload), so
`bench.py --gpus N` runs N independent replicas; what crosses ranks is only
the timing: the elapsed time is the maximum over ranks and the throughput is
all ranks' work divided by it.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, lr = bench.dist_setup()
        assert (w, r, lr) == (world, rank, rank)
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, dist, torch.device("cpu"))
        gbs = bench.job_throughput_gbs(world, 1000, 4_000_000, ms)
        out[rank] = (ms, gbs)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_replicated_timing_takes_the_slowest_rank():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for rank in range(world):
        ms, gbs = out[rank]
        assert ms == 15.0                                   # max over ranks
        assert gbs == pytest.approx(2 * 1000 * 4e6 / 15e-3 / 1e9)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, None, None) == 3.5
    assert bench.job_throughput_gbs(1, 10, 1000, 1.0) == pytest.approx(10 * 1000 / 1e-3 / 1e9)

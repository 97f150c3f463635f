"""The multi-GPU benchmark path on CPU: two gloo ranks reduce their timings
with a max (the slowest rank sets the job time) and report weak-scaling
throughput; no collective touches the operator's data (CPU only)."""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        per_rank_ms = [1.5, 2.25][rank]
        ms, e2e = bench.max_over_ranks([per_rank_ms, 10.0 + rank], dist, "cpu")
        out[rank] = (ms, e2e, bench.job_throughput(1000, world, ms))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_max_and_weak_scale():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for rank in range(world):
        ms, e2e, value = out[rank]
        assert ms == 2.25 and e2e == 11.0
        assert value == pytest.approx(1000 * 2 / 2.25e-3)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks([3.0, 4.0], None, "cpu") == [3.0, 4.0]
    assert bench.job_throughput(10, 1, 1.0) == pytest.approx(1e4)

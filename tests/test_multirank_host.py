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


# ------------------------------------------------------------ channel shards --

def test_channel_ranges_cover_every_channel_once():
    from long_convolution_sequence_hyena_b200.sharding import channel_range
    for D in (1, 2, 7, 768):
        for world in (1, 2, 3, 8):
            ranges = [channel_range(D, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == D
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        channel_range(4, 2, 2)


def _shard_worker(rank, world, port, out):
    """Each rank computes its channel slice with the fp64 oracle on its own filter rows; the
    slices are gathered over gloo along the channel axis."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import numpy as np

        import oracle
        from long_convolution_sequence_hyena_b200.sharding import channel_range, shard_inputs
        from long_convolution_sequence_hyena_b200.workloads import WORKLOADS, make_inputs
        w = WORKLOADS["order2_bf16_b8_d768_l2048"].scaled(B=2, D=7, shape=(96,), name="shard_case")
        inp = make_inputs(w)
        d0, d1 = channel_range(w.D, world, rank)
        s = shard_inputs(inp, d0, d1)
        B, Dl, L = s["v"].shape
        y = oracle.hyena_1d(s["v"].double().reshape(B * Dl, L).numpy(),
                            s["gates"].double().reshape(w.order, B * Dl, L).numpy(),
                            s["h"].double().numpy(), s["dskip"].double().numpy(),
                            fidx=np.arange(B * Dl) % Dl).reshape(B, Dl, L)
        # gather the ragged slices: pad to the largest, then trim
        dmax = -(-w.D // world)
        pad = torch.zeros(B, dmax, L, dtype=torch.float64)
        pad[:, :Dl] = torch.from_numpy(y)
        parts = [torch.zeros_like(pad) for _ in range(world)]
        dist.all_gather(parts, pad)
        sizes = [channel_range(w.D, world, r) for r in range(world)]
        full = torch.cat([p[:, :b - a] for p, (a, b) in zip(parts, sizes)], dim=1)
        out[rank] = full.numpy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_channel_shards_gather_to_the_single_rank_result(world):
    import numpy as np

    import oracle
    from long_convolution_sequence_hyena_b200.workloads import WORKLOADS, make_inputs
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_shard_worker, args=(world, port, out), nprocs=world, join=True)
    w = WORKLOADS["order2_bf16_b8_d768_l2048"].scaled(B=2, D=7, shape=(96,), name="shard_case")
    inp = make_inputs(w)
    R, L = w.B * w.D, 96
    ref = oracle.hyena_1d(inp["v"].double().reshape(R, L).numpy(),
                          inp["gates"].double().reshape(w.order, R, L).numpy(), inp["h"].double().numpy(),
                          inp["dskip"].double().numpy(), fidx=np.arange(R) % w.D).reshape(w.B, w.D, L)
    for rank in range(world):
        np.testing.assert_array_equal(out[rank], ref)

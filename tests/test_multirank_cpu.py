"""The N > 1 path of bench.py on CPU: two gloo ranks check the per-rank input seeds,
the max-over-ranks reduction of the device time and the whole-job throughput."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from exact_tiled_attention_34_b200.inputs import make_qkv
        # each rank draws its own shard
        q = make_qkv(1, 1, 128, 64, seed=bench.rank_seed(rank), with_do=False)["q"]
        gathered = [torch.zeros_like(q, dtype=torch.float32) for _ in range(world)]
        dist.all_gather(gathered, q.float())
        distinct = not torch.equal(gathered[0], gathered[1])
        # rank r "measured" 10 + 5 r ms for 3 steps of 1e12 FLOPs each
        t = bench.max_over_ranks(10.0 + 5.0 * rank)
        v = bench.job_throughput(world, 1e12, 3, t)
        out[rank] = (t, v, distinct)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    for rank in range(world):
        t, v, distinct = out[rank]
        assert t == 15.0  # the slowest rank's time
        assert v == pytest.approx(2 * 1e12 * 3 / 15e-3 / 1e12)
        assert distinct


def test_single_process_helpers():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_throughput(1, 2e12, 4, 8.0) == pytest.approx(1000.0)
    assert bench.rank_seed(0) != bench.rank_seed(1)

"""The N > 1 path of bench.py on CPU: two gloo ranks check the per-rank input seeds,
the max-over-ranks reduction of the device time and the whole-job throughput; the
reference arm is launched through torch.distributed.run with two ranks."""
import json
import os
import signal
import socket
import subprocess
import sys

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


def test_reference_arm_under_the_launcher():
    """bench.py --impl reference launched as for N > 1 GPUs (it needs none): rank 0 alone
    prints one line, timed on all the cores it may use although the launcher sets
    OMP_NUM_THREADS=1; the other rank exits 0 without work."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    proc = subprocess.Popen(cmd, cwd=root, stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True,
                            start_new_session=True)
    try:
        out, err = proc.communicate(timeout=240)
    except subprocess.TimeoutExpired:
        os.killpg(proc.pid, signal.SIGKILL)
        proc.communicate()
        raise
    assert proc.returncode == 0, err[-2000:]
    lines = [json.loads(ln) for ln in out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["e2e"]["value"] == line["value"]
    # the same config object as the kernels' line, so the two arms compare
    import bench
    wl_name = line["config"]["workload"]
    assert line["config"] == bench.line_config(wl_name, bench.workload(wl_name), 2)
    ncpu = len(os.sched_getaffinity(0))
    assert line["cpu_baseline"]["cores"] > 1 or ncpu == 1, line["cpu_baseline"]

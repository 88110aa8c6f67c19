"""Multi-rank host logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

Each rank runs its own copy of the workload (the mixer shares nothing across
sequences), so the only cross-rank steps are the max-over-ranks timing and
the whole-job rate computed from it."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [12.5, 40.0][rank]
        worst = bench.max_over_ranks(local_ms)
        rate = bench.job_throughput(4096, world, worst * 1e-3)
        q.put((rank, worst, rate))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_rate_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, worst, rate in got:
        assert worst == 40.0                       # every rank sees the slowest rank's time
        assert rate == pytest.approx(2 * 4096 / 0.040)  # all ranks' tokens over that time


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_throughput(10, 1, 2.0) == 5.0


def test_bench_gpus_2_starts_two_ranks():
    """`bench.py --gpus 2` outside torchrun starts two ranks itself (the same
    launch path the GPU run takes; here the ranks only join a gloo group and
    report who they are)."""
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                        "--launcher-selftest"], capture_output=True, text=True, timeout=180)
    assert r.returncode == 0, r.stderr[-2000:]
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("{")][-1]
    got = json.loads(line)
    assert got["world"] == 2 and sorted(got["ranks"]) == [0, 1] and sorted(got["local_ranks"]) == [0, 1]
    assert len(set(got["pids"])) == 2


def test_bench_refuses_world_size_mismatch():
    """Under a launcher whose WORLD_SIZE differs from --gpus the bench fails
    instead of timing the wrong number of GPUs."""
    import subprocess
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2"],
                       capture_output=True, text=True, timeout=120, env=env)
    assert r.returncode != 0
    assert "differs from --gpus" in r.stdout

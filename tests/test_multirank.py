"""The N > 1 host logic of bench.py on CPU: two gloo ranks.

On several GPUs every rank runs an independent replica of the layer; the
only cross-rank steps are the barrier around the timed region and the
max-over-ranks reduction of the per-step times, and the whole-job rate is
every rank's tokens over the slowest rank's time.  The reference arm runs on
rank 0 alone; the other ranks leave without work."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, q):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        ms = bench.max_over_ranks(times[rank], torch.device("cpu"))
        q.put((rank, ms, bench.whole_job_rate(8, world, ms)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("times", [(1.25, 0.5), (0.5, 3.0)])
def test_two_ranks_take_the_slowest_time(times):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, times, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    slowest = max(times)
    for rank, ms, rate in got:
        assert ms == slowest
        assert rate == pytest.approx(8 * 2 / (slowest * 1e-3))


def test_single_rank_returns_own_time():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5, None) == 2.5
    assert bench.whole_job_rate(4096, 1, 2.0) == pytest.approx(4096 / 2e-3)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""

"""The multi-rank path of bench.py on CPU (gloo, world size 2): independent replicas, no
data-path collective; the timing is the maximum over ranks and the rate counts every rank's
tokens.  The reference arm runs on rank 0 only."""
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, ms_by_rank, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(ms_by_rank[rank], dist, world, "cpu")
        rate = bench.whole_job_rate(2048, 10, world, ms)
        out.put((rank, ms, rate))
    finally:
        dist.destroy_process_group()


def _free_port():
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_two_ranks_take_the_slowest_time_and_count_all_tokens():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ms_by_rank = [12.5, 31.25]
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, ms_by_rank, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, rate in res:
        assert ms == 31.25                                  # every rank sees the slowest rank's time
        assert rate == pytest.approx(2048 * 10 * 2 / 31.25e-3)   # all ranks' tokens / that time


def test_single_rank_is_unchanged():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.0, None, 1, "cpu") == 7.0
    assert bench.whole_job_rate(100, 3, 1, 1000.0) == pytest.approx(300.0)


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""

"""bench.py's multi-process host logic, on CPU: two gloo ranks on 127.0.0.1.

The path has no exchange step (independent sequences and channels), so N GPUs run N
replicas of the same fixed work and the only collective is the timing reduction: the
job's time is the slowest rank's, and the job's throughput counts every rank's tokens.
"""
import datetime
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, queue):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank 1 is slower on the step, rank 0 on the end-to-end pass
        got = bench.max_over_ranks([10.0 + 5.0 * rank, 100.0 - rank], dist)
        queue.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(queue.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert results[0] == [15.0, 100.0]
    assert results[1] == [15.0, 100.0]


def test_max_over_ranks_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks([3.5, 7.0], None) == [3.5, 7.0]


def test_job_throughput_counts_all_ranks_over_the_slowest():
    sys.path.insert(0, ROOT)
    import bench

    # 2 ranks x 1000 tokens x 10 steps in 20 ms
    assert bench.job_tokens_per_s(2, 1000, 10, 20.0) == 2 * 1000 * 10 / 0.020


def test_reference_arm_other_ranks_exit_without_output():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True, env=env,
                       timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""

"""bench.py's multi-rank plumbing on CPU: two gloo ranks (the replicas of `bench.py --gpus 2`).

The decode step does not shard (every rank is an independent replica, no
collective on the data path); what the ranks share is the timing: the job's
time is the slowest rank's, and the throughput counts every rank's tokens.
"""
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


def _rank_main(rank, world, port, times, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(times[rank], world)
        dist.barrier()
        out.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    world, port = 2, _free_port()
    times = [[3.0, 9.0, 1.5], [4.0, 2.0, 1.5]]  # per rank: step, end-to-end, greedy times
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] == res[1] == [4.0, 9.0, 1.5]


def test_one_rank_is_identity_and_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.25, 2.5], 1) == [1.25, 2.5]
    # 2 replicas x batch 4 x 10 steps in 20 ms = 4000 tokens/s
    assert bench.job_tokens_per_s(2, 4, 10, 20.0) == pytest.approx(4000.0)


def test_reference_arm_other_ranks_exit_without_output():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""

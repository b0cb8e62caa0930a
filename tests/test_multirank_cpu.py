"""The multi-rank host logic of bench.py on CPU ranks (gloo, world size 2).

The decode path does not shard: N GPUs run N independent replicas, and the
only collectives are the barrier and the max-over-ranks of the timing.
These tests run that logic in two gloo processes on 127.0.0.1: each rank
reports a different time and both must see the slowest; the whole-job
throughput counts every rank's bytes over that time; the reference arm does
its work on rank 0 only.
"""
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        t_local = 0.5 + rank                       # rank 1 is the slow one
        dist.barrier()
        t = bench.max_over_ranks(t_local, world, "cpu")
        q.put((rank, t, bench.job_gbs(1_000_000, 100, world, t)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, t, gbs in got:
        assert t == 1.5                            # the slowest rank's time on every rank
        assert abs(gbs - 2 * 1_000_000 * 100 / 1.5 / 1e9) < 1e-12


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(0.25, 1, "cpu") == 0.25
    assert bench.job_gbs(10 ** 9, 3, 1, 1.5) == 2.0


def test_reference_arm_works_on_rank_0_only():
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2", MASTER_ADDR="127.0.0.1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "", (r.returncode, r.stdout, r.stderr[-500:])

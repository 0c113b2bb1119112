"""The benchmark's multi-rank host logic on CPU: N ranks run N independent
replicas of the attention call (no collective on the data path), the job's
time is the slowest rank's device time, and the aggregate ms per call is that
time per step divided by the number of ranks.  Two `gloo` ranks on 127.0.0.1
take the same reduction path as the NCCL ranks on GPUs; the reference arm's
non-zero ranks exit without work."""
import datetime
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# per-rank device time over the timed steps (ms) and end-to-end ms per call
T_TOTAL = [120.0, 150.0, 90.0, 149.0]
E2E = [13.0, 11.0, 12.5, 9.0]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, steps, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        mx = bench.max_over_ranks([T_TOTAL[rank], -float(rank)], dist)
        jt = bench.job_time(T_TOTAL[rank], E2E[rank], steps, world, dist)
        q.put((rank, mx, jt))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _run(world, steps):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, steps, q))
             for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    try:
        for _ in range(world):
            rank, mx, jt = q.get(timeout=120)
            out[rank] = (mx, jt)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    return out


@pytest.mark.parametrize("world", [2, 4])
def test_job_time_is_the_slowest_rank_over_world(world):
    steps = 10
    out = _run(world, steps)
    assert sorted(out) == list(range(world))
    t_max = max(T_TOTAL[:world])
    e2e_max = max(E2E[:world])
    for rank, (mx, (ms_call, value, e2e_value)) in out.items():
        assert mx == [t_max, 0.0]  # element-wise max; every rank sees the same
        assert ms_call == pytest.approx(t_max / steps)
        assert value == pytest.approx(t_max / steps / world)
        assert e2e_value == pytest.approx(e2e_max / world)


def test_job_time_single_rank_is_the_identity():
    ms_call, value, e2e_value = bench.job_time(120.0, 13.0, 10, 1)
    assert (ms_call, value, e2e_value) == (12.0, 12.0, 13.0)
    assert bench.max_over_ranks([3, 4.5]) == [3.0, 4.5]


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, cwd=ROOT, capture_output=True, text=True,
                       timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""

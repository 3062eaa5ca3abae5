"""The multi-process (one process per GPU) host path of bench.py on CPU: two gloo ranks take
part in the same collective steps, the timing reported is the slowest rank's, and the value
is the whole job's (weak scaling: every rank processes the same units).  The GPU work itself
is not exercised here (one GPU per box on this pool)."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import datetime
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        torch.distributed.barrier()
        ms = bench.max_over_ranks(times[rank], world, "cpu")
        value = bench.job_value(1000, world, ms)
        torch.distributed.barrier()
        out.put((rank, ms, value))
    finally:
        torch.distributed.destroy_process_group()


def test_two_ranks_report_the_slowest_time_and_the_whole_job_value():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    times = [3.0, 5.0]
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, times, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [5.0, 5.0]                      # both see the maximum
    assert all(abs(r[2] - 2 * 1000 / 5e-3) < 1e-6 for r in res)  # units of both ranks / slowest


def test_single_rank_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(4.0, 1, "cpu") == 4.0
    assert bench.job_value(500, 1, 2.0) == 500 / 2e-3


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2"],
                       capture_output=True, text=True, env=env, timeout=300, cwd=ROOT)
    assert r.returncode == 0
    assert r.stdout.strip() == ""

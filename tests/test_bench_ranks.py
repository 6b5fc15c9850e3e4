"""The multi-process path of bench.py, on CPU: two gloo ranks.

With N GPUs the bench runs one process per GPU, each on its own replica of
the workload (no data-path collective).  The only cross-rank steps are the
job time, the slowest rank's (a MAX all-reduce), and the whole-job
throughput, every rank's work over that time.  Both are exercised here with
ranks whose local times differ.
"""
import datetime
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, local_s, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        job = bench.max_over_ranks(local_s[rank], world, "cpu")
        q.put((rank, job, bench.job_tflops(2.0e12, 4, world, job)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_single_rank_time_is_its_own():
    assert bench.max_over_ranks(0.125, 1, None) == 0.125
    assert bench.job_tflops(2.0e12, 4, 1, 0.5) == pytest.approx(16.0)


def test_two_ranks_take_the_slowest_time_and_add_their_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    local_s = (0.25, 0.75)
    procs = [ctx.Process(target=_rank, args=(r, 2, port, local_s, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        got = sorted(q.get(timeout=120) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [p.exitcode for p in procs] == [0, 0]
    for rank, job, tflops in got:
        assert job == 0.75, rank
        # two replicas of 4 steps x 2 TFLOP each, over the slowest rank's 0.75 s
        assert tflops == pytest.approx(2 * 4 * 2.0 / 0.75)


@pytest.mark.skipif(torch.cuda.is_available(), reason="gloo ranks on CPU hosts; GPU hosts give each rank a GPU")
def test_gpus_flag_launches_that_many_ranks():
    """`bench.py --gpus 2` outside torchrun relaunches itself as two ranks
    (here the launch check only: each rank joins the group and reports)."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--probe-ranks"],
                         capture_output=True, text=True, timeout=180, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads([l for l in out.stdout.splitlines() if l.startswith("{")][-1])
    assert line["n_gpus"] == 2 and line["ranks_seen"] == [0, 1] and line["backend"] == "gloo"
    assert line["max_over_ranks"] == pytest.approx(0.2)

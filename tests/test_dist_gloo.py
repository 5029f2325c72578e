"""The N>1 host path of bench.py on CPU ranks (gloo, world size 2).

The benchmark runs N independent replicas (one process per GPU, no
data-path collective): the process group only brackets the timed region with
barriers and takes the maximum of the ranks' device times.  These tests run
that plumbing as two gloo processes on the CPU: the whole-job rate is the
units all ranks processed over the slowest rank's time, every rank sees the
same maximum, and the reference arm runs on rank 0 alone.
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


def _rank_main(rank, world, port, local_ms, units, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist()
    d.init("gloo")
    d.barrier()
    value, ms = bench.job_rate(d, units, local_ms[rank])
    d.barrier()
    out_q.put((rank, value, ms))
    d.close()


def _run_ranks(local_ms, units):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, len(local_ms), port, local_ms, units, q))
             for r in range(len(local_ms))]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(res)


def test_job_rate_max_over_two_gloo_ranks():
    # rank 1 is the slower: both ranks report its time, and the rate counts
    # the units of both replicas
    res = _run_ranks([10.0, 25.0], units=1000)
    for rank, value, ms in res:
        assert ms == 25.0
        assert value == pytest.approx(2 * 1000 / 0.025)


def test_job_rate_single_process_is_local():
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist()
    assert d.world == int(os.environ.get("WORLD_SIZE", "1"))
    if d.world == 1:
        value, ms = bench.job_rate(d, 50, 5.0)
        assert ms == 5.0 and value == pytest.approx(50 / 0.005)


def test_reference_arm_other_ranks_exit_quietly():
    # under torchrun the reference arm runs on rank 0 alone; rank 1 exits 0
    # without output and without joining a process group
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1",
               MASTER_PORT=str(_free_port()))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""

"""The bench's N > 1 path (replicas, one process per GPU) on CPU: two gloo ranks.

Every rank times the same workload on its own device; the job's time is the
slowest rank's (a MAX all-reduce), and the whole-job value counts every rank's
units over that time.  The processes here stand in for the GPUs: the timing
reduction and the value arithmetic are the host logic the bench runs.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, local_ms, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        ms_max = bench.max_over_ranks(local_ms[rank])
        value = bench.whole_job_tflops(2.0e11, world, ms_max)
        q.put((rank, ms_max, value))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("local_ms", [(0.130, 0.142), (0.5, 0.25)])
def test_two_ranks_take_the_slowest_time(local_ms):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, local_ms, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get() for _ in range(world))
    expect_ms = max(local_ms)
    for rank, ms_max, value in got:
        assert ms_max == expect_ms
        assert value == pytest.approx(2.0e11 * world / (expect_ms * 1e-3) / 1e12, rel=1e-12)


def test_single_process_is_its_own_maximum():
    assert bench.max_over_ranks(0.123) == 0.123
    assert bench.whole_job_tflops(2.0e11, 1, 0.1) == pytest.approx(2000.0)


def test_reference_arm_under_torchrun_prints_once():
    # `bench.py --impl reference` launched as two ranks: rank 0 runs the oracle arm
    # and prints the one JSON line, the other rank exits 0 without work
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "2", "--warmup", "3", "--config", "0"]
    res = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, res.stdout[-2000:]
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["steps"] == 2 and line["warmup"] == 3 and line["higher_is_better"] is True
    assert line["cpu_baseline"]["value"] == line["value"] == line["e2e"]["value"]
    assert line["config"]["workload"] and line["cpu_baseline"]["cores"] >= 1

"""The N > 1 host path of bench.py on CPU: two gloo ranks on 127.0.0.1.

Each rank runs its own replica of the workload (no data-path collective). The bench's
only collectives are the barrier and the max over ranks of the timed duration, and the
job's value is all ranks' units over the slowest rank's time. The reference arm under a
multi-rank launch runs on rank 0 alone; the other ranks exit 0 without output.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        dev = torch.device("cpu")
        bench.barrier(True, dev)
        elapsed = [0.5, 2.0][rank]                      # rank 1 is the slow one
        value, tmax = bench.weak_scaling_value(1000.0, elapsed, True, dev, world)
        bench.barrier(True, dev)
        out[rank] = (value, tmax)
    finally:
        dist.destroy_process_group()


def test_two_rank_weak_scaling_aggregation():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    assert set(res) == {0, 1}
    for rank in (0, 1):
        value, tmax = res[rank]
        assert tmax == pytest.approx(2.0)               # the max over ranks, seen by every rank
        assert value == pytest.approx(1000.0 * world / 2.0)


def test_reference_arm_nonzero_rank_exits_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1",
               MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""

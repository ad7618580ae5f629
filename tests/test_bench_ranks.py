"""Host-side multi-rank logic of bench.py, on CPU.

bench.py runs one replica of the layer per GPU (the layer needs no collective);
the only cross-rank steps are a barrier around the timed region and the
max-over-ranks reduction of the measured times.  Here two gloo ranks check that
reduction and the whole-job aggregate, and the reference arm's rule that only
rank 0 works and prints.
"""
import json
import os
import socket
import sys
from argparse import Namespace
from datetime import timedelta

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        dist.barrier()
        slowest = bench.max_over_ranks(times[rank], dist, "cpu")
        dist.barrier()
        q.put((rank, slowest))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("times", [(1.5, 3.5), (4.25, 0.5)])
def test_max_over_ranks_gloo(times):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        got = sorted(q.get(timeout=120) for _ in range(world))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    assert got == [(0, max(times)), (1, max(times))]


def test_max_over_ranks_single_process():
    assert bench.max_over_ranks(2.5) == 2.5


def test_job_gbps_is_whole_job():
    # 12,091,392 compressed weight bytes a step per replica, 9.25 us a step
    one = bench.job_gbps(1, 12_091_392, 0.00925)
    assert one == pytest.approx(1307.178, rel=1e-6)
    assert bench.job_gbps(8, 12_091_392, 0.00925) == pytest.approx(8 * one)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    args = Namespace(m=16, steps=1, warmup=3, gpus=2)
    bench.run_reference(args, rank=1, world=2)
    assert capsys.readouterr().out == ""
    bench.run_reference(args, rank=0, world=2)
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"

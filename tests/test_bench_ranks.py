"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

Under torchrun every rank runs an independent replica; the only collectives
are the barrier and the max-over-ranks reduction of the timed totals, from
which the whole-job rate is formed.  These run here with the gloo backend.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, totals, out):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        m = bench.max_over_ranks(totals[rank], world, "cpu")
        rate = bench.whole_job_rate(world, 64, m, 20)
        out.put((rank, m, rate))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_gloo():
    world = 2
    totals = [12.5, 17.25]          # ms over 20 steps on each rank
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, totals, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, rate in res:
        assert m == max(totals)                               # every rank sees the slowest rank's time
        assert rate == pytest.approx(world * 64 / (max(totals) / 20 * 1e-3))


def test_single_rank_helpers():
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.whole_job_rate(1, 64, 10.0, 10) == pytest.approx(64 / 1e-3)


def test_kernels_per_step_and_config():
    from hierarchical_kv_pruning_b200 import synth
    dev = synth.shape(2)
    host = synth.shape(4)
    assert bench.kernels_per_step(dev) == 10
    assert host.batch >= 8 and bench.kernels_per_step(host) == 4 * 14   # four query chunks
    import dataclasses
    assert bench.kernels_per_step(dataclasses.replace(host, batch=7)) == 14
    c = bench.config_of(dev, 4)
    assert c["workload"] == dev.name and c["parallelism"] == "replicas x4"
    assert c["B"] == dev.batch and c["K"] == list(dev.keep)

"""Host logic of the N-GPU benchmark on CPU: two gloo ranks on 127.0.0.1.

bench.py --gpus N runs N independent layers (weak scaling, no data-path
collective); the only cross-rank steps are the timing barrier and the max of
the ranks' times. These tests run that host logic with the gloo backend.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from block_sparse_bidirectional_select_b200.inputs import WORKLOADS, make_inputs
        # each rank times a different amount; every rank must see the maximum
        mine = 10.0 + 5.0 * rank
        dist.barrier()
        got = bench.reduce_max(mine, world, torch.device("cpu"))
        # each rank's layer has its own seed, so its own inputs
        wl = bench.rank_workload(WORKLOADS["tiny"].scaled(H=1, L=128), rank)
        q, _, _ = make_inputs(wl)
        sums = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(sums, q.double().sum().reshape(1))
        out[rank] = (got, wl.seed, [float(x) for x in sums])
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_run_distinct_layers():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    assert res[0][1] != res[1][1]
    assert res[0][2] == res[1][2] and res[0][2][0] != res[0][2][1]


def test_job_value_counts_every_rank_over_the_slowest_time():
    import bench
    # 2 ranks x 3 steps x 1e12 flop in 1.5 s -> 4 TFLOP/s of whole-job throughput
    assert bench.job_value(1e12, 3, 2, 1500.0) == pytest.approx(4.0)
    assert bench.reduce_max(7.5, 1, torch.device("cpu")) == 7.5


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import argparse
    import bench
    args = argparse.Namespace(workload="tiny", cpu_seconds=0.1, warmup=1, steps=1)
    assert bench.run_reference(args, rank=1, world=2) == 0
    assert capsys.readouterr().out == ""

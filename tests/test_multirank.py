"""Host logic of the N-GPU benchmark on CPU: two gloo ranks on 127.0.0.1.

bench.py --gpus N splits one layer's heads evenly over N ranks (strong
scaling); the cross-rank steps are the timing barrier, the max of the ranks'
times, the sum of the ranks' flops, and (entropy budget) the all-gather of the
per-head entropies. These tests run that host logic with the gloo backend.
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
        # the ranks hold disjoint heads of one layer (same seed, same inputs)
        wl = WORKLOADS["tiny"].scaled(L=128)
        h0, h1 = bench.head_range(wl.H, world, rank)
        q, _, _ = make_inputs(wl)
        part = q[h0:h1].double().sum()
        total = bench.reduce_sum(float(part), world, torch.device("cpu"))
        out[rank] = (got, (h0, h1), total, float(q.double().sum()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_split_one_layer():
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
    assert res[0][1] == (0, 2) and res[1][1] == (2, 4)      # tiny has H = 4
    assert res[0][2] == pytest.approx(res[0][3]) and res[1][2] == pytest.approx(res[1][3])


def test_job_value_is_the_layer_over_the_slowest_time():
    import bench
    # the layer's 3e12 flop per step x 2 steps in 1.5 s -> 4 TFLOP/s
    assert bench.job_value(3e12, 2, 1500.0) == pytest.approx(4.0)
    assert bench.reduce_max(7.5, 1, torch.device("cpu")) == 7.5
    assert bench.reduce_sum(7.5, 1, torch.device("cpu")) == 7.5
    assert bench.head_range(32, 8, 3) == (12, 16)
    with pytest.raises(SystemExit):
        bench.head_range(32, 3, 0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import argparse
    import bench
    args = argparse.Namespace(workload="tiny", cpu_seconds=0.1, warmup=1, steps=1)
    assert bench.run_reference(args, rank=1, world=2) == 0
    assert capsys.readouterr().out == ""

"""Head-sharded selection with the entropy budget (the heads of one layer
split over ranks; only the per-head entropies cross ranks).

CPU: the library's host allocation against the oracle's entropy budget, and
two gloo ranks gathering their heads' entropies and reaching the same
allocation. GPU: two shards of a layer, run one after the other on one GPU
and joined by hand, give exactly the pattern of the unsharded selection."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
import block_sparse_bidirectional_select_b200 as sp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("seed", range(12))
def test_host_budget_matches_oracle(seed):
    rng = np.random.default_rng(seed)
    H = int(rng.integers(1, 40))
    nkb = int(rng.integers(2, 80))
    keep = float(np.float32(rng.choice([0.05, 0.1, 0.25, 0.5, 0.9])))
    ent = rng.random(H) * rng.choice([0.0, 1.0, 3.0])
    if seed % 3 == 0:
        ent[int(rng.integers(H))] = 50.0  # one dominant head: its share is capped
    got = sp.entropy_budget(ent.tolist(), nkb, keep)
    ref, _ = O.entropy_budget(list(ent), nkb, keep)
    assert got == [int(x) for x in ref]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import block_sparse_bidirectional_select_b200 as spw
        local = torch.tensor([0.3 + rank, 1.7 * rank, 0.9], dtype=torch.float64)  # this rank's 3 heads
        ent_all, r = spw.gather_head_entropies(local, dist.group.WORLD)
        k_all = spw.entropy_budget(ent_all.tolist(), 64, 0.1)
        out[rank] = (r, ent_all.tolist(), k_all, k_all[3 * r:3 * r + 3])
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_share_one_allocation():
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
    assert res[0][1] == res[1][1] == [0.3, 0.0, 0.9, 1.3, 1.7, 0.9]
    assert res[0][2] == res[1][2]
    k_all = res[0][2]
    ref, _ = O.entropy_budget(res[0][1], 64, 0.1)
    assert k_all == [int(x) for x in ref]
    assert sum(k_all) == max(6, int(np.ceil(float(np.float32(0.1)) * 6 * 64 - 1e-6)))
    assert res[0][3] + res[1][3] == k_all


@pytest.mark.gpu
def test_two_shards_on_one_gpu_equal_the_unsharded_selection():
    from block_sparse_bidirectional_select_b200.inputs import WORKLOADS, make_inputs
    wl = WORKLOADS["tiny"].scaled(H=6, L=2048, d=128, bq=128, bk=128, seed=303, structure="band")
    q, k, v = (t.cuda() for t in make_inputs(wl))
    keep = 0.15
    full = sp.select_pattern(q, k, v, keep=keep, budget="entropy")
    shards = [slice(0, 3), slice(3, 6)]
    runs = [sp.select_head_entropy(q[s].contiguous(), k[s].contiguous(), v[s].contiguous()) for s in shards]
    ent_all = torch.cat([r[2].cpu() for r in runs])
    nkb = -(-wl.L // 128)
    k_all = sp.entropy_budget(ent_all.tolist(), nkb, keep)
    assert k_all == full.head_k.cpu().tolist()
    for (o, lse, _, ws), s in zip(runs, shards):
        kv_idx, kv_count, _ = sp.select_with_head_k(3, wl.L, k_all[s], ws)
        sp.device_check()
        stride = full.kv_idx.shape[2]
        assert torch.equal(kv_count, full.kv_count[s])
        for h in range(3):
            for i in range(kv_count.shape[1]):
                c = int(kv_count[h, i])
                assert torch.equal(kv_idx[h, i, :c], full.kv_idx[s][h, i, :c])
        assert torch.equal(o.view(torch.int16), full.o[s].view(torch.int16))
        assert torch.equal(lse, full.lse[s])

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


@pytest.mark.gpu
def test_sharded_denoising_loop_two_shards_in_two_threads():
    """Two ranks emulated by two host threads on one GPU (each its own stream;
    the all-gather replaced by an in-process exchange behind a barrier; no
    kernel waits on another): the loop with the entropy budget, anchors
    included, gives each shard exactly the heads of the unsharded loop."""
    import threading

    from block_sparse_bidirectional_select_b200.inputs import WORKLOADS, make_inputs
    wl = WORKLOADS["tiny"].scaled(H=4, L=1024, d=128, bq=128, bk=128, seed=404, structure="band")
    q, k, v = (t.cuda() for t in make_inputs(wl))
    T, w, r, keep = 8, 0.3, 2, 0.2  # selects at steps 2, 4, 6; the last step is block-sparse
    full = sp.run_steps_sharded(q, k, v, T, w, keep, "entropy", r)
    sp.device_check()
    shards = [slice(0, 2), slice(2, 4)]
    barrier = threading.Barrier(2)
    slots = [None, None]
    results = [None, None]
    errors = []

    def make_gather(rank):
        def gather(ent):
            slots[rank] = ent.cpu()
            barrier.wait(timeout=120)
            ent_all = torch.cat(slots)
            barrier.wait(timeout=120)
            return ent_all, rank
        return gather

    def worker(rank):
        try:
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                sl = shards[rank]
                res = sp.run_steps_sharded(q[sl].contiguous(), k[sl].contiguous(), v[sl].contiguous(), T, w,
                                           keep, "entropy", r, stream=s, gather=make_gather(rank), rank=rank,
                                           world=2)
                s.synchronize()
                results[rank] = res
        except Exception as e:  # reported below; the barrier times out for the other thread
            errors.append(e)
            barrier.abort()

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(300)
    assert not errors, errors
    sp.device_check()
    assert full.kinds.count(sp.STEP_SELECT) == 3 and full.kinds[-1] == sp.STEP_SPARSE
    for res, sl in zip(results, shards):
        assert torch.equal(res.kv_count, full.kv_count[sl])
        for h in range(2):
            for i in range(res.kv_count.shape[1]):
                c = int(res.kv_count[h, i])
                assert torch.equal(res.kv_idx[h, i, :c], full.kv_idx[sl][h, i, :c])
        assert torch.equal(res.o.view(torch.int16), full.o[sl].view(torch.int16))
        assert torch.equal(res.lse, full.lse[sl])
    # the last step's output is the block-sparse attention over the final pattern
    qh, kh, vh = (t.float().cpu().numpy().astype(np.float64) for t in (q, k, v))
    idx, cnt = full.kv_idx.cpu().numpy(), full.kv_count.cpu().numpy()
    for h in range(4):
        lists = [idx[h, i, :cnt[h, i]] for i in range(idx.shape[1])]
        o_ref, l_ref = O.masked_attention(qh[h], kh[h], vh[h], wl.scale, lists, cnt[h], 128, 128)
        assert np.abs(full.o[h].float().cpu().numpy() - o_ref).max() <= 2e-2
        assert np.abs(full.lse[h].cpu().numpy() - l_ref).max() <= 1e-3


def _gpu_shard_worker(rank, world, port, out):
    """One rank of a two-process head-sharded loop on cuda:0: its half of the
    heads, the per-head entropies all-gathered over a gloo group on the host
    (no kernel of one process waits on the other's)."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        import block_sparse_bidirectional_select_b200 as spw
        from block_sparse_bidirectional_select_b200.inputs import WORKLOADS, make_inputs
        torch.cuda.set_device(0)
        wl = WORKLOADS["tiny"].scaled(H=4, L=1024, d=128, bq=128, bk=128, seed=505, structure="band")
        q, k, v = make_inputs(wl)
        sl = slice(2 * rank, 2 * rank + 2)
        qs, ks, vs = (t[sl].contiguous().cuda() for t in (q, k, v))
        res = spw.run_steps_sharded(qs, ks, vs, 8, 0.3, 0.2, "entropy", 2, group=dist.group.WORLD)
        torch.cuda.synchronize()
        spw.device_check()
        out[rank] = (res.kinds, res.kv_idx.cpu().numpy(), res.kv_count.cpu().numpy(),
                     res.o.view(torch.int16).cpu().numpy(), res.lse.cpu().numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.gpu
def test_sharded_denoising_loop_two_processes_gloo():
    """Two processes on one GPU, a gloo group between them, each running the
    head-sharded loop (entropy budget, anchors) on its half of the heads: each
    rank's heads equal the unsharded loop's bit for bit."""
    from block_sparse_bidirectional_select_b200.inputs import WORKLOADS, make_inputs
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_gpu_shard_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(300)
            assert p.exitcode == 0
        res = dict(out)
    wl = WORKLOADS["tiny"].scaled(H=4, L=1024, d=128, bq=128, bk=128, seed=505, structure="band")
    q, k, v = (t.cuda() for t in make_inputs(wl))
    full = sp.run_steps_sharded(q, k, v, 8, 0.3, 0.2, "entropy", 2)
    sp.device_check()
    assert full.kinds.count(sp.STEP_SELECT) == 3
    idx, cnt = full.kv_idx.cpu().numpy(), full.kv_count.cpu().numpy()
    o16, lse = full.o.view(torch.int16).cpu().numpy(), full.lse.cpu().numpy()
    for rank in range(world):
        kinds, r_idx, r_cnt, r_o16, r_lse = res[rank]
        sl = slice(2 * rank, 2 * rank + 2)
        assert kinds == full.kinds
        assert (r_cnt == cnt[sl]).all()
        for h in range(2):
            for i in range(r_cnt.shape[1]):
                c = int(r_cnt[h, i])
                assert (r_idx[h, i, :c] == idx[sl][h, i, :c]).all()
        assert (r_o16 == o16[sl]).all()
        assert (r_lse == lse[sl]).all()

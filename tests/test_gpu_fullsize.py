"""Full workload sizes, in the launch configuration the bench uses, checked on
sampled (head, query block) tiles the oracle computes one by one: the dense
pass, the block-mass row, the selection (margin rule and kernel-precision
exactness), and the block-sparse output with the GPU's own pattern. The
denoising loop's own selection (the block mass fused into its full pass, the
pattern the benchmark runs with) is compared with the separate selection pass
over the whole grid and with the oracle on tiles spread over every head.
Configuration 1 runs at its stated shape and is checked in full."""
import numpy as np
import pytest
import torch

import oracle as O
import block_sparse_bidirectional_select_b200 as sp
from block_sparse_bidirectional_select_b200.inputs import WORKLOADS, make_inputs
from gpu_common import MASS_RTOL, SELECT_MARGIN, assert_o_lse, check_selection, f64

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _samples(wl, rng, n=4):
    nqb = -(-wl.L // wl.bq)
    picks = {(0, 0), (wl.H - 1, nqb - 1)}
    while len(picks) < n:
        picks.add((int(rng.integers(wl.H)), int(rng.integers(nqb))))
    return sorted(picks)


@pytest.mark.parametrize("name", ["c2_8k", "c3_16k", "c4_64k", "c5_32k_entropy"])
def test_fullsize_select_and_sparse_sampled(name):
    wl = WORKLOADS[name]
    q, k, v = make_inputs(wl)
    qc, kc, vc = (t.cuda() for t in (q, k, v))
    p = sp.select_pattern(qc, kc, vc, keep=wl.keep, budget=wl.budget, bq=wl.bq, bk=wl.bk, return_mass=True)
    o_s, l_s = sp.block_sparse_attn(qc, kc, vc, p.kv_idx, p.kv_count, bq=wl.bq, bk=wl.bk)
    sp.device_check()
    nkb = -(-wl.L // wl.bk)
    mass = p.block_mass.cpu().numpy().astype(np.float64)
    head_k = p.head_k.cpu().numpy()
    idx = p.kv_idx.cpu().numpy()
    cnt = p.kv_count.cpu().numpy()
    if wl.budget == "uniform":
        assert (head_k == O.uniform_keep(nkb, wl.keep)).all()
    else:
        ent = [O.head_entropy(mass[h]) for h in range(wl.H)]
        k_ref, B = O.entropy_budget(ent, nkb, wl.keep)
        assert list(head_k) == k_ref and int(head_k.sum()) == B
    assert (cnt == head_k[:, None]).all()
    rng = np.random.default_rng(sum(map(ord, name)))
    cache = {}
    for h, i in _samples(wl, rng):
        if h not in cache:
            cache = {h: (f64(q[h]), f64(k[h]), f64(v[h]))}
        qh, kh, vh = cache[h]
        r0, r1 = i * wl.bq, min((i + 1) * wl.bq, wl.L)
        od, ld = O.dense_attention(qh, kh, vh, wl.scale, rows=np.arange(r0, r1))
        assert_o_lse(p.o[h, r0:r1], p.lse[h, r0:r1], od, ld, f"{name} dense h{h} i{i}")
        lse_full = np.zeros(wl.L)
        lse_full[r0:r1] = ld
        m_ref = O.block_mass(qh, kh, wl.scale, lse_full, wl.bq, wl.bk, qblocks=[i])[0]
        np.testing.assert_allclose(mass[h, i], m_ref, rtol=MASS_RTOL, atol=1e-6)
        kk = int(head_k[h])
        check_selection(idx[h, i], cnt[h, i], m_ref, kk, f"{name} h{h} i{i}")
        assert list(idx[h, i, :kk]) == list(O.topk_blocks(mass[h, i], kk))
        keys = O.kept_keys(idx[h, i, :kk], wl.bk, wl.L)
        om, lm = O.softmax_attention(qh[r0:r1], kh[keys], vh[keys], wl.scale)
        assert_o_lse(o_s[h, r0:r1], l_s[h, r0:r1], om, lm, f"{name} sparse h{h} i{i}")


def test_fullsize_run_steps_64k():
    wl = WORKLOADS["c4_64k"]
    q, k, v = make_inputs(wl)
    qc, kc, vc = (t.cuda() for t in (q, k, v))
    r = sp.run_steps(qc, kc, vc, T=4, warmup_frac=0.5, keep=wl.keep, bq=wl.bq, bk=wl.bk, time_steps=True)
    sp.device_check()
    assert r.kinds == [O.DENSE, O.SELECT, O.SPARSE, O.SPARSE]
    idx = r.kv_idx.cpu().numpy()
    rng = np.random.default_rng(4)
    for h, i in _samples(wl, rng, n=3):
        qh, kh, vh = f64(q[h]), f64(k[h]), f64(v[h])
        r0, r1 = i * wl.bq, (i + 1) * wl.bq
        keys = O.kept_keys(idx[h, i, :O.uniform_keep(-(-wl.L // wl.bk), wl.keep)], wl.bk, wl.L)
        om, lm = O.softmax_attention(qh[r0:r1], kh[keys], vh[keys], wl.scale)
        assert_o_lse(r.o[h, r0:r1], r.lse[h, r0:r1], om, lm, f"run_steps h{h} i{i}")


def _gpu_margins(mass, cnt):
    """Relative gap between the k-th and (k+1)-th largest mass of every row of
    a GPU mass grid [H, nqb, nkb] with per-row k = cnt [H, nqb]."""
    nkb = mass.shape[-1]
    ms = torch.sort(mass, dim=-1, descending=True).values
    kk = cnt.long()
    mk = ms.gather(-1, (kk - 1).clamp(min=0)[..., None])[..., 0]
    mk1 = ms.gather(-1, kk.clamp(max=nkb - 1)[..., None])[..., 0]
    mk1 = torch.where(kk < nkb, mk1, torch.full_like(mk1, -float("inf")))
    return (mk - mk1) / mk, mk


@pytest.mark.parametrize("name,T,warmup,refresh", [
    ("c4_64k", 3, 0.5, 0),           # dense, select (fused), sparse
    ("c3_16k", 4, 0.5, 2),           # dense, select, sparse, refresh select (fused, LSE of the earlier pass)
    ("c5_32k_entropy", 3, 0.5, 0),   # ragged per-head budgets
])
def test_fullsize_loop_selection(name, T, warmup, refresh):
    wl = WORKLOADS[name]
    q, k, v = make_inputs(wl)
    qc, kc, vc = (t.cuda() for t in (q, k, v))
    r = sp.run_steps(qc, kc, vc, T=T, warmup_frac=warmup, keep=wl.keep, budget=wl.budget,
                     refresh_every=refresh, bq=wl.bq, bk=wl.bk)
    sp.device_check()
    kinds = O.schedule(T, warmup, refresh)
    assert r.kinds == kinds and O.SELECT in kinds and kinds[kinds.index(O.SELECT) - 1] == O.DENSE
    # the separate selection pass over the same inputs
    p = sp.select_pattern(qc, kc, vc, keep=wl.keep, budget=wl.budget, bq=wl.bq, bk=wl.bk, return_mass=True)
    sp.device_check()
    nqb, nkb = -(-wl.L // wl.bq), -(-wl.L // wl.bk)
    assert torch.equal(r.kv_count, p.kv_count), "per-row counts of the loop's and the separate selection"
    # whole grid: equal lists wherever the GPU mass margin exceeds the tolerance,
    # and within the margin otherwise
    margin, mk = _gpu_margins(p.block_mass, p.kv_count)
    clear = margin > SELECT_MARGIN
    stride = min(r.kv_idx.shape[2], p.kv_idx.shape[2])
    used = torch.arange(stride, device="cuda")[None, None, :] < r.kv_count[..., None]
    same = ((r.kv_idx[..., :stride] == p.kv_idx[..., :stride]) | ~used).all(dim=-1)
    assert bool(same[clear].all()), f"{name}: {int((~same & clear).sum())} clear-margin rows differ"
    picked = torch.gather(p.block_mass, -1, r.kv_idx[..., :stride].clamp(min=0).long())
    low = (picked < (mk * (1 - SELECT_MARGIN))[..., None]) & used
    assert not bool(low.any()), f"{name}: the loop kept a block below the k-th mass"
    assert clear.float().mean().item() > 0.5
    # the oracle on one tile of every head, plus the grid's corners
    rng = np.random.default_rng(7 + sum(map(ord, name)))
    tiles = sorted({(h, int(rng.integers(nqb))) for h in range(wl.H)} | {(0, 0), (wl.H - 1, nqb - 1)})
    assert len(tiles) >= 32
    idx = r.kv_idx.cpu().numpy()
    cnt = r.kv_count.cpu().numpy()
    sparse_last = r.kinds[-1] == O.SPARSE
    checked = 0
    for h, i in tiles:
        qh, kh, vh = f64(q[h]), f64(k[h]), f64(v[h])
        r0, r1 = i * wl.bq, min((i + 1) * wl.bq, wl.L)
        _, ld = O.dense_attention(qh, kh, vh, wl.scale, rows=np.arange(r0, r1))
        lse_full = np.zeros(wl.L)
        lse_full[r0:r1] = ld
        m_ref = O.block_mass(qh, kh, wl.scale, lse_full, wl.bq, wl.bk, qblocks=[i])[0]
        kk = int(cnt[h, i])
        check_selection(idx[h, i], kk, m_ref, kk, f"{name} loop h{h} i{i}")
        if sparse_last and checked < 6:
            keys = O.kept_keys(idx[h, i, :kk], wl.bk, wl.L)
            om, lm = O.softmax_attention(qh[r0:r1], kh[keys], vh[keys], wl.scale)
            assert_o_lse(r.o[h, r0:r1], r.lse[h, r0:r1], om, lm, f"{name} loop sparse h{h} i{i}")
            checked += 1
    if wl.budget == "entropy":
        mass = p.block_mass.cpu().numpy().astype(np.float64)
        k_ref, B = O.entropy_budget([O.head_entropy(mass[h]) for h in range(wl.H)], nkb, wl.keep)
        assert list(cnt[:, 0]) == k_ref and int(cnt[:, 0].sum()) == B


def test_config1_tiny_in_full():
    """Configuration 1 at its stated shape (H=4, L=1024, d=64, bq=bk=64, keep
    0.25, i.i.d. N(0,1), seed 1001): one selection pass, then one block-sparse
    call; every O / LSE row, every block-mass entry and every selection row
    against the oracle."""
    wl = WORKLOADS["tiny"]
    assert (wl.H, wl.L, wl.d, wl.bq, wl.bk, wl.keep, wl.structure, wl.seed) == \
        (4, 1024, 64, 64, 64, 0.25, "iid", 1001)
    q, k, v = make_inputs(wl)
    qc, kc, vc = (t.cuda() for t in (q, k, v))
    p = sp.select_pattern(qc, kc, vc, keep=wl.keep, bq=wl.bq, bk=wl.bk, return_mass=True)
    o_s, l_s = sp.block_sparse_attn(qc, kc, vc, p.kv_idx, p.kv_count, bq=wl.bq, bk=wl.bk)
    sp.device_check()
    nqb, nkb = wl.L // wl.bq, wl.L // wl.bk
    kk = O.uniform_keep(nkb, wl.keep)
    assert kk == 4
    mass = p.block_mass.cpu().numpy().astype(np.float64)
    idx = p.kv_idx.cpu().numpy()
    cnt = p.kv_count.cpu().numpy()
    assert (cnt == kk).all()
    clear = 0
    for h in range(wl.H):
        qh, kh, vh = f64(q[h]), f64(k[h]), f64(v[h])
        od, ld = O.dense_attention(qh, kh, vh, wl.scale)
        assert_o_lse(p.o[h], p.lse[h], od, ld, f"config 1 dense h{h}")
        m_ref = O.block_mass(qh, kh, wl.scale, ld, wl.bq, wl.bk)
        np.testing.assert_allclose(mass[h], m_ref, rtol=MASS_RTOL, atol=1e-6)
        for i in range(nqb):
            clear += check_selection(idx[h, i], cnt[h, i], m_ref[i], kk, f"config 1 h{h} i{i}")
            assert list(idx[h, i, :kk]) == list(O.topk_blocks(mass[h, i], kk))
        lists = [idx[h, i, :kk] for i in range(nqb)]
        om, lm = O.masked_attention(qh, kh, vh, wl.scale, lists, cnt[h], wl.bq, wl.bk)
        assert_o_lse(o_s[h], l_s[h], om, lm, f"config 1 sparse h{h}")
    assert clear >= wl.H * nqb // 2

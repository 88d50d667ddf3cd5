"""Full workload sizes, in the launch configuration the bench uses, checked on
sampled (head, query block) tiles the oracle computes one by one: the dense
pass, the block-mass row, the selection (margin rule and kernel-precision
exactness), and the block-sparse output with the GPU's own pattern."""
import numpy as np
import pytest

import oracle as O
import block_sparse_bidirectional_select_b200 as sp
from block_sparse_bidirectional_select_b200.inputs import WORKLOADS, make_inputs
from gpu_common import MASS_RTOL, assert_o_lse, check_selection, f64

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
        keys = O.kept_keys(idx[h, i, :52], wl.bk, wl.L)
        om, lm = O.softmax_attention(qh[r0:r1], kh[keys], vh[keys], wl.scale)
        assert_o_lse(r.o[h, r0:r1], r.lse[h, r0:r1], om, lm, f"run_steps h{h} i{i}")

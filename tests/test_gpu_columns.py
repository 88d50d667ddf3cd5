"""Column-sparse path (PulseCol abstract: per-head key columns instead of
blocks) on the GPU against the fp64 oracle: the selection pass (dense O/LSE,
column mass, top-k columns), the attention over given columns, the step loop,
and a full-size 64k case on sampled rows plus invariants."""
import numpy as np
import pytest
import torch

import oracle as O
import block_sparse_bidirectional_select_b200 as sp
from block_sparse_bidirectional_select_b200 import _lib
from block_sparse_bidirectional_select_b200.inputs import WORKLOADS, make_inputs
from gpu_common import MASS_RTOL, assert_o_lse, check_selection, f64, oracle_dense_heads

pytestmark = pytest.mark.gpu


def _inputs(H, L, d, seed, structure="iid"):
    wl = WORKLOADS["tiny"].scaled(H=H, L=L, d=d, seed=seed, structure=structure)
    q, k, v = make_inputs(wl)
    return q, k, v, wl.scale


@pytest.mark.parametrize("d,L,keep,structure", [(64, 1000, 0.1, "iid"), (128, 2048, 0.05, "band"),
                                                 (128, 777, 0.3, "key_bias"), (64, 100, 0.2, "iid")])
def test_select_columns_parity(d, L, keep, structure):
    """Selection pass, column mass and kept columns against the oracle. The
    column-mass kernel takes one 128-key block per CTA: L=1000 and L=777 end
    in a ragged block, L=100 is a single ragged block."""
    H = 3
    q, k, v, scale = _inputs(H, L, d, seed=900 + d + L, structure=structure)
    pat = sp.select_columns(*(t.cuda() for t in (q, k, v)), keep=keep, return_mass=True)
    sp.device_check()
    o_ref, l_ref = oracle_dense_heads(q, k, v, scale)
    assert_o_lse(pat.o, pat.lse, o_ref, l_ref, f"column select pass d={d} L={L}")
    kc = O.column_keep(L, keep)
    assert pat.cols.shape == (H, kc)
    qh, kh = f64(q), f64(k)
    mass = pat.col_mass.cpu().numpy().astype(np.float64)
    cols = pat.cols.cpu().numpy()
    exact = 0
    for h in range(H):
        m_ref = O.column_mass(qh[h], kh[h], scale, l_ref[h])
        np.testing.assert_allclose(mass[h], m_ref, rtol=MASS_RTOL, atol=1e-6)
        exact += check_selection(cols[h], kc, m_ref, kc, f"columns h={h}")
    assert exact >= 1


@pytest.mark.parametrize("d,bk", [(64, 64), (128, 128), (128, 64)])
@pytest.mark.parametrize("kc", [1, 5, 300, 1000])
def test_column_sparse_attn_given_columns(d, bk, kc):
    H, L = 2, 1000
    q, k, v, scale = _inputs(H, L, d, seed=31 + d + kc)
    rng = np.random.default_rng(kc * 7 + d)
    cols = np.stack([np.sort(rng.choice(L, kc, replace=False)) for _ in range(H)]).astype(np.int32)
    o, lse = sp.column_sparse_attn(*(t.cuda() for t in (q, k, v)), torch.from_numpy(cols).cuda(), bk=bk)
    sp.device_check()
    qh, kh, vh = f64(q), f64(k), f64(v)
    o_ref = np.empty(qh.shape)
    l_ref = np.empty(qh.shape[:2])
    for h in range(H):
        o_ref[h], l_ref[h] = O.column_sparse_attention(qh[h], kh[h], vh[h], scale, cols[h])
    assert_o_lse(o, lse, o_ref, l_ref, f"column attention d={d} bk={bk} kc={kc}")


def test_all_columns_bitwise_equals_dense():
    H, L, d = 2, 1000, 128
    q, k, v, _ = _inputs(H, L, d, seed=4)
    qc, kc_, vc = (t.cuda() for t in (q, k, v))
    cols = torch.arange(L, dtype=torch.int32, device="cuda").repeat(H, 1).contiguous()
    o1, l1 = sp.dense_attn(qc, kc_, vc)
    o2, l2 = sp.column_sparse_attn(qc, kc_, vc, cols)
    sp.device_check()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1, l2)


def test_run_steps_columns_matches_oracle_loop():
    H, L, d = 2, 640, 64
    q, k, v, scale = _inputs(H, L, d, seed=55, structure="band")
    res = sp.run_steps_columns(*(t.cuda() for t in (q, k, v)), T=6, warmup_frac=0.5, keep=0.2,
                               refresh_every=2, time_steps=True)
    sp.device_check()
    o_ref, l_ref, kinds, pat = O.run_steps_columns(f64(q), f64(k), f64(v), scale, 0.2, 6, 0.5, 2)
    assert res.kinds == kinds
    assert all(ms > 0 for ms in res.step_ms)
    cols = res.kv_idx.cpu().numpy()
    qh, kh = f64(q), f64(k)
    for h in range(H):
        check_selection(cols[h], len(cols[h]), pat["col_mass"][h], len(cols[h]), f"run_steps h={h}")
    # the last step attends over the GPU's own cached columns
    for h in range(H):
        o_h, l_h = O.column_sparse_attention(qh[h], kh[h], f64(v)[h], scale, cols[h])
        assert_o_lse(res.o[h:h + 1], res.lse[h:h + 1], o_h[None], l_h[None], f"run_steps last step h={h}")


def test_bad_columns_are_reported_not_faulted():
    H, L, d = 1, 256, 64
    q, k, v, _ = _inputs(H, L, d, seed=3)
    bad = torch.tensor([[5, 3, 400]], dtype=torch.int32, device="cuda")  # not ascending, out of range
    sp.column_sparse_attn(*(t.cuda() for t in (q, k, v)), bad)
    with pytest.raises(sp.SparsedError) as e:
        sp.device_check()
    assert e.value.status == _lib.ERR_BAD_PATTERN


def test_fullsize_64k_sampled_rows_and_invariants():
    wl = WORKLOADS["c4_64k"]
    q, k, v = make_inputs(wl)
    qc, kc_, vc = (t.cuda() for t in (q, k, v))
    pat = sp.select_columns(qc, kc_, vc, keep=wl.keep, return_mass=True)
    o, lse = sp.column_sparse_attn(qc, kc_, vc, pat.cols)
    sp.device_check()
    kc = O.column_keep(wl.L, wl.keep)
    cols = pat.cols.cpu().numpy()
    mass = pat.col_mass.cpu().numpy().astype(np.float64)
    assert cols.shape == (wl.H, kc)
    # every query's probabilities sum to one: a head's columns hold L in total
    np.testing.assert_allclose(mass.sum(axis=1), wl.L, rtol=1e-3)
    rng = np.random.default_rng(64)
    for h in rng.choice(wl.H, 4, replace=False):
        c = cols[h]
        assert (np.diff(c) > 0).all() and c[0] >= 0 and c[-1] < wl.L
        keep = np.zeros(wl.L, dtype=bool)
        keep[c] = True
        # top-k property on the GPU's own masses (ties to the lower column)
        assert mass[h, keep].min() >= mass[h, ~keep].max()
        rows = rng.choice(wl.L, 48, replace=False)
        qh, kh, vh = f64(q[h]), f64(k[h]), f64(v[h])
        o_ref, l_ref = O.column_sparse_attention(qh[rows], kh, vh, wl.scale, c)
        assert_o_lse(o[h, rows], lse[h, rows], o_ref, l_ref, f"64k columns h={h}")

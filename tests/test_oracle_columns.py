"""Pins of the oracle's column-sparse path (PulseCol abstract: column-level
sparsity, pattern identified early and reused) against a hand-computed case,
torch float64 softmax, closed forms and brute force. CPU only."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")))
rng = np.random.default_rng(2468)


def test_column_mass_and_selection_hand_case():
    c = GOLD["column_mass_two_rows"]
    q, k = np.array(c["q"]), np.array(c["k"])
    m = O.column_mass(q, k, c["scale"], np.array(c["lse"]))
    np.testing.assert_allclose(m, c["mass"], rtol=0, atol=1e-15)
    assert O.topk_columns(m, c["keep"]).tolist() == c["cols"]
    v = rng.standard_normal((3, 2))
    _, lse = O.column_sparse_attention(q, k, v, c["scale"], c["cols"])
    assert lse[1] == pytest.approx(c["row1_lse_over_cols"], abs=1e-15)


@pytest.mark.parametrize("R,C,d", [(9, 17, 4), (40, 33, 8)])
def test_column_mass_matches_torch_softmax_column_sums(R, C, d):
    q, k = rng.standard_normal((R, d)), rng.standard_normal((C, d))
    scale = 0.41
    s = torch.from_numpy(q) @ torch.from_numpy(k).T * scale
    lse = torch.logsumexp(s, dim=-1).numpy()
    ref = torch.softmax(s, dim=-1).sum(dim=0).numpy()
    got = O.column_mass(q, k, scale, lse, chunk=7)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=0)
    # every row's probabilities sum to one, so the columns hold R in total
    assert got.sum() == pytest.approx(R, rel=1e-12)


def test_column_keep_rounding():
    assert O.column_keep(65536, 0.10) == 6554
    assert O.column_keep(8192, 0.10) == 820
    assert O.column_keep(10, 0.0) == 1
    assert O.column_keep(10, 1.0) == 10
    assert O.column_keep(30, 0.1) == 3  # 0.1f * 30 lands a hair above 3


def test_topk_columns_brute_force_and_ties():
    for _ in range(20):
        n = int(rng.integers(1, 30))
        m = np.round(rng.random(n) * 4) / 4  # many exact ties
        k = int(rng.integers(1, n + 1))
        brute = sorted(sorted(range(n), key=lambda j: (-m[j], j))[:k])
        assert O.topk_columns(m, k).tolist() == brute


def test_column_sparse_matches_explicit_mask():
    L, d = 23, 6
    q, k, v = (rng.standard_normal((L, d)) for _ in range(3))
    cols = np.array([1, 4, 5, 11, 22])
    scale = 0.3
    s = scale * (q @ k.T)
    mask = np.full(L, -np.inf)
    mask[cols] = 0.0
    sm = s + mask
    p = np.exp(sm - sm.max(axis=1, keepdims=True))
    o_ref = (p / p.sum(axis=1, keepdims=True)) @ v
    lse_ref = sm.max(axis=1) + np.log(p.sum(axis=1))
    o, lse = O.column_sparse_attention(q, k, v, scale, cols)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-13, atol=1e-13)


def test_all_columns_is_dense_bit_identical():
    L, d = 19, 5
    q, k, v = (rng.standard_normal((L, d)) for _ in range(3))
    o1, l1 = O.dense_attention(q, k, v, 0.5)
    o2, l2 = O.column_sparse_attention(q, k, v, 0.5, np.arange(L))
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_zero_query_closed_form():
    H, L, d = 2, 40, 4
    q = np.zeros((H, L, d))
    k, v = rng.standard_normal((H, L, d)), rng.standard_normal((H, L, d))
    pat = O.select_columns(q, k, v, 0.25, 0.1)
    kc = O.column_keep(L, 0.1)
    for h in range(H):
        # every probability is 1/L, so every column holds L * 1/L = 1: all tie
        np.testing.assert_allclose(pat["col_mass"][h], np.ones(L), rtol=1e-14)
        assert pat["cols"][h].tolist() == list(range(kc))
        o, lse = O.column_sparse_attention(q[h], k[h], v[h], 0.25, pat["cols"][h])
        np.testing.assert_allclose(o, np.broadcast_to(v[h, :kc].mean(axis=0), o.shape), rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(lse, math.log(kc), rtol=1e-15)


def test_planted_column_is_selected():
    L, d = 64, 8
    q = rng.standard_normal((1, L, d))
    k = rng.standard_normal((1, L, d)) * 0.1
    v = rng.standard_normal((1, L, d))
    k[0, 37] += 3.0 * q[0].mean(axis=0) / np.linalg.norm(q[0].mean(axis=0))
    pat = O.select_columns(q, k, v, 1.0, 1.0 / L)
    assert pat["cols"][0].tolist() == [37]


def test_run_steps_columns_small():
    H, L, d = 1, 32, 4
    q, k, v = (rng.standard_normal((H, L, d)) for _ in range(3))
    o, lse, kinds, pat = O.run_steps_columns(q, k, v, 0.5, 0.25, 6, 0.5, 2)
    assert kinds == [O.DENSE, O.DENSE, O.SELECT, O.SPARSE, O.SELECT, O.SPARSE]
    o_ref, l_ref = O.column_sparse_attention(q[0], k[0], v[0], 0.5, pat["cols"][0])
    assert np.array_equal(o[0], o_ref) and np.array_equal(lse[0], l_ref)
    assert len(pat["cols"][0]) == O.column_keep(L, 0.25)

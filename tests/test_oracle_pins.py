"""Pins of the fp64 oracle against things other than itself: hand-computed
fixtures (tests/golden/hand_cases.json), closed forms, brute force on tiny
inputs, invariants, and torch float64 library routines. CPU only.

A plausible slip anywhere in the oracle (a dropped term, a wrong sign or index,
a transposed operand, a wrong tie-break, an off-by-one in a block range or in
the schedule) fails at least one test here.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")))
rng = np.random.default_rng(12345)


def _rand(*shape):
    return rng.standard_normal(shape)


# ---------------------------------------------------------------- O1 dense

def test_softmax_hand_case():
    c = GOLD["softmax_four_keys"]
    o, lse = O.softmax_attention(np.array(c["q"]), np.array(c["k"]), np.array(c["v"]), c["scale"])
    np.testing.assert_allclose(o, c["o"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, c["lse"], rtol=0, atol=1e-14)


@pytest.mark.parametrize("R,C,d", [(7, 13, 5), (33, 64, 16), (1, 1, 3)])
def test_dense_matches_torch_library(R, C, d):
    q, k, v = _rand(R, d), _rand(C, d), _rand(C, d)
    scale = 0.37
    o, lse = O.softmax_attention(q, k, v, scale)
    s = torch.from_numpy(q) @ torch.from_numpy(k).T * scale
    ref_o = torch.softmax(s, dim=-1) @ torch.from_numpy(v)
    ref_lse = torch.logsumexp(s, dim=-1)
    np.testing.assert_allclose(o, ref_o.numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, ref_lse.numpy(), rtol=1e-13, atol=1e-13)


def test_probability_rows_sum_to_one():
    # With V = identity (d = number of keys) the output row IS the probability row.
    C = 40
    q, k = _rand(9, 6), _rand(C, 6) * 3
    o, _ = O.softmax_attention(q, k, np.eye(C), 0.5)
    assert (o >= 0).all()
    np.testing.assert_allclose(o.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    # and the largest score gets the largest probability (not a sign flip)
    s = 0.5 * q @ k.T
    assert (o.argmax(axis=1) == s.argmax(axis=1)).all()


def test_zero_query_closed_form():
    L, d = 50, 4
    k, v = _rand(L, d), _rand(L, d)
    o, lse = O.dense_attention(np.zeros((L, d)), k, v, 0.3)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=0), o.shape), atol=1e-14)
    np.testing.assert_allclose(lse, math.log(L), atol=1e-14)


def test_constant_value_rows():
    L, d = 30, 5
    o, _ = O.dense_attention(_rand(L, d), _rand(L, d), np.full((L, d), 2.5), 0.8)
    np.testing.assert_allclose(o, 2.5, atol=1e-13)


def test_dense_rows_subset_and_chunking():
    L, d = 70, 8
    q, k, v = _rand(L, d), _rand(L, d), _rand(L, d)
    o_all, l_all = O.dense_attention(q, k, v, 0.2, chunk=16)
    rows = [3, 69, 0, 17]
    o_s, l_s = O.dense_attention(q, k, v, 0.2, rows=rows, chunk=3)
    # BLAS may round differently for different row counts: equal to fp64 rounding
    np.testing.assert_allclose(o_s, o_all[rows], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(l_s, l_all[rows], rtol=1e-14)


def test_lse_shift_invariance():
    # adding a constant to every key score of a row shifts lse by it and leaves o
    L, d = 20, 3
    q, k, v = _rand(1, d), _rand(L, d), _rand(L, d)
    q2 = np.concatenate([q, [[1.0]]], axis=1)
    k2 = np.concatenate([k, np.full((L, 1), 2.0)], axis=1)
    o1, l1 = O.softmax_attention(q, k, v, 1.0)
    o2, l2 = O.softmax_attention(q2, k2, v, 1.0)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l2 - l1, 2.0, atol=1e-13)


# ---------------------------------------------------------------- O2 block mass

def test_block_mass_hand_case():
    c = GOLD["block_mass_two_by_two"]
    q, k = np.array(c["q"]), np.array(c["k"])
    _, lse = O.dense_attention(q, k, np.zeros((4, 1)), c["scale"])
    M = O.block_mass(q, k, c["scale"], lse, c["bq"], c["bk"])
    np.testing.assert_allclose(M, c["mass"], atol=1e-14)


def _brute_mass(q, k, scale, bq, bk):
    # independent: explicit probability matrix from torch, summed by loops
    s = torch.from_numpy(q) @ torch.from_numpy(k).T * scale
    p = torch.softmax(s, dim=-1).numpy()
    L = q.shape[0]
    nqb, nkb = -(-L // bq), -(-k.shape[0] // bk)
    M = np.zeros((nqb, nkb))
    for r in range(L):
        for c in range(k.shape[0]):
            M[r // bq, c // bk] += p[r, c]
    return M


@pytest.mark.parametrize("L,bq,bk", [(32, 8, 8), (37, 8, 4), (20, 16, 8), (5, 8, 8)])
def test_block_mass_brute_force_and_ragged(L, bq, bk):
    d = 6
    q, k = _rand(L, d), _rand(L, d)
    _, lse = O.dense_attention(q, k, np.zeros((L, 1)), 0.6)
    M = O.block_mass(q, k, 0.6, lse, bq, bk)
    np.testing.assert_allclose(M, _brute_mass(q, k, 0.6, bq, bk), rtol=1e-12, atol=1e-14)
    # each query block's row sums to its number of (valid) rows; the grid sums to L
    rows_in_block = [min(bq, L - i * bq) for i in range(M.shape[0])]
    np.testing.assert_allclose(M.sum(axis=1), rows_in_block, atol=1e-10)
    assert abs(M.sum() - L) < 1e-9


def test_block_mass_key_permutation_within_block():
    L, d, b = 32, 5, 8
    q, k = _rand(L, d), _rand(L, d)
    _, lse = O.dense_attention(q, k, np.zeros((L, 1)), 0.5)
    M = O.block_mass(q, k, 0.5, lse, b, b)
    perm = np.concatenate([rng.permutation(b) + j * b for j in range(L // b)])
    M2 = O.block_mass(q, k[perm], 0.5, lse, b, b)
    np.testing.assert_allclose(M, M2, rtol=1e-12)
    # but swapping whole blocks moves the mass columns
    sw = np.concatenate([np.arange(8, 16), np.arange(0, 8), np.arange(16, 32)])
    M3 = O.block_mass(q, k[sw], 0.5, lse, b, b)
    np.testing.assert_allclose(M3[:, [1, 0, 2, 3]], M, rtol=1e-12)


def test_block_mass_qblock_subset():
    L, d = 48, 4
    q, k = _rand(L, d), _rand(L, d)
    _, lse = O.dense_attention(q, k, np.zeros((L, 1)), 0.5)
    M = O.block_mass(q, k, 0.5, lse, 16, 8)
    np.testing.assert_array_equal(O.block_mass(q, k, 0.5, lse, 16, 8, qblocks=[2, 0]), M[[2, 0]])


# ---------------------------------------------------------------- O3 budgets

def test_uniform_keep_cases():
    for nkb, rho, k in GOLD["uniform_keep_pages_workloads"]["cases"]:
        assert O.uniform_keep(nkb, rho) == k, (nkb, rho)


@pytest.mark.parametrize("name", ["entropy_budget_three_heads", "entropy_budget_equal"])
def test_entropy_budget_hand_cases(name):
    c = GOLD[name]
    k, B = O.entropy_budget(c["entropies"], c["nkb"], c["keep"])
    assert B == c["B"]
    assert k == c["head_k"]


def test_entropy_budget_invariants():
    for trial in range(200):
        H = int(rng.integers(1, 12))
        nkb = int(rng.integers(1, 40))
        rho = float(rng.uniform(0.01, 1.0))
        E = rng.uniform(0, 3, H) * (rng.uniform(0, 1, H) > 0.2)
        k, B = O.entropy_budget(E, nkb, rho)
        assert sum(k) == B
        assert all(1 <= x <= nkb for x in k)
        assert H <= B <= H * nkb
        # monotone in entropy: a more concentrated head never gets more blocks
        for a in range(H):
            for b in range(H):
                if E[a] < E[b]:
                    assert k[a] <= k[b] + 1  # rounding can differ by one unit at most


def test_entropy_budget_one_hot_head_and_all_zero():
    # B = 20, X = 16: shares 16/3 = 5.33 for the three E=2 heads, 0 for the one-hot head
    k, B = O.entropy_budget([2.0, 0.0, 2.0, 2.0], 10, 0.5)
    assert B == 20 and k == [7, 1, 6, 6]
    # B = 10, X = 6, all entropies 0 -> even split 1.5 each -> [2,2,1,1] extra
    k, B = O.entropy_budget([0.0] * 4, 10, 0.25)
    assert k == [3, 3, 2, 2]


def test_entropy_budget_clamps_at_nkb():
    # B = 9, X = 6, cap 3: head 0 share 5.88 > 3 -> capped; 3 left split 1.5/1.5
    k, B = O.entropy_budget([10.0, 0.1, 0.1], 4, 0.75)
    assert k == [4, 3, 2]
    # overflow goes back to one-hot heads when nothing else can take it
    k, B = O.entropy_budget([0.0, 1.0, 0.0], 27, 0.654)    # B = ceil(52.97) = 53
    assert B == 53 and k == [13, 27, 13]


def test_head_entropy_closed_forms():
    assert abs(O.head_entropy(np.ones((3, 8)))) - math.log(8) < 1e-14
    assert O.head_entropy(np.array([[0.0, 5.0, 0.0]])) == 0.0
    M = np.array([[1.0, 1.0, 0.0, 0.0], [2.0, 2.0, 2.0, 2.0]])  # ln2 and ln4 -> mean 1.5 ln2
    assert abs(O.head_entropy(M) - 1.5 * math.log(2)) < 1e-14


def test_largest_remainder():
    assert O.largest_remainder(10, [1, 1, 1])[0] == [4, 3, 3]
    assert O.largest_remainder(5, [3, 1])[0] == [4, 1]        # 3.75 / 1.25
    assert O.largest_remainder(7, [0.0, 0.0])[0] == [4, 3]


# ---------------------------------------------------------------- O4 top-k

def _is_valid_topk(m, sel, k):
    sel = set(int(x) for x in sel)
    if len(sel) != k:
        return False
    for a in sel:
        for b in range(len(m)):
            if b in sel:
                continue
            if not (m[a] > m[b] or (m[a] == m[b] and a < b)):
                return False
    return True


def test_topk_brute_force_definition():
    for trial in range(300):
        n = int(rng.integers(1, 9))
        k = int(rng.integers(1, n + 1))
        m = rng.integers(0, 4, n).astype(float)  # many ties on purpose
        sel = O.topk_blocks(m, k)
        assert list(sel) == sorted(sel)
        assert _is_valid_topk(m, sel, k)
        # exhaustive: exactly one k-subset satisfies the ordered-cut definition
        valid = [c for c in itertools.combinations(range(n), k) if _is_valid_topk(m, c, k)]
        assert valid == [tuple(int(x) for x in sel)]


def test_topk_all_ties_lowest_indices():
    assert list(O.topk_blocks(np.full(10, 0.25), 4)) == [0, 1, 2, 3]


def test_topk_planted_block():
    L, d, b = 128, 16, 16
    q, k = _rand(L, d), _rand(L, d)
    i_star, j_star = 2, 5
    k[j_star * b:(j_star + 1) * b] += 3.0 * q[i_star * b:(i_star + 1) * b].mean(axis=0)
    _, lse = O.dense_attention(q, k, np.zeros((L, 1)), 0.25)
    M = O.block_mass(q, k, 0.25, lse, b, b)
    assert j_star in O.topk_blocks(M[i_star], 1)


# ---------------------------------------------------------------- O5 masked attention

def _brute_masked(q, k, v, scale, kv_idx, kv_count, bq, bk):
    # independent: explicit L x L mask of -inf, torch float64 softmax
    L = q.shape[0]
    mask = torch.full((L, k.shape[0]), float("-inf"), dtype=torch.float64)
    for r in range(L):
        i = r // bq
        for j in kv_idx[i][: kv_count[i]]:
            mask[r, j * bk: (j + 1) * bk] = 0.0
    s = torch.from_numpy(q) @ torch.from_numpy(k).T * scale + mask
    lse = torch.logsumexp(s, dim=-1)
    p = torch.softmax(s, dim=-1)
    return (p @ torch.from_numpy(v)).numpy(), lse.numpy()


@pytest.mark.parametrize("L,bq,bk", [(64, 16, 16), (60, 16, 8), (50, 8, 16)])
def test_masked_matches_explicit_mask(L, bq, bk):
    d = 7
    q, k, v = _rand(L, d), _rand(L, d), _rand(L, d)
    nqb, nkb = -(-L // bq), -(-L // bk)
    kv_idx, kv_count = [], []
    for i in range(nqb):
        c = int(rng.integers(1, nkb + 1))
        kv_idx.append(np.sort(rng.choice(nkb, c, replace=False)))
        kv_count.append(c)
    o, lse = O.masked_attention(q, k, v, 0.4, kv_idx, kv_count, bq, bk)
    ro, rl = _brute_masked(q, k, v, 0.4, kv_idx, kv_count, bq, bk)
    np.testing.assert_allclose(o, ro, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, rl, rtol=1e-13, atol=1e-13)


def test_masked_keep_all_is_dense_bit_identical():
    L, d, b = 96, 8, 16
    q, k, v = _rand(L, d), _rand(L, d), _rand(L, d)
    nb = L // b
    o, lse = O.masked_attention(q, k, v, 0.3, [np.arange(nb)] * nb, [nb] * nb, b, b)
    od, ld = O.dense_attention(q, k, v, 0.3, chunk=b)
    np.testing.assert_array_equal(o, od)
    np.testing.assert_array_equal(lse, ld)


def test_masked_lse_bounded_by_dense_and_single_block():
    L, d, b = 64, 6, 16
    q, k, v = _rand(L, d), _rand(L, d), _rand(L, d)
    nb = L // b
    idx = [np.array([j % nb]) for j in range(nb)]
    o, lse = O.masked_attention(q, k, v, 0.5, idx, [1] * nb, b, b)
    _, ld = O.dense_attention(q, k, v, 0.5)
    assert (lse <= ld + 1e-12).all()
    for i in range(nb):  # one kept block = plain softmax over that block alone
        j = i % nb
        ob, lb = O.softmax_attention(q[i * b:(i + 1) * b], k[j * b:(j + 1) * b], v[j * b:(j + 1) * b], 0.5)
        np.testing.assert_array_equal(o[i * b:(i + 1) * b], ob)
        np.testing.assert_array_equal(lse[i * b:(i + 1) * b], lb)


def test_masked_zero_query_closed_form_and_empty_list():
    L, d, b, kk = 64, 4, 8, 3
    k, v = _rand(L, d), _rand(L, d)
    nb = L // b
    M = np.full((nb, nb), b * b / L)
    idx = [O.topk_blocks(M[i], kk) for i in range(nb)]
    assert all(list(x) == [0, 1, 2] for x in idx)
    o, lse = O.masked_attention(np.zeros((L, d)), k, v, 1.0, idx, [kk] * nb, b, b)
    np.testing.assert_allclose(o, np.broadcast_to(v[: kk * b].mean(axis=0), o.shape), atol=1e-14)
    np.testing.assert_allclose(lse, math.log(kk * b), atol=1e-14)
    o, lse = O.masked_attention(np.zeros((L, d)), k, v, 1.0, idx, [0] * nb, b, b)
    assert (o == 0).all() and np.isneginf(lse).all()


# ---------------------------------------------------------------- select + O6

def test_select_pattern_uniform_small():
    H, L, d, b = 2, 64, 8, 16
    q, k, v = _rand(H, L, d), _rand(H, L, d), _rand(H, L, d)
    P = O.select_pattern(q, k, v, 0.3, b, b, 0.5, "uniform")
    assert P["mass"].shape == (H, 4, 4)
    assert (P["kv_count"] == 2).all()
    for h in range(H):
        od, ld = O.dense_attention(q[h], k[h], v[h], 0.3)
        np.testing.assert_array_equal(P["o"][h], od)
        for i in range(4):
            assert _is_valid_topk(P["mass"][h, i], P["kv_idx"][h][i], 2)


def test_select_pattern_entropy_gives_concentrated_head_fewer_blocks():
    H, L, d, b = 2, 128, 16, 16
    q, k, v = _rand(H, L, d), _rand(H, L, d), _rand(H, L, d)
    q[0] *= 0.01                         # head 0: near-uniform attention (high entropy)
    k[1] += 4.0 * q[1]                   # head 1: strongly diagonal (low entropy)
    P = O.select_pattern(q, k, v, 0.25, b, b, 0.25, "entropy")
    assert P["entropies"][0] > P["entropies"][1]
    assert P["head_k"][0] > P["head_k"][1]
    assert P["head_k"].sum() == math.ceil(0.25 * 2 * 8 - 1e-6)


def test_schedule_counts():
    for c in GOLD["schedule_counts"]["cases"]:
        kinds = O.schedule(c["T"], c["w"], c["R"])
        assert len(kinds) == c["T"]
        assert kinds.count(O.DENSE) == c["dense"]
        assert [t for t, x in enumerate(kinds) if x == O.SELECT] == c["select_at"]
        assert kinds.count(O.SPARSE) == c["sparse"]


def test_run_steps_small():
    H, L, d, b = 2, 48, 8, 16
    q, k, v = _rand(H, L, d), _rand(H, L, d), _rand(H, L, d)
    o, lse, kinds, pat = O.run_steps(q, k, v, 0.3, b, b, 0.4, "uniform", T=5, warmup_frac=0.4)
    assert kinds == [O.DENSE, O.SELECT, O.SPARSE, O.SPARSE, O.SPARSE]
    for h in range(H):
        om, lm = O.masked_attention(q[h], k[h], v[h], 0.3, pat["kv_idx"][h], pat["kv_count"][h], b, b)
        np.testing.assert_array_equal(o[h], om)
        np.testing.assert_array_equal(lse[h], lm)

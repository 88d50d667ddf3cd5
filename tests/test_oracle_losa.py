"""Pins of the oracle's block-wise path (LoSA: Locality Aware Sparse Attention
for Block-Wise Diffusion Language Models, sections 1-3: active tokens by query
MSE, the union of their selections, reuse of the cached prefix output for
stable tokens, prefix and in-block parts merged by online softmax) against
hand-computed cases, torch float64 softmax over the concatenated keys, closed
forms, invariants and brute force. CPU only."""
import json
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")))
rng = np.random.default_rng(97531)


def torch_attention(q, k, v, scale):
    """Library reference: torch float64 softmax attention and logsumexp."""
    s = torch.from_numpy(np.asarray(q, dtype=np.float64)) @ torch.from_numpy(np.asarray(k, dtype=np.float64)).T
    s = s * scale
    p = torch.softmax(s, dim=-1)
    return (p @ torch.from_numpy(np.asarray(v, dtype=np.float64))).numpy(), torch.logsumexp(s, dim=-1).numpy()


def test_merge_hand_case():
    c = GOLD["losa_merge_one_prefix_one_block_key"]
    q = np.array(c["q"])
    o1, l1 = O.softmax_attention(q, np.array(c["k_pre"]), np.array(c["v_pre"]), c["scale"])
    o2, l2 = O.softmax_attention(q, np.array(c["k_blk"]), np.array(c["v_blk"]), c["scale"])
    assert o1[0, 0] == 2.0 and l1[0] == pytest.approx(1.0, abs=1e-15)
    o, lse = O.merge_partials(o1, l1, o2, l2)
    np.testing.assert_allclose(o, c["o"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, c["lse"], rtol=0, atol=1e-15)


@pytest.mark.parametrize("n1,n2,d", [(7, 5, 4), (40, 3, 16), (1, 1, 2)])
def test_merge_equals_attention_over_both_key_sets(n1, n2, d):
    R = 6
    q = rng.standard_normal((R, d))
    k1, v1 = rng.standard_normal((n1, d)) * 2, rng.standard_normal((n1, d))
    k2, v2 = rng.standard_normal((n2, d)) * 2, rng.standard_normal((n2, d))
    scale = 0.37
    o1, l1 = O.softmax_attention(q, k1, v1, scale)
    o2, l2 = O.softmax_attention(q, k2, v2, scale)
    o, lse = O.merge_partials(o1, l1, o2, l2)
    ref_o, ref_l = torch_attention(q, np.vstack([k1, k2]), np.vstack([v1, v2]), scale)
    np.testing.assert_allclose(o, ref_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_l, rtol=0, atol=1e-12)
    # the order of the parts does not matter
    o_sw, l_sw = O.merge_partials(o2, l2, o1, l1)
    np.testing.assert_allclose(o_sw, o, rtol=0, atol=1e-14)
    np.testing.assert_allclose(l_sw, lse, rtol=0, atol=1e-14)


def test_merge_with_an_empty_part_is_the_other_part():
    o1 = rng.standard_normal((3, 4))
    l1 = rng.standard_normal(3)
    empty_o, empty_l = np.zeros((3, 4)), np.full(3, -np.inf)
    o, lse = O.merge_partials(o1, l1, empty_o, empty_l)
    np.testing.assert_array_equal(o, o1)
    np.testing.assert_array_equal(lse, l1)
    o, lse = O.merge_partials(empty_o, empty_l, empty_o, empty_l)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


def test_query_mse_hand_case_and_strict_threshold():
    c = GOLD["losa_query_mse_two_tokens"]
    mse = O.query_mse(np.array(c["q_t"]), np.array(c["q_prev"]))
    np.testing.assert_array_equal(mse, c["mse"])
    assert O.active_tokens(mse, 0.125).tolist() == c["active_tau_0.125"]
    assert O.active_tokens(mse, 0.1).tolist() == c["active_tau_0.1"]


def test_query_mse_closed_forms():
    H, B, d = 3, 5, 8
    q = np.round(rng.standard_normal((H, B, d)) * 64) / 64
    np.testing.assert_array_equal(O.query_mse(q, q), np.zeros(B))
    np.testing.assert_array_equal(O.query_mse(q, q - 0.5), np.full(B, 0.25))
    p = q.copy()
    p[1, 3, 5] += 0.25  # one element of token 3 changed
    expect = np.zeros(B)
    expect[3] = 0.0625 / (H * d)
    np.testing.assert_allclose(O.query_mse(p, q), expect, rtol=1e-15, atol=0)


def test_threshold_is_the_fp32_value():
    # tau = 0.1 reaches the oracle as fp32(0.1) = 0.100000001490116..., above the double 0.1
    assert not O.active_tokens(np.array([0.1]), 0.1)[0]
    assert O.active_tokens(np.array([0.1000000015]), 0.1)[0]


@pytest.mark.parametrize("B,P,bk", [(5, 23, 4), (9, 64, 16), (3, 50, 64)])
def test_token_block_mass_matches_torch_softmax_block_sums(B, P, bk):
    d = 6
    q, k = rng.standard_normal((B, d)), rng.standard_normal((P, d))
    scale = 0.5
    s = torch.from_numpy(q) @ torch.from_numpy(k).T * scale
    lse = torch.logsumexp(s, dim=-1).numpy()
    p = torch.softmax(s, dim=-1).numpy()
    nkb = -(-P // bk)
    ref = np.stack([p[:, j * bk:(j + 1) * bk].sum(axis=1) for j in range(nkb)], axis=1)
    got = O.token_block_mass(q, k, scale, lse, bk)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-15)
    # with the row's own LSE every token's masses sum to one
    np.testing.assert_allclose(got.sum(axis=1), np.ones(B), rtol=1e-12)


def test_token_block_mass_ignores_key_order_inside_a_block():
    B, P, bk, d = 4, 32, 8, 5
    q, k = rng.standard_normal((B, d)), rng.standard_normal((P, d))
    lse = rng.standard_normal(B)
    perm = np.arange(P)
    for j in range(P // bk):
        perm[j * bk:(j + 1) * bk] = rng.permutation(np.arange(j * bk, (j + 1) * bk))
    a = O.token_block_mass(q, k, 0.3, lse, bk)
    b = O.token_block_mass(q, k[perm], 0.3, lse, bk)
    np.testing.assert_allclose(a, b, rtol=1e-13)


def test_token_select_brute_force_with_ties():
    for _ in range(20):
        B, nkb = int(rng.integers(1, 6)), int(rng.integers(1, 12))
        M = np.round(rng.random((B, nkb)) * 3) / 3  # many exact ties
        k = int(rng.integers(1, nkb + 3))
        sel = O.token_select(M, k)
        kk = min(k, nkb)
        assert sel.shape == (B, kk)
        for b in range(B):
            brute = sorted(sorted(range(nkb), key=lambda j: (-M[b, j], j))[:kk])
            assert sel[b].tolist() == brute


def test_planted_block_is_selected():
    B, P, bk, d = 6, 64, 8, 16
    q = rng.standard_normal((B, d))
    k = rng.standard_normal((P, d)) * 0.1
    b_star, j_star = 4, 5
    k[j_star * bk:(j_star + 1) * bk] += 3.0 * q[b_star] / np.linalg.norm(q[b_star])
    s = q @ k.T * 0.25
    lse = np.log(np.exp(s).sum(axis=1))
    sel = O.token_select(O.token_block_mass(q, k, 0.25, lse, bk), 1)
    assert sel[b_star, 0] == j_star


def test_kv_union_brute_force_and_bounds():
    for _ in range(30):
        B, nkb = int(rng.integers(1, 10)), int(rng.integers(1, 20))
        k = int(rng.integers(1, nkb + 1))
        sel = np.stack([np.sort(rng.choice(nkb, k, replace=False)) for _ in range(B)]).astype(np.int32)
        active = rng.random(B) < 0.5
        u = O.kv_union(sel, active)
        brute = set()
        for b in range(B):
            if active[b]:
                brute |= set(sel[b].tolist())
        assert u.tolist() == sorted(brute)
        na = int(active.sum())
        assert len(u) <= min(nkb, na * k)
        if na:
            assert len(u) >= k
        else:
            assert len(u) == 0


def _concat_reference(q, k_pre, v_pre, k, v, scale):
    """Every block token over all prefix keys and all block keys (torch)."""
    H = q.shape[0]
    o = np.empty(q.shape)
    lse = np.empty(q.shape[:2])
    for h in range(H):
        o[h], lse[h] = torch_attention(q[h], np.vstack([k_pre[h], k[h]]), np.vstack([v_pre[h], v[h]]), scale)
    return o, lse


def _block_case(H=2, P=45, B=7, d=8, T=4, seed=5):
    r = np.random.default_rng(seed)
    k_pre, v_pre = r.standard_normal((H, P, d)), r.standard_normal((H, P, d))
    qs = np.empty((T, H, B, d))
    qs[0] = r.standard_normal((H, B, d))
    for t in range(1, T):
        qs[t] = qs[t - 1] + r.standard_normal((H, B, d)) * 0.01
        qs[t][:, t % B] += r.standard_normal((H, d))  # one active token per step
    ks = r.standard_normal((T, H, B, d))
    vs = r.standard_normal((T, H, B, d))
    return k_pre, v_pre, qs, ks, vs


def test_init_step_is_dense_attention_over_prefix_and_block():
    k_pre, v_pre, qs, ks, vs = _block_case()
    r = O.losa_init(qs[0], ks[0], vs[0], k_pre, v_pre, 0.4, 8, 2)
    ref_o, ref_l = _concat_reference(qs[0], k_pre, v_pre, ks[0], vs[0], 0.4)
    np.testing.assert_allclose(r["o"], ref_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["lse"], ref_l, rtol=0, atol=1e-12)
    assert r["state"]["sel"].shape == (2, 7, 2)


def test_every_token_active_and_every_block_selected_is_dense():
    k_pre, v_pre, qs, ks, vs = _block_case()
    nkb = -(-45 // 8)
    first = O.losa_init(qs[0], ks[0], vs[0], k_pre, v_pre, 0.4, 8, nkb)
    r = O.losa_step(qs[1], ks[1], vs[1], qs[0], k_pre, v_pre, 0.4, 8, 0.0, first["state"])
    # tau = 0 and every query changed: all active, union = all blocks
    assert r["active"].all()
    assert all(u.tolist() == list(range(nkb)) for u in r["union"])
    ref_o, ref_l = _concat_reference(qs[1], k_pre, v_pre, ks[1], vs[1], 0.4)
    np.testing.assert_allclose(r["o"], ref_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["lse"], ref_l, rtol=0, atol=1e-12)


def test_no_active_token_reuses_the_whole_cache():
    k_pre, v_pre, qs, ks, vs = _block_case()
    first = O.losa_init(qs[0], ks[0], vs[0], k_pre, v_pre, 0.4, 8, 2)
    o_pre = first["state"]["o_pre"].copy()
    lse_pre = first["state"]["lse_pre"].copy()
    r = O.losa_step(qs[1], ks[1], vs[1], qs[0], k_pre, v_pre, 0.4, 8, 1e9, first["state"])
    assert not r["active"].any() and all(len(u) == 0 for u in r["union"])
    np.testing.assert_array_equal(first["state"]["o_pre"], o_pre)
    np.testing.assert_array_equal(first["state"]["lse_pre"], lse_pre)
    # output = the cached prefix part merged with this step's block part
    for h in range(2):
        o_s, l_s = torch_attention(qs[1][h], ks[1][h], vs[1][h], 0.4)
        o, lse = O.merge_partials(o_pre[h], lse_pre[h], o_s, l_s)
        np.testing.assert_allclose(r["o"][h], o, rtol=0, atol=1e-12)
        np.testing.assert_allclose(r["lse"][h], lse, rtol=0, atol=1e-12)


def test_active_token_attends_to_the_union_stable_token_keeps_its_cache():
    k_pre, v_pre, qs, ks, vs = _block_case()
    scale, bk, tau = 0.4, 8, 0.05
    first = O.losa_init(qs[0], ks[0], vs[0], k_pre, v_pre, scale, bk, 2)
    st = first["state"]
    cached = st["o_pre"].copy()
    r = O.losa_step(qs[1], ks[1], vs[1], qs[0], k_pre, v_pre, scale, bk, tau, st)
    act = r["active"]
    assert act.tolist() == [b == 1 for b in range(7)]  # the planted change of step 1
    for h in range(2):
        u = r["union"][h]
        assert u.tolist() == sorted(set(st["sel"][h][1].tolist()))
        keys = [c for j in u for c in range(j * bk, min((j + 1) * bk, 45))]
        o_a, l_a = torch_attention(qs[1][h][[1]], k_pre[h][keys], v_pre[h][keys], scale)
        np.testing.assert_allclose(st["o_pre"][h][1], o_a[0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(st["lse_pre"][h][1], l_a[0], rtol=0, atol=1e-12)
        stable = [b for b in range(7) if b != 1]
        np.testing.assert_array_equal(st["o_pre"][h][stable], cached[h][stable])


def test_block_run_records_and_density_bound():
    k_pre, v_pre, qs, ks, vs = _block_case(T=5)
    r = O.losa_block(qs, ks, vs, k_pre, v_pre, 0.4, 8, 2, 0.05)
    nkb = -(-45 // 8)
    assert r["active"][0].all() and (r["union_count"][0] == nkb).all()
    for t in range(1, 5):
        na = int(r["active"][t].sum())
        assert na == 1 and r["active"][t][t % 7]
        assert (r["union_count"][t] <= min(nkb, na * 2)).all()
    ref_o, ref_l = _concat_reference(qs[0], k_pre, v_pre, ks[0], vs[0], 0.4)
    np.testing.assert_allclose(r["o"][0], ref_o, rtol=0, atol=1e-12)


def test_block_run_hand_case():
    c = GOLD["losa_block_three_steps"]
    r = O.losa_block(np.array(c["qs"]), np.array(c["ks"]), np.array(c["vs"]), np.array(c["k_pre"]),
                     np.array(c["v_pre"]), c["scale"], c["bk"], c["n_sel"], c["tau"])
    np.testing.assert_allclose(r["o"][:, 0, 0, 0], c["o"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(r["lse"][:, 0, 0], c["lse"], rtol=0, atol=1e-14)
    assert r["active"].tolist() == c["active"]
    assert r["state"]["sel"][0, 0].tolist() == c["sel"]
    np.testing.assert_allclose(r["state"]["o_pre"][0, :, 0], c["o_pre_after"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(r["state"]["lse_pre"][0], c["lse_pre_after"], rtol=0, atol=1e-14)
    assert r["union_count"].tolist() == [[2], [1], [0]]

"""Property-based pins of the oracle (hypothesis): identities and invariants
that hold for every input the strategies draw, not only for the fixed cases
of the other pin files. CPU only, a few seconds.

* the LSE merge of two disjoint key sets is attention over their union
  (torch float64), whatever the split, empty parts included;
* adding key blocks never lowers a row's LSE (log-sum-exp over a superset);
* the entropy budget always spends exactly B blocks, keeps 1 <= k_h <= nkb,
  and never gives a head fewer blocks than a head of lower entropy;
* top-k keeps the k largest in the order (mass desc, index asc);
* the union over active tokens grows with the active set;
* the query MSE scales with the square of an exact scale factor.
"""
import math

import numpy as np
import torch
from hypothesis import assume, given, settings
from hypothesis import strategies as st

import oracle as O

SETTINGS = settings(max_examples=60, deadline=None)


def _torch_attention(q, k, v, scale):
    s = torch.from_numpy(q) @ torch.from_numpy(k).T * scale
    return (torch.softmax(s, -1) @ torch.from_numpy(v)).numpy(), torch.logsumexp(s, -1).numpy()


@SETTINGS
@given(seed=st.integers(0, 2 ** 31 - 1), n=st.integers(1, 24), d=st.integers(1, 8), rows=st.integers(1, 4),
       cut=st.floats(0.0, 1.0), scale=st.floats(0.05, 2.0))
def test_merge_of_any_split_is_attention_over_the_union(seed, n, d, rows, cut, scale):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((rows, d))
    k = rng.standard_normal((n, d)) * 2
    v = rng.standard_normal((n, d))
    perm = rng.permutation(n)
    m = int(round(cut * n))
    a, b = perm[:m], perm[m:]
    o1, l1 = O.softmax_attention(q, k[a], v[a], scale)
    o2, l2 = O.softmax_attention(q, k[b], v[b], scale)
    o, lse = O.merge_partials(o1, l1, o2, l2)
    ref_o, ref_l = _torch_attention(q, k, v, scale)
    np.testing.assert_allclose(o, ref_o, rtol=0, atol=1e-11)
    np.testing.assert_allclose(lse, ref_l, rtol=0, atol=1e-11)


@SETTINGS
@given(seed=st.integers(0, 2 ** 31 - 1), L=st.integers(2, 90), bk=st.sampled_from([4, 8, 16]),
       extra=st.integers(1, 5))
def test_more_key_blocks_never_lower_the_lse(seed, L, bk, extra):
    rng = np.random.default_rng(seed)
    d = 4
    q, k, v = (rng.standard_normal((L, d)) for _ in range(3))
    nkb = O.n_blocks(L, bk)
    small = np.sort(rng.choice(nkb, max(1, nkb // 3), replace=False))
    rest = np.setdiff1d(np.arange(nkb), small)
    big = np.sort(np.concatenate([small, rest[:extra]]))
    nqb = O.n_blocks(L, bk)
    _, l_small = O.masked_attention(q, k, v, 0.5, [small] * nqb, [len(small)] * nqb, bk, bk)
    _, l_big = O.masked_attention(q, k, v, 0.5, [big] * nqb, [len(big)] * nqb, bk, bk)
    assert np.all(l_big >= l_small - 1e-12)


@SETTINGS
@given(H=st.integers(1, 24), nkb=st.integers(1, 64),
       keep=st.sampled_from([0.01, 0.05, 0.1, 0.25, 0.5, 0.9, 1.0]),
       ent=st.lists(st.floats(0.0, 8.0), min_size=24, max_size=24))
def test_entropy_budget_invariants(H, nkb, keep, ent):
    e = ent[:H]
    k, _ = O.entropy_budget(e, nkb, keep)
    k = [int(x) for x in k]
    rho = float(np.float32(keep))
    B = min(max(math.ceil(rho * H * nkb - 1e-6), H), H * nkb)
    assert sum(k) == B
    assert all(1 <= x <= nkb for x in k)
    for a in range(H):
        for b in range(H):
            if e[a] > e[b]:
                assert k[a] >= k[b], (e, k)


@SETTINGS
@given(total=st.integers(0, 5000), w=st.lists(st.one_of(st.floats(0.0, 10.0), st.sampled_from([0.1, 1 / 3, 0.7, 1.0])),
                                                min_size=1, max_size=40))
def test_largest_remainder_against_exact_rationals(total, w):
    """Largest remainder against the same split in exact rational arithmetic
    (fractions.Fraction of the same fp64 weights): every head gets the floor
    or the ceiling of its exact quota, the shares sum to the total, and where
    the exact fractional parts at the cut are separated the two agree."""
    from fractions import Fraction
    base, quota = O.largest_remainder(total, w)
    wf = [Fraction(x) for x in w]
    if sum(wf) == 0:
        wf = [Fraction(1)] * len(w)
    qf = [total * x / sum(wf) for x in wf]
    fl = [math.floor(x) for x in qf]
    rem = total - sum(fl)
    assert sum(base) == total
    assert all(b in (f, f + 1) for b, f in zip(base, fl))
    order = sorted(range(len(w)), key=lambda a: (-(qf[a] - fl[a]), a))
    fr = sorted((qf[a] - fl[a] for a in range(len(w))), reverse=True)
    separated = rem == 0 or rem == len(w) or fr[rem - 1] - fr[rem] > Fraction(1, 10 ** 9)
    if separated and all(abs(Fraction(q) - x) < Fraction(1, 10 ** 6) for q, x in zip(quota, qf)):
        exact = list(fl)
        for a in order[:rem]:
            exact[a] += 1
        assert base == exact, (total, w)


@SETTINGS
@given(seed=st.integers(0, 2 ** 31 - 1), n=st.integers(1, 40), k=st.integers(1, 40), levels=st.integers(1, 6))
def test_topk_blocks_is_the_head_of_the_order(seed, n, k, levels):
    rng = np.random.default_rng(seed)
    m = rng.integers(0, levels, n) / levels  # few distinct values: many ties
    kk = min(k, n)
    got = O.topk_blocks(m, kk).tolist()
    assert got == sorted(got) and len(set(got)) == kk
    order = sorted(range(n), key=lambda j: (-m[j], j))
    assert got == sorted(order[:kk])
    # everything kept is at least as large as everything left out
    out = [j for j in range(n) if j not in got]
    if out:
        assert min(m[got]) >= max(m[out])


@SETTINGS
@given(seed=st.integers(0, 2 ** 31 - 1), B=st.integers(1, 12), nkb=st.integers(1, 30), n_sel=st.integers(1, 6))
def test_union_grows_with_the_active_set(seed, B, nkb, n_sel):
    rng = np.random.default_rng(seed)
    k = min(n_sel, nkb)
    sel = np.stack([np.sort(rng.choice(nkb, k, replace=False)) for _ in range(B)]).astype(np.int32)
    act = rng.random(B) < 0.5
    u = set(O.kv_union(sel, act).tolist())
    for b in range(B):
        more = act.copy()
        more[b] = True
        u2 = set(O.kv_union(sel, more).tolist())
        assert u <= u2 and set(sel[b].tolist()) <= u2


@SETTINGS
@given(seed=st.integers(0, 2 ** 31 - 1), H=st.integers(1, 4), B=st.integers(1, 6), d=st.integers(1, 8),
       p=st.integers(-4, 4))
def test_query_mse_scales_with_the_square_of_an_exact_factor(seed, H, B, d, p):
    rng = np.random.default_rng(seed)
    base = np.round(rng.standard_normal((H, B, d)) * 256) / 256
    delta = np.round(rng.standard_normal((H, B, d)) * 256) / 256
    assume(np.any(delta != 0))
    c = 2.0 ** p  # a power of two: every product and square below is exact
    a = O.query_mse(base + delta, base)
    b = O.query_mse(base + c * delta, base)
    np.testing.assert_allclose(b, c * c * a, rtol=1e-14, atol=0)

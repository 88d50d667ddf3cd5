"""GPU parity of the per-step queries (inputs that change across the
denoising steps): the drifted queries bit for bit against the oracle, the
denoising loop with drift against the oracle, and the loop's fused selection
against the separate selection pass under drift, within the bound that the
stale LSE of the fused pass implies."""
import math

import numpy as np
import pytest
import torch

import oracle as O
import block_sparse_bidirectional_select_b200 as sp
from block_sparse_bidirectional_select_b200.inputs import WORKLOADS, make_inputs
from gpu_common import SELECT_MARGIN, assert_o_lse, f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("seed,t,amp", [(0, 0, 2 ** -6), (12345, 7, 2 ** -6), (2 ** 31 + 11, 1000, 2 ** -4),
                                        (99, 3, 0.0)])
def test_drift_queries_bit_exact(seed, t, amp):
    wl = WORKLOADS["tiny"].scaled(H=3, L=1000, d=128, seed=77)
    q, _, _ = make_inputs(wl)
    got = sp.drift_queries(q.cuda(), seed, t, amp)
    sp.device_check()
    ref = O.drift_queries(f64(q), seed, t, amp)
    assert np.array_equal(got.to(torch.float64).cpu().numpy(), ref)


def _lse(q, k, v, scale):
    return np.stack([O.dense_attention(q[h], k[h], v[h], scale)[1] for h in range(q.shape[0])])


def _check_loop_selection(idx, cnt, mass_ref, k, slack, what):
    """Selections of a fused pass whose row masses are scaled by factors
    within [exp(-slack/2), exp(slack/2)]: equal to the oracle where the margin
    exceeds 1 - exp(-slack) (plus the usual tolerance), else every chosen block
    within that band of the k-th mass."""
    n = len(mass_ref)
    sel = [int(x) for x in idx[:k]]
    assert int(cnt) == k and all(a < b for a, b in zip(sel, sel[1:])) and all(0 <= j < n for j in sel), what
    srt = np.sort(mass_ref)[::-1]
    mk, mk1 = srt[k - 1], (srt[k] if k < n else -math.inf)
    margin = (mk - mk1) / mk
    band = 1 - math.exp(-slack) + SELECT_MARGIN
    if margin > band:
        assert sel == [int(x) for x in O.topk_blocks(mass_ref, k)], (what, margin, band)
        return True
    assert all(mass_ref[j] >= mk * (1 - band) for j in sel), what
    return False


@pytest.mark.parametrize("d,b,L", [(64, 64, 768), (128, 128, 1024)])
def test_run_steps_drift_against_oracle(d, b, L):
    wl = WORKLOADS["tiny"].scaled(H=2, L=L, d=d, bq=b, bk=b, seed=81 + d, structure="band")
    q, k, v = make_inputs(wl)
    qc, kc, vc = (t.cuda() for t in (q, k, v))
    T, w, R, keep, seed = 8, 0.3, 2, 0.25, 4242   # D D S P S P S P
    r = sp.run_steps(qc, kc, vc, T=T, warmup_frac=w, keep=keep, refresh_every=R, bq=b, bk=b, drift_seed=seed)
    sp.device_check()
    kinds = O.schedule(T, w, R)
    assert r.kinds == kinds and kinds[-1] == O.SPARSE
    qh, kh, vh = f64(q), f64(k), f64(v)
    t_sel = [t for t, kd in enumerate(kinds) if kd == O.SELECT]
    # the last selection (fused: its pass weights with the LSE of the full pass two steps before)
    t_last, t_prev = t_sel[-1], t_sel[-2]
    q_last, q_prev = O.drift_queries(qh, seed, t_last), O.drift_queries(qh, seed, t_prev)
    lse_last = _lse(q_last, kh, vh, wl.scale)
    delta = float(np.abs(lse_last - _lse(q_prev, kh, vh, wl.scale)).max())
    assert 0 < delta < 0.5
    idx, cnt = r.kv_idx.cpu().numpy(), r.kv_count.cpu().numpy()
    kk = O.uniform_keep(-(-L // b), keep)
    clear = 0
    for h in range(wl.H):
        mass = O.block_mass(q_last[h], kh[h], wl.scale, lse_last[h], b, b)
        for i in range(mass.shape[0]):
            clear += _check_loop_selection(idx[h, i], cnt[h, i], mass[i], kk, 2 * delta, f"h{h} i{i}")
    assert clear > 0
    # the last step: masked attention over step T-1's queries with the loop's pattern
    q_T = O.drift_queries(qh, seed, T - 1)
    for h in range(wl.H):
        lists = [idx[h, i, :cnt[h, i]] for i in range(idx.shape[1])]
        om, lm = O.masked_attention(q_T[h], kh[h], vh[h], wl.scale, lists, cnt[h], b, b)
        assert_o_lse(r.o[h], r.lse[h], om, lm, f"drift last step h{h}")


def test_fused_selection_under_drift_matches_separate_pass_within_the_bound():
    H, L, d, b = 4, 1536, 128, 128
    wl = WORKLOADS["tiny"].scaled(H=H, L=L, d=d, bq=b, bk=b, seed=93, structure="band")
    q, k, v = make_inputs(wl)
    qc, kc, vc = (t.cuda() for t in (q, k, v))
    T, w, R, keep, seed = 6, 0.3, 1, 0.25, 7   # D S S S S S: every select after the first is fused
    kw = dict(T=T, warmup_frac=w, keep=keep, refresh_every=R, bq=b, bk=b, drift_seed=seed)
    small = torch.empty(sp.workspace_bytes(H, L, b, b), dtype=torch.uint8, device="cuda")
    r_fused = sp.run_steps(qc, kc, vc, **kw)
    r_sep = sp.run_steps(qc, kc, vc, workspace=small, **kw)
    sp.device_check()
    assert r_fused.kinds == r_sep.kinds and r_fused.kinds[-1] == O.SELECT
    # the separate pass is exact; the fused one scales row r's masses by
    # exp(lse_r(T-1) - lse_r(T-2)): its selection is the same wherever the
    # margin exceeds 1 - exp(-2 * max |lse change|)
    qh, kh, vh = f64(q), f64(k), f64(v)
    q1, q0 = O.drift_queries(qh, seed, T - 1), O.drift_queries(qh, seed, T - 2)
    delta = float(np.abs(_lse(q1, kh, vh, wl.scale) - _lse(q0, kh, vh, wl.scale)).max())
    band = 1 - math.exp(-2 * delta) + SELECT_MARGIN
    p = sp.select_pattern(sp.drift_queries(qc, seed, T - 1), kc, vc, keep=keep, bq=b, bk=b, return_mass=True)
    sp.device_check()
    assert torch.equal(p.kv_idx, r_sep.kv_idx) and torch.equal(p.kv_count, r_sep.kv_count)
    mass = p.block_mass
    ms = torch.sort(mass, dim=-1, descending=True).values
    kk = O.uniform_keep(L // b, keep)
    margin = (ms[..., kk - 1] - ms[..., kk]) / ms[..., kk - 1]
    clear = margin > band
    same = (r_fused.kv_idx == r_sep.kv_idx).all(dim=-1)
    assert bool(same[clear].all())
    assert clear.float().mean().item() > 0.25   # the bound is conservative; the check must not be vacuous
    picked = torch.gather(mass, -1, r_fused.kv_idx.long())
    assert bool((picked >= (ms[..., kk - 1] * (1 - band))[..., None]).all())

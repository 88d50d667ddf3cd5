"""Block-wise generation with active-token reuse (LoSA: Locality Aware Sparse
Attention for Block-Wise Diffusion Language Models, section 3) on the GPU
against the fp64 oracle: the dense first step (output, cache, per-token block
mass and selection), later steps (active flags, unions, cache updates,
outputs), whole block runs, the split count, degenerate cases, and the
full-size block on sampled rows."""
import numpy as np
import pytest
import torch

import oracle as O
import block_sparse_bidirectional_select_b200 as sp
from block_sparse_bidirectional_select_b200 import _lib
from block_sparse_bidirectional_select_b200.inputs import BLOCK_WORKLOADS, make_block_inputs
from gpu_common import MASS_RTOL, assert_o_lse, check_selection, f64

pytestmark = pytest.mark.gpu

MSE_MARGIN = 1e-9  # relative: closer to tau than this, either classification is correct


def _case(H, P, B, d, bq, bk, n_sel, T=3, seed=0):
    wl = BLOCK_WORKLOADS["losa_tiny"].scaled(H=H, P=P, B=B, d=d, bq=bq, bk=bk, n_sel=n_sel, T=T,
                                             seed=2100 + seed)
    return wl, make_block_inputs(wl)


def _cuda(*ts):
    return [t.cuda() for t in ts]


def _oracle_init(wl, k_pre, v_pre, qs, ks, vs, sel=None):
    return O.losa_init(f64(qs[0]), f64(ks[0]), f64(vs[0]), f64(k_pre), f64(v_pre), wl.scale, wl.bk, wl.n_sel,
                       sel=sel)


def _check_sel(sel_gpu, mass_ref, n_sel, what):
    exact = 0
    H, B, _ = mass_ref.shape
    k = min(n_sel, mass_ref.shape[2])
    for h in range(H):
        for b in range(B):
            exact += check_selection(sel_gpu[h, b], k, mass_ref[h, b], k, f"{what} h={h} b={b}")
    return exact


CASES = [
    # H, P, B, d, bq, bk, n_sel
    (2, 1000, 48, 64, 64, 64, 3),
    (2, 4096, 128, 128, 64, 128, 2),
    (3, 777, 100, 128, 128, 64, 4),
    (2, 2048, 64, 128, 64, 64, 40),   # more blocks per token than the union can split finely
]


@pytest.mark.parametrize("H,P,B,d,bq,bk,n_sel", CASES)
@pytest.mark.parametrize("splits", [None, 1])
def test_init_parity(H, P, B, d, bq, bk, n_sel, splits):
    wl, (k_pre, v_pre, qs, ks, vs) = _case(H, P, B, d, bq, bk, n_sel, seed=P + B)
    kp, vp, q0, k0, v0 = _cuda(k_pre, v_pre, qs[0], ks[0], vs[0])
    o, lse, st, mass = sp.losa_init(q0, k0, v0, kp, vp, n_sel=n_sel, bq=bq, bk=bk, splits=splits,
                                    return_mass=True)
    sp.device_check()
    ref = _oracle_init(wl, k_pre, v_pre, qs, ks, vs)
    what = f"init H={H} P={P} B={B} d={d} bq={bq} bk={bk} splits={st.splits}"
    assert_o_lse(o, lse, ref["o"], ref["lse"], what)
    assert_o_lse(st.o_cache, st.lse_cache, ref["state"]["o_pre"], ref["state"]["lse_pre"], what + " cache")
    np.testing.assert_allclose(mass.cpu().numpy(), ref["mass"], rtol=MASS_RTOL, atol=1e-7)
    exact = _check_sel(st.sel.cpu().numpy(), ref["mass"], n_sel, what)
    assert exact >= H * B // 2


def _state_from(st):
    return dict(o_pre=f64(st.o_cache), lse_pre=st.lse_cache.cpu().numpy().astype(np.float64),
                sel=st.sel.cpu().numpy())


def _assert_active(active_gpu, q, q_prev, tau):
    mse = O.query_mse(f64(q), f64(q_prev))
    ref = O.active_tokens(mse, tau)
    t32 = float(np.float32(tau))
    clear = np.abs(mse - t32) > MSE_MARGIN * max(t32, 1e-30)
    got = active_gpu.cpu().numpy().astype(bool)
    assert (got[clear] == ref[clear]).all(), f"active flags {got.astype(int)} != {ref.astype(int)}"
    return got


@pytest.mark.parametrize("H,P,B,d,bq,bk,n_sel", CASES)
def test_step_parity(H, P, B, d, bq, bk, n_sel):
    wl, (k_pre, v_pre, qs, ks, vs) = _case(H, P, B, d, bq, bk, n_sel, T=3, seed=7 * P + B)
    kp, vp = _cuda(k_pre, v_pre)
    q0, k0, v0 = _cuda(qs[0], ks[0], vs[0])
    _, _, st = sp.losa_init(q0, k0, v0, kp, vp, n_sel=n_sel, bq=bq, bk=bk)
    sp.device_check()
    ref_state = _oracle_init(wl, k_pre, v_pre, qs, ks, vs, sel=st.sel.cpu().numpy())["state"]
    for t in (1, 2):
        q, k, v, qp = _cuda(qs[t], ks[t], vs[t], qs[t - 1])
        r = sp.losa_step(q, k, v, qp, kp, vp, st, wl.tau, return_union=True)
        sp.device_check()
        act = _assert_active(r.active, qs[t], qs[t - 1], wl.tau)
        assert 0 < act.sum() < B
        ref = O.losa_step(f64(qs[t]), f64(ks[t]), f64(vs[t]), f64(qs[t - 1]), f64(k_pre), f64(v_pre), wl.scale,
                          wl.bk, wl.tau, ref_state)
        assert (ref["active"] == act).all()
        ucount = r.union_count.cpu().numpy()
        uidx = r.union_idx.cpu().numpy()
        for h in range(H):
            assert ucount[h] == len(ref["union"][h]), f"t={t} h={h} union size"
            assert uidx[h, :ucount[h]].tolist() == ref["union"][h].tolist(), f"t={t} h={h} union"
        what = f"step {t} H={H} P={P} B={B} d={d} bq={bq} bk={bk}"
        assert_o_lse(r.o, r.lse, ref["o"], ref["lse"], what)
        assert_o_lse(st.o_cache, st.lse_cache, ref_state["o_pre"], ref_state["lse_pre"], what + " cache")


def test_stable_tokens_keep_their_cache_bit_for_bit():
    wl, (k_pre, v_pre, qs, ks, vs) = _case(2, 1000, 48, 64, 64, 64, 3, seed=3)
    kp, vp, q0, k0, v0 = _cuda(k_pre, v_pre, qs[0], ks[0], vs[0])
    _, _, st = sp.losa_init(q0, k0, v0, kp, vp, n_sel=3)
    before_o, before_l = st.o_cache.clone(), st.lse_cache.clone()
    q, k, v, qp = _cuda(qs[1], ks[1], vs[1], qs[0])
    r = sp.losa_step(q, k, v, qp, kp, vp, st, wl.tau)
    sp.device_check()
    stable = r.active == 0
    assert stable.any() and (~stable).any()
    assert torch.equal(st.o_cache[:, stable], before_o[:, stable])
    assert torch.equal(st.lse_cache[:, stable], before_l[:, stable])
    assert not torch.equal(st.o_cache[:, ~stable], before_o[:, ~stable])


def test_no_active_token():
    wl, (k_pre, v_pre, qs, ks, vs) = _case(2, 1000, 48, 64, 64, 64, 3, seed=4)
    kp, vp, q0, k0, v0 = _cuda(k_pre, v_pre, qs[0], ks[0], vs[0])
    _, _, st = sp.losa_init(q0, k0, v0, kp, vp, n_sel=3)
    before = st.o_cache.clone()
    state = _state_from(st)
    q, k, v, qp = _cuda(qs[1], ks[1], vs[1], qs[0])
    r = sp.losa_step(q, k, v, qp, kp, vp, st, 1e30)
    sp.device_check()
    assert int(r.active.sum()) == 0 and int(r.union_count.sum()) == 0
    assert torch.equal(st.o_cache, before)
    ref = O.losa_step(f64(qs[1]), f64(ks[1]), f64(vs[1]), f64(qs[0]), f64(k_pre), f64(v_pre), wl.scale, wl.bk,
                      1e30, state)
    assert_o_lse(r.o, r.lse, ref["o"], ref["lse"], "no active token")


@pytest.mark.parametrize("P,bk", [(1, 64), (50, 64), (200, 128)])
def test_every_token_active_and_every_block_kept_is_dense(P, bk):
    H, B, d = 2, 40, 128
    wl, (k_pre, v_pre, qs, ks, vs) = _case(H, P, B, d, 64, bk, 64, seed=P)
    kp, vp, q0, k0, v0 = _cuda(k_pre, v_pre, qs[0], ks[0], vs[0])
    _, _, st = sp.losa_init(q0, k0, v0, kp, vp, n_sel=64, bk=bk)
    q, k, v, qp = _cuda(qs[1], ks[1], vs[1], qs[0])
    r = sp.losa_step(q, k, v, qp, kp, vp, st, 0.0)
    sp.device_check()
    assert int(r.active.sum()) == B
    assert (r.union_count.cpu() == -(-P // bk)).all()
    o_ref = np.empty((H, B, d))
    l_ref = np.empty((H, B))
    for h in range(H):
        o_ref[h], l_ref[h] = O.softmax_attention(f64(qs[1][h]), np.vstack([f64(k_pre[h]), f64(ks[1][h])]),
                                                 np.vstack([f64(v_pre[h]), f64(vs[1][h])]), wl.scale)
    assert_o_lse(r.o, r.lse, o_ref, l_ref, f"all active P={P} bk={bk}")


def test_block_run_matches_stepwise_calls_and_oracle():
    wl, (k_pre, v_pre, qs, ks, vs) = _case(2, 1000, 48, 64, 64, 64, 3, T=4, seed=11)
    kp, vp, qg, kg, vg = _cuda(k_pre, v_pre, qs, ks, vs)
    res = sp.losa_block(qg, kg, vg, kp, vp, n_sel=3, tau=wl.tau)
    sp.device_check()
    # the same steps issued one by one give the same bits
    o0, l0, st = sp.losa_init(qg[0], kg[0], vg[0], kp, vp, n_sel=3, splits=res.state.splits)
    assert torch.equal(o0, res.o[0]) and torch.equal(l0, res.lse[0])
    for t in range(1, 4):
        r = sp.losa_step(qg[t], kg[t], vg[t], qg[t - 1], kp, vp, st, wl.tau)
        assert torch.equal(r.o, res.o[t]) and torch.equal(r.lse, res.lse[t]), f"step {t}"
        assert torch.equal(r.active, res.active[t]) and torch.equal(r.union_count, res.union_count[t])
    assert (res.active[0] == 1).all() and (res.union_count[0] == -(-1000 // 64)).all()
    ref = O.losa_block(f64(qs), f64(ks), f64(vs), f64(k_pre), f64(v_pre), wl.scale, wl.bk, wl.n_sel, wl.tau,
                       sel=res.state.sel.cpu().numpy())
    for t in range(4):
        assert_o_lse(res.o[t], res.lse[t], ref["o"][t], ref["lse"][t], f"block step {t}")
    assert (res.active.cpu().numpy().astype(bool) == ref["active"]).all()
    assert (res.union_count.cpu().numpy() == ref["union_count"]).all()


def test_split_count_changes_rounding_only():
    wl, (k_pre, v_pre, qs, ks, vs) = _case(2, 4096, 64, 128, 64, 64, 6, T=2, seed=21)
    kp, vp, qg, kg, vg = _cuda(k_pre, v_pre, qs, ks, vs)
    # the first step with one split and with eight
    results = {}
    for splits in (1, 8):
        o, lse, st = sp.losa_init(qg[0], kg[0], vg[0], kp, vp, n_sel=6, splits=splits)
        sp.device_check()
        results[splits] = st
        ref = _oracle_init(wl, k_pre, v_pre, qs, ks, vs)
        assert_o_lse(o, lse, ref["o"], ref["lse"], f"init splits={splits}")
    # the next step from one state, with one split and with eight
    base = results[1]
    ref_state = _oracle_init(wl, k_pre, v_pre, qs, ks, vs, sel=base.sel.cpu().numpy())["state"]
    outs = []
    for splits in (1, 8):
        need = sp.losa_workspace_bytes(2, 64, 4096, 128, 64, 64, splits)
        st = sp.BlockState(base.o_cache.clone(), base.lse_cache.clone(), base.sel.clone(), base.scale, 64, 64,
                           splits, torch.empty(need, dtype=torch.uint8, device="cuda"))
        outs.append(sp.losa_step(qg[1], kg[1], vg[1], qg[0], kp, vp, st, wl.tau, return_union=True))
        sp.device_check()
    a, b = outs
    assert torch.equal(a.active, b.active) and torch.equal(a.union_count, b.union_count)
    for h in range(2):
        n = int(a.union_count[h])
        assert torch.equal(a.union_idx[h, :n], b.union_idx[h, :n])
    ref = O.losa_step(f64(qs[1]), f64(ks[1]), f64(vs[1]), f64(qs[0]), f64(k_pre), f64(v_pre), wl.scale, wl.bk,
                      wl.tau, ref_state)
    for splits, r in zip((1, 8), outs):
        assert_o_lse(r.o, r.lse, ref["o"], ref["lse"], f"step splits={splits}")


def test_selection_entry_out_of_range_is_reported():
    wl, (k_pre, v_pre, qs, ks, vs) = _case(2, 1000, 48, 64, 64, 64, 3, seed=5)
    kp, vp, q0, k0, v0 = _cuda(k_pre, v_pre, qs[0], ks[0], vs[0])
    _, _, st = sp.losa_init(q0, k0, v0, kp, vp, n_sel=3)
    sp.device_check()
    st.sel[1, :, 0] = 10 ** 6
    q, k, v, qp = _cuda(qs[1], ks[1], vs[1], qs[0])
    sp.losa_step(q, k, v, qp, kp, vp, st, 0.0)
    with pytest.raises(sp.SparsedError) as e:
        sp.device_check()
    assert e.value.status == _lib.ERR_BAD_PATTERN


def test_argument_errors():
    wl, (k_pre, v_pre, qs, ks, vs) = _case(2, 1000, 48, 64, 64, 64, 3, seed=6)
    kp, vp, q0, k0, v0 = _cuda(k_pre, v_pre, qs[0], ks[0], vs[0])
    _, _, st = sp.losa_init(q0, k0, v0, kp, vp, n_sel=3)
    with pytest.raises(sp.SparsedError) as e:
        sp.losa_step(q0, k0, v0, q0, kp, vp, st, float("nan"))
    assert e.value.status == _lib.ERR_INVALID_ARG
    small = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(sp.SparsedError) as e:
        sp.losa_init(q0, k0, v0, kp, vp, n_sel=3, workspace=small)
    assert e.value.status == _lib.ERR_WORKSPACE
    big = torch.zeros((2, 1025, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sp.SparsedError) as e:
        sp.losa_init(big, big, big, kp, vp, n_sel=3)
    assert e.value.status == _lib.ERR_UNSUPPORTED
    sp.device_check()


def test_full_size_block_sampled():
    """losa_32k (H=32, P=32768, B=64, d=128, 2 blocks per token, T=16) as the
    benchmark runs it; the oracle checks sampled rows and exact invariants."""
    wl = BLOCK_WORKLOADS["losa_32k"]
    k_pre, v_pre, qs, ks, vs = make_block_inputs(wl)
    kp, vp, qg, kg, vg = _cuda(k_pre, v_pre, qs, ks, vs)
    res = sp.losa_block(qg, kg, vg, kp, vp, n_sel=wl.n_sel, tau=wl.tau, bq=wl.bq, bk=wl.bk)
    sp.device_check()
    T, H, B = wl.T, wl.H, wl.B
    nkb = wl.P // wl.bk
    sel = res.state.sel.cpu().numpy()
    active = res.active.cpu().numpy().astype(bool)
    ucount = res.union_count.cpu().numpy()
    n_act = int(round(wl.active_frac * B))
    for t in range(1, T):
        got = _assert_active(res.active[t], qs[t], qs[t - 1], wl.tau)
        assert got.sum() == n_act
        for h in range(H):
            assert ucount[t, h] == len(O.kv_union(sel[h], active[t])) <= n_act * wl.n_sel
    assert (ucount[0] == nkb).all()
    rng = np.random.default_rng(0)
    kh, vh = f64(k_pre), f64(v_pre)
    # step 0: dense over prefix and block, and the selection of sampled tokens
    o0, l0 = res.o[0].float().cpu().numpy(), res.lse[0].cpu().numpy()
    exact = 0
    for h in rng.choice(H, 4, replace=False):
        rows = rng.choice(B, 4, replace=False)
        q = f64(qs[0][h])[rows]
        o_p, l_p = O.softmax_attention(q, kh[h], vh[h], wl.scale)
        o_s, l_s = O.softmax_attention(q, f64(ks[0][h]), f64(vs[0][h]), wl.scale)
        o_r, l_r = O.merge_partials(o_p, l_p, o_s, l_s)
        assert_o_lse(o0[h, rows], l0[h, rows], o_r, l_r, f"full size step 0 h={h}")
        m = O.token_block_mass(q, kh[h], wl.scale, l_p, wl.bk)
        for i, b in enumerate(rows):
            exact += check_selection(sel[h, b], wl.n_sel, m[i], wl.n_sel, f"full size sel h={h} b={b}")
    assert exact >= 8
    # last step: its active tokens attend to the step's union
    t = T - 1
    ot, lt = res.o[t].float().cpu().numpy(), res.lse[t].cpu().numpy()
    act_rows = np.nonzero(active[t])[0]
    for h in rng.choice(H, 4, replace=False):
        u = O.kv_union(sel[h], active[t])
        rows = rng.choice(act_rows, 3, replace=False)
        q = f64(qs[t][h])[rows]
        o_p, l_p = O.prefix_attention(q, kh[h], vh[h], wl.scale, u, wl.bk)
        o_s, l_s = O.softmax_attention(q, f64(ks[t][h]), f64(vs[t][h]), wl.scale)
        o_r, l_r = O.merge_partials(o_p, l_p, o_s, l_s)
        assert_o_lse(ot[h, rows], lt[h, rows], o_r, l_r, f"full size step {t} h={h}")


def test_block_run_replayed_from_a_cuda_graph_gives_the_eager_bits():
    """The block run captured in a CUDA graph: the side stream joins the
    capture through its fork and join events, and the list, prefix and merge
    kernels enter it as programmatic dependents of the kernel before them.
    Every replay gives the bits of the eager run."""
    wl, (k_pre, v_pre, qs, ks, vs) = _case(2, 2048, 64, 128, 64, 64, 3, T=5, seed=23)
    kp, vp, qg, kg, vg = _cuda(k_pre, v_pre, qs, ks, vs)
    eager = sp.losa_block(qg, kg, vg, kp, vp, n_sel=3, tau=wl.tau)
    sp.device_check()
    out = torch.empty_like(qg)
    lse = torch.empty_like(eager.lse)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        cap = sp.losa_block(qg, kg, vg, kp, vp, n_sel=3, tau=wl.tau, splits=eager.state.splits, out=out, lse=lse)
    for _ in range(2):
        out.zero_()
        lse.zero_()
        graph.replay()
        torch.cuda.synchronize()
        sp.device_check()
        assert torch.equal(out.view(torch.int16), eager.o.view(torch.int16))
        assert torch.equal(lse, eager.lse)
        assert torch.equal(cap.active, eager.active) and torch.equal(cap.union_count, eager.union_count)
    assert (eager.active[1:].sum(dim=1) > 0).any()  # later steps with active tokens took the sparse path

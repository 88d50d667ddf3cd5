"""CUDA path against the fp64 oracle, element by element, at sizes the oracle
finishes in seconds (several tiles, ragged tails, every kernel variant), plus
bitwise properties of the kernels and device-side error reporting."""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle as O
import block_sparse_bidirectional_select_b200 as sp
from block_sparse_bidirectional_select_b200.inputs import WORKLOADS, make_inputs
from gpu_common import (assert_o_lse, check_selection, f64, oracle_dense_heads, pattern_lists,
                        MASS_RTOL)

pytestmark = pytest.mark.gpu

VARIANTS = [(d, bq, bk) for d in (64, 128) for bq in (64, 128) for bk in (64, 128)]


def _inputs(H, L, d, seed, structure="iid"):
    wl = WORKLOADS["tiny"].scaled(H=H, L=L, d=d, seed=seed, structure=structure)
    q, k, v = make_inputs(wl)
    return q, k, v, wl.scale


def _cuda(*ts):
    return [t.cuda() for t in ts]


def _random_pattern(H, nqb, nkb, stride, rng, allow_empty=True):
    idx = np.full((H, nqb, stride), -1, dtype=np.int32)
    cnt = np.zeros((H, nqb), dtype=np.int32)
    for h in range(H):
        for i in range(nqb):
            lo = 0 if allow_empty else 1
            c = int(rng.integers(lo, min(stride, nkb) + 1))
            sel = np.sort(rng.choice(nkb, c, replace=False)) if c else np.zeros(0, np.int32)
            idx[h, i, :c] = sel
            cnt[h, i] = c
    return torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()


@pytest.mark.parametrize("d,bq,bk", VARIANTS)
@pytest.mark.parametrize("L", [1024, 1000])
def test_dense_parity(d, bq, bk, L):
    q, k, v, scale = _inputs(2, L, d, seed=7 + d + L)
    qc, kc, vc = _cuda(q, k, v)
    o, lse = sp.dense_attn(qc, kc, vc, bq=bq, bk=bk)
    sp.device_check()
    o_ref, l_ref = oracle_dense_heads(q, k, v, scale)
    assert_o_lse(o, lse, o_ref, l_ref, f"dense d={d} bq={bq} bk={bk} L={L}")


@pytest.mark.parametrize("L", [1, 63, 64, 130, 257])
def test_dense_tiny_lengths(L):
    q, k, v, scale = _inputs(3, L, 128, seed=100 + L)
    o, lse = sp.dense_attn(*_cuda(q, k, v))
    sp.device_check()
    o_ref, l_ref = oracle_dense_heads(q, k, v, scale)
    assert_o_lse(o, lse, o_ref, l_ref, f"dense L={L}")


@pytest.mark.parametrize("d,bq,bk", VARIANTS)
def test_sparse_parity_given_pattern(d, bq, bk):
    H, L = 2, 1000
    q, k, v, scale = _inputs(H, L, d, seed=31 + d + bq + bk)
    nqb, nkb = -(-L // bq), -(-L // bk)
    rng = np.random.default_rng(d * 1000 + bq * 10 + bk)
    kv_idx, kv_count = _random_pattern(H, nqb, nkb, nkb, rng)
    o, lse = sp.block_sparse_attn(*_cuda(q, k, v), kv_idx, kv_count, bq=bq, bk=bk)
    sp.device_check()
    lists, cnt = pattern_lists(kv_idx, kv_count)
    qh, kh, vh = f64(q), f64(k), f64(v)
    o_ref = np.empty(qh.shape)
    l_ref = np.empty(qh.shape[:2])
    for h in range(H):
        o_ref[h], l_ref[h] = O.masked_attention(qh[h], kh[h], vh[h], scale, lists[h], cnt[h], bq, bk)
    assert_o_lse(o, lse, o_ref, l_ref, f"sparse d={d} bq={bq} bk={bk}")
    # empty lists: exactly zero output and -inf LSE
    empty = (kv_count.cpu().numpy() == 0)
    for h, i in zip(*np.nonzero(empty)):
        rows = slice(i * bq, min((i + 1) * bq, L))
        assert (o[h, rows] == 0).all()
        assert torch.isneginf(lse[h, rows]).all()


@pytest.mark.parametrize("d,bq,bk", [(64, 64, 64), (128, 128, 128)])
def test_many_items_per_persistent_cta(d, bq, bk):
    """More work items than SMs, so every CTA walks several (head, query
    block) items and its pipelines cross item boundaries: ragged L, random
    list lengths including empty lists between non-empty ones, then a dense
    pass over the same shape."""
    H, L = 8, 4000
    q, k, v, scale = _inputs(H, L, d, seed=77 + d)
    nqb, nkb = -(-L // bq), -(-L // bk)
    assert H * nqb > 148 * (2 if bq == 64 else 1)
    rng = np.random.default_rng(4242 + d)
    kv_idx, kv_count = _random_pattern(H, nqb, nkb, nkb, rng)
    qc, kc, vc = _cuda(q, k, v)
    o, lse = sp.block_sparse_attn(qc, kc, vc, kv_idx, kv_count, bq=bq, bk=bk)
    od, ld = sp.dense_attn(qc, kc, vc, bq=bq, bk=bk)
    sp.device_check()
    lists, cnt = pattern_lists(kv_idx, kv_count)
    qh, kh, vh = f64(q), f64(k), f64(v)
    o_ref = np.empty(qh.shape)
    l_ref = np.empty(qh.shape[:2])
    for h in range(H):
        o_ref[h], l_ref[h] = O.masked_attention(qh[h], kh[h], vh[h], scale, lists[h], cnt[h], bq, bk)
    assert_o_lse(o, lse, o_ref, l_ref, f"sparse, many items, d={d} bq={bq}")
    od_ref, ld_ref = oracle_dense_heads(q, k, v, scale)
    assert_o_lse(od, ld, od_ref, ld_ref, f"dense, many items, d={d} bq={bq}")


@pytest.mark.parametrize("d,bk", [(64, 64), (128, 128), (128, 64)])
def test_keep_all_equals_dense(d, bk):
    """A list that keeps every block in ascending order is dense attention:
    the block-sparse kernel and the dense kernel (two different kernels, the
    same sums in a different grouping) agree to fp32 rounding of the row sums
    and one bf16 rounding of O, and both match the oracle."""
    H, L, bq = 2, 1024 + 64, 128
    q, k, v, scale = _inputs(H, L, d, seed=5)
    qc, kc, vc = _cuda(q, k, v)
    nqb, nkb = -(-L // bq), -(-L // bk)
    kv_idx = torch.arange(nkb, dtype=torch.int32, device="cuda").repeat(H, nqb, 1).contiguous()
    kv_count = torch.full((H, nqb), nkb, dtype=torch.int32, device="cuda")
    o1, l1 = sp.dense_attn(qc, kc, vc, bq=bq, bk=bk)
    o2, l2 = sp.block_sparse_attn(qc, kc, vc, kv_idx, kv_count, bq=bq, bk=bk)
    sp.device_check()
    assert (o1.float() - o2.float()).abs().max().item() <= 2 ** -7
    assert (l1 - l2).abs().max().item() <= 1e-5
    o_ref, l_ref = oracle_dense_heads(q, k, v, scale)
    assert_o_lse(o2, l2, o_ref, l_ref, f"keep-all sparse d={d} bk={bk}")


def test_determinism():
    q, k, v, _ = _inputs(2, 2048, 128, seed=9, structure="band")
    qc, kc, vc = _cuda(q, k, v)
    p1 = sp.select_pattern(qc, kc, vc, keep=0.2, return_mass=True)
    p2 = sp.select_pattern(qc, kc, vc, keep=0.2, return_mass=True)
    s1 = sp.block_sparse_attn(qc, kc, vc, p1.kv_idx, p1.kv_count)
    s2 = sp.block_sparse_attn(qc, kc, vc, p1.kv_idx, p1.kv_count)
    sp.device_check()
    assert torch.equal(p1.o.view(torch.int16), p2.o.view(torch.int16))
    assert torch.equal(p1.lse, p2.lse)
    assert torch.equal(p1.block_mass, p2.block_mass)
    assert torch.equal(p1.kv_idx, p2.kv_idx)
    assert torch.equal(s1[0].view(torch.int16), s2[0].view(torch.int16))
    assert torch.equal(s1[1], s2[1])


@pytest.mark.parametrize("d,b", [(64, 64), (128, 128)])
def test_zero_query_closed_forms(d, b):
    H, L, keep = 2, 1024, 0.25
    _, k, v, _ = _inputs(H, L, d, seed=11)
    q = torch.zeros_like(k)
    qc, kc, vc = _cuda(q, k, v)
    p = sp.select_pattern(qc, kc, vc, keep=keep, bq=b, bk=b, return_mass=True)
    sp.device_check()
    nkb = L // b
    kk = O.uniform_keep(nkb, keep)
    vh = f64(v)
    # dense: P = 1/L everywhere, O = mean(V), LSE = ln L
    assert_o_lse(p.o, p.lse, np.broadcast_to(vh.mean(axis=1, keepdims=True), vh.shape),
                 np.full((H, L), math.log(L)), "Q=0 dense")
    # every block ties exactly: the tie-break keeps blocks 0..k-1
    m = p.block_mass.cpu()
    assert torch.equal(m, m[0, 0, 0].expand_as(m))
    assert (p.kv_idx[:, :, :kk].cpu() == torch.arange(kk, dtype=torch.int32)).all()
    o, lse = sp.block_sparse_attn(qc, kc, vc, p.kv_idx, p.kv_count, bq=b, bk=b)
    sp.device_check()
    ref = vh[:, : kk * b].mean(axis=1, keepdims=True)
    assert_o_lse(o, lse, np.broadcast_to(ref, vh.shape), np.full((H, L), math.log(kk * b)), "Q=0 sparse")


def test_constant_v():
    H, L, d = 2, 777, 128
    q, k, _, _ = _inputs(H, L, d, seed=12)
    v = torch.full_like(q, 1.5)
    o, _ = sp.dense_attn(*_cuda(q, k, v))
    sp.device_check()
    assert (o.float() - 1.5).abs().max().item() <= 1e-2


@pytest.mark.parametrize("d,bq,bk", [(64, 64, 64), (128, 128, 128), (128, 64, 128), (64, 128, 64)])
def test_select_pattern_parity(d, bq, bk):
    H, L, keep = 3, 1000, 0.25
    q, k, v, scale = _inputs(H, L, d, seed=21 + d, structure="band")
    qc, kc, vc = _cuda(q, k, v)
    p = sp.select_pattern(qc, kc, vc, keep=keep, bq=bq, bk=bk, return_mass=True)
    sp.device_check()
    ref = O.select_pattern(f64(q), f64(k), f64(v), scale, bq, bk, keep, "uniform")
    assert_o_lse(p.o, p.lse, ref["o"], ref["lse"], "select dense pass")
    mass = p.block_mass.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(mass, ref["mass"], rtol=MASS_RTOL, atol=1e-6)
    nkb = -(-L // bk)
    kk = O.uniform_keep(nkb, keep)
    assert (p.head_k.cpu().numpy() == kk).all()
    idx = p.kv_idx.cpu().numpy()
    cnt = p.kv_count.cpu().numpy()
    exact = 0
    for h in range(H):
        for i in range(mass.shape[1]):
            exact += check_selection(idx[h, i], cnt[h, i], ref["mass"][h, i], kk, f"h{h} i{i}")
            # the same decision taken in the kernel's precision is bit-exact
            assert list(idx[h, i, :kk]) == list(O.topk_blocks(mass[h, i], kk))
    assert exact > 0


def test_select_entropy_budget_parity():
    H, L, d, b, keep = 4, 2048, 128, 128, 0.2
    q, k, v, scale = _inputs(H, L, d, seed=41, structure="band")
    qc, kc, vc = _cuda(q, k, v)
    p = sp.select_pattern(qc, kc, vc, keep=keep, budget="entropy", return_mass=True)
    sp.device_check()
    nkb = L // b
    mass_gpu = p.block_mass.cpu().numpy().astype(np.float64)
    head_k = p.head_k.cpu().numpy()
    # decision in the kernel's precision (entropies from the GPU mass grid): exact
    ent_gpu = [O.head_entropy(mass_gpu[h]) for h in range(H)]
    k_ref, B = O.entropy_budget(ent_gpu, nkb, keep)
    assert list(head_k) == k_ref and head_k.sum() == B
    # against the fp64 oracle end to end (unless a quota sits on a rounding edge)
    ref = O.select_pattern(f64(q), f64(k), f64(v), scale, b, b, keep, "entropy")
    if list(ref["head_k"]) != list(head_k):
        X = B - H
        ent = ref["entropies"]
        quotas = [X * e / sum(ent) for e in ent]
        assert min(abs(x - round(x)) for x in quotas) < 1e-4
    assert len(set(head_k.tolist())) > 1  # band heads are concentrated: budgets differ
    idx = p.kv_idx.cpu().numpy()
    cnt = p.kv_count.cpu().numpy()
    for h in range(H):
        for i in range(mass_gpu.shape[1]):
            check_selection(idx[h, i], cnt[h, i], ref["mass"][h, i], int(head_k[h]), f"h{h} i{i}")


def test_run_steps_matches_calls_and_oracle():
    H, L, d, b = 2, 512, 128, 128
    q, k, v, scale = _inputs(H, L, d, seed=51, structure="band")
    qc, kc, vc = _cuda(q, k, v)
    r = sp.run_steps(qc, kc, vc, T=6, warmup_frac=0.34, keep=0.5, refresh_every=2, time_steps=True)
    sp.device_check()
    assert r.kinds == O.schedule(6, 0.34, 2)
    assert all(ms > 0 for ms in r.step_ms)
    o_ref, l_ref, kinds, pat = O.run_steps(f64(q), f64(k), f64(v), scale, b, b, 0.5, "uniform", 6, 0.34, 2)
    assert kinds == r.kinds
    assert_o_lse(r.o, r.lse, o_ref, l_ref, "run_steps")
    idx, cnt = r.kv_idx.cpu().numpy(), r.kv_count.cpu().numpy()
    for h in range(H):
        for i in range(idx.shape[1]):
            check_selection(idx[h, i], cnt[h, i], pat["mass"][h, i], int(pat["head_k"][h]), f"h{h} i{i}")
    # the last (sparse) step runs on the cached pattern, bit for bit
    if r.kinds[-1] == O.SPARSE:
        o2, _ = sp.block_sparse_attn(qc, kc, vc, r.kv_idx, r.kv_count)
        assert torch.equal(r.o.view(torch.int16), o2.view(torch.int16))


@pytest.mark.parametrize("budget,d,L,bq,bk", [("uniform", 128, 1536, 128, 128), ("entropy", 128, 1536, 128, 128),
                                               ("uniform", 64, 1000, 64, 64), ("entropy", 128, 1000, 128, 64)])
def test_run_steps_fused_selection_matches_separate_pass(budget, d, L, bq, bk):
    """With the larger workspace, SELECT steps after a full pass take the block
    mass from their own pass; with the selection workspace alone they run the
    separate block-mass pass. Both must pick the oracle's pattern (margin
    rule) and agree with each other wherever the oracle's margin is clear."""
    H = 4
    q, k, v, scale = _inputs(H, L, d, seed=88 + d + bk, structure="band")
    qc, kc, vc = _cuda(q, k, v)
    small = torch.empty(sp.workspace_bytes(H, L, bq, bk), dtype=torch.uint8, device="cuda")
    assert sp.run_steps_workspace_bytes(H, L, bq, bk) > small.numel()
    kw = dict(T=8, warmup_frac=0.3, keep=0.25, budget=budget, refresh_every=3, bq=bq, bk=bk)
    r_fused = sp.run_steps(qc, kc, vc, **kw)
    r_sep = sp.run_steps(qc, kc, vc, workspace=small, **kw)
    sp.device_check()
    o_ref, l_ref, kinds, pat = O.run_steps(f64(q), f64(k), f64(v), scale, bq, bk, 0.25, budget, 8, 0.3, 3)
    assert kinds == r_fused.kinds and kinds.count(O.SELECT) >= 2
    assert_o_lse(r_fused.o, r_fused.lse, o_ref, l_ref, f"fused run_steps {budget}")
    for r in (r_fused, r_sep):
        idx, cnt = r.kv_idx.cpu().numpy(), r.kv_count.cpu().numpy()
        for h in range(H):
            for i in range(idx.shape[1]):
                check_selection(idx[h, i], cnt[h, i], pat["mass"][h, i], int(pat["head_k"][h]), f"h{h} i{i}")
    assert torch.equal(r_fused.kv_count, r_sep.kv_count)
    same = (r_fused.kv_idx == r_sep.kv_idx).all(dim=-1).float().mean().item()
    assert same > 0.95


def test_run_steps_resume_with_pattern():
    H, L, d = 2, 512, 64
    q, k, v, _ = _inputs(H, L, d, seed=52)
    qc, kc, vc = _cuda(q, k, v)
    p = sp.select_pattern(qc, kc, vc, keep=0.5)
    r = sp.run_steps(qc, kc, vc, T=10, warmup_frac=0.2, keep=0.5, start_step=5,
                     pattern=(p.kv_idx.clone(), p.kv_count.clone()))
    o2, l2 = sp.block_sparse_attn(qc, kc, vc, p.kv_idx, p.kv_count)
    sp.device_check()
    assert torch.equal(r.o.view(torch.int16), o2.view(torch.int16))
    with pytest.raises(sp.SparsedError):
        sp.run_steps(qc, kc, vc, T=10, warmup_frac=0.2, keep=0.5, start_step=5)  # no pattern yet


def test_bad_pattern_is_reported_not_faulted():
    H, L, d = 1, 512, 128
    q, k, v, _ = _inputs(H, L, d, seed=61)
    qc, kc, vc = _cuda(q, k, v)
    nqb = nkb = 4
    idx = torch.tensor([[[0, 1], [2, 9], [1, 0], [3, 3]]], dtype=torch.int32, device="cuda")
    cnt = torch.tensor([[2, 2, 2, 2]], dtype=torch.int32, device="cuda")
    sp.block_sparse_attn(qc, kc, vc, idx, cnt)
    with pytest.raises(sp.SparsedError) as e:
        sp.device_check()
    assert e.value.status == sp._lib.ERR_BAD_PATTERN
    sp.device_check()  # the error word was cleared
    cnt = torch.tensor([[2, 5, 0, 1]], dtype=torch.int32, device="cuda")  # count > stride
    idx = torch.tensor([[[0, 1], [2, 3], [0, 0], [3, 0]]], dtype=torch.int32, device="cuda")
    sp.block_sparse_attn(qc, kc, vc, idx, cnt)
    with pytest.raises(sp.SparsedError):
        sp.device_check()
    # a good pattern afterwards runs clean
    cnt = torch.tensor([[2, 2, 0, 1]], dtype=torch.int32, device="cuda")
    sp.block_sparse_attn(qc, kc, vc, idx, cnt)
    sp.device_check()


def test_expired_device_wait_is_reported_and_the_context_stays_usable():
    """A bounded device wait that runs out (an mbarrier nothing arrives on)
    records SPARSED_ERR_DEVICE_TIMEOUT; the next check reports and clears it,
    and the library keeps working."""
    lib = sp._lib.load()
    stream = torch.cuda.current_stream()
    assert lib.sparsed_selftest_wait_timeout(2_000_000, ctypes.c_void_p(stream.cuda_stream)) == 0
    with pytest.raises(sp.SparsedError) as e:
        sp.device_check()
    assert e.value.status == sp._lib.ERR_DEVICE_TIMEOUT
    sp.device_check()
    q, k, v, scale = _inputs(1, 256, 64, seed=9)
    o, lse = sp.dense_attn(*_cuda(q, k, v), bq=64, bk=64)
    sp.device_check()
    o_ref, l_ref = oracle_dense_heads(q, k, v, scale)
    assert_o_lse(o, lse, o_ref, l_ref, "after an expired wait")


def test_empty_problem_is_noop():
    q = torch.zeros((0, 128, 64), dtype=torch.bfloat16, device="cuda")
    o, lse = sp.dense_attn(q, q, q)
    assert o.numel() == 0 and lse.numel() == 0
    q = torch.zeros((2, 0, 64), dtype=torch.bfloat16, device="cuda")
    o, lse = sp.dense_attn(q, q, q)
    sp.device_check()


@pytest.mark.parametrize("d,L", [(64, 1000), (128, 2048)])
def test_dense_attn_agrees_with_torch_sdpa(d, L):
    """A library cross-check beside the oracle: torch's scaled_dot_product_attention
    (flash / cuDNN kernels) on the same bf16 inputs, and the LSE of fp32 scores."""
    import torch.nn.functional as F
    q, k, v, scale = _inputs(2, L, d, seed=500 + d)
    qc, kc, vc = _cuda(q, k, v)
    o, lse = sp.dense_attn(qc, kc, vc)
    sp.device_check()
    ref = F.scaled_dot_product_attention(qc.unsqueeze(0), kc.unsqueeze(0), vc.unsqueeze(0), scale=scale)[0]
    err = (o.float() - ref.float()).abs()
    assert err.max().item() <= 2e-2 and err.mean().item() <= 2e-3
    s = torch.matmul(qc.float(), kc.float().transpose(1, 2)) * scale
    assert (lse - torch.logsumexp(s, dim=-1)).abs().max().item() <= 1e-3


@pytest.mark.parametrize("H,L,d,bq,bk", [(8, 4000, 128, 128, 128), (4, 8200, 64, 64, 64),
                                         (16, 16384 + 100, 128, 128, 128), (3, 640, 128, 128, 64)])
def test_counter_scheduled_passes_equal_static(H, L, d, bq, bk):
    """The step loop's full passes take their pairs of query blocks from a
    counter in the workspace; a standalone dense_attn takes them by a static
    stride. A pair's arithmetic does not depend on which CTA runs it, so every
    pass of a loop of dense steps (the counter slots alternating from launch to
    launch, and starting over in a second call on the same workspace) gives
    the bits of the static pass. The cases cover fewer pairs than SMs, an odd
    number of query blocks (a pair without a second block) and several waves."""
    q, k, v, scale = _inputs(H, L, d, seed=31 + d + H, structure="band")
    qc, kc, vc = _cuda(q, k, v)
    od, ld = sp.dense_attn(qc, kc, vc, bq=bq, bk=bk)
    ws = torch.empty(sp.run_steps_workspace_bytes(H, L, bq, bk), dtype=torch.uint8, device="cuda")
    for _ in range(2):
        r = sp.run_steps(qc, kc, vc, T=5, warmup_frac=1.0, bq=bq, bk=bk, workspace=ws)
        sp.device_check()
        assert set(r.kinds) == {sp.STEP_DENSE}
        assert torch.equal(r.o.view(torch.int16), od.view(torch.int16))
        assert torch.equal(r.lse, ld)
    if L <= 4000:
        o_ref, l_ref = oracle_dense_heads(q, k, v, scale)
        assert_o_lse(r.o, r.lse, o_ref, l_ref, f"counter-scheduled dense d={d} bq={bq} bk={bk}")

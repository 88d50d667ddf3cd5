"""The seeded input generators: shapes, determinism, and the structure each
workload recipe describes (CPU only, scaled-down sizes)."""
import torch

from block_sparse_bidirectional_select_b200.inputs import WORKLOADS, make_inputs, zero_q


def test_shapes_dtype_and_determinism():
    wl = WORKLOADS["tiny"].scaled(H=2, L=256)
    a = make_inputs(wl)
    b = make_inputs(wl)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and x.shape == (2, 256, 64)
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))
    c = make_inputs(wl.scaled(seed=wl.seed + 1))
    assert not torch.equal(a[0], c[0])


def test_key_bias_hot_columns_per_head():
    wl = WORKLOADS["c2_8k"].scaled(H=3, L=1000)
    q, k, v = make_inputs(wl)
    qn, kn, vn = make_inputs(wl.scaled(structure="iid"))
    assert torch.equal(q, qn) and torch.equal(v, vn)
    for h in range(3):
        shifted = ((k[h].float() - kn[h].float()).abs().mean(dim=1) > 1.0).sum().item()
        assert shifted == 100  # round(0.1 * L) positions, all d components
    hot = [set(torch.nonzero((k[h].float() - kn[h].float()).abs().mean(dim=1) > 1.0).flatten().tolist())
           for h in range(3)]
    assert hot[0] != hot[1]


def test_band_structure_on_half_the_heads():
    wl = WORKLOADS["c4_64k"].scaled(H=4, L=2048)
    q, k, _ = make_inputs(wl)
    qn, kn, _ = make_inputs(wl.scaled(structure="iid"))
    changed = [not torch.equal(q[h], qn[h]) for h in range(4)]
    assert sum(changed) == 2
    for h in range(4):
        assert changed[h] == (not torch.equal(k[h], kn[h]))
        if changed[h]:  # the local term raises near-diagonal scores
            s = q[h].float() @ k[h].float().T
            near = torch.diagonal(s).mean() - s.mean()
            assert near.item() > 30.0


def test_low_rank_scores_concentrated():
    wl = WORKLOADS["c3_16k"].scaled(H=2, L=512, d=128)
    q, k, _ = make_inputs(wl)
    s = (q[0].float() @ k[0].float().T) * wl.scale
    p = torch.softmax(s, dim=-1)
    # attention is concentrated: the top 10% of keys hold most of each row's mass
    top = p.topk(51, dim=-1).values.sum(dim=-1)
    assert top.mean().item() > 0.5


def test_zero_q():
    q, k, v = zero_q(WORKLOADS["tiny"].scaled(H=1, L=64))
    assert (q == 0).all() and k.abs().sum() > 0


def test_block_workload_recipe():
    """The block-wise inputs: deterministic per seed, bf16, and at every step
    after the first exactly round(0.25*B) tokens change by far more than tau
    while every other token's query MSE stays far below it."""
    import numpy as np

    import oracle as O
    from block_sparse_bidirectional_select_b200.inputs import BLOCK_WORKLOADS, make_block_inputs, to_f64
    wl = BLOCK_WORKLOADS["losa_tiny"]
    a = make_block_inputs(wl)
    b = make_block_inputs(wl)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and torch.equal(x.view(torch.int16), y.view(torch.int16))
    k_pre, v_pre, qs, ks, vs = a
    assert k_pre.shape == (wl.H, wl.P, wl.d) and qs.shape == (wl.T, wl.H, wl.B, wl.d)
    n_act = round(wl.active_frac * wl.B)
    for t in range(1, wl.T):
        mse = O.query_mse(to_f64(qs[t]), to_f64(qs[t - 1]))
        act = mse > wl.tau
        assert act.sum() == n_act
        assert mse[act].min() > 10 * wl.tau and mse[~act].max() < wl.tau / 10

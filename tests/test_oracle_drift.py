"""Pins of the oracle's per-step query drift (queries that change across the
denoising steps), on the CPU.

- fmix32 against the published MurmurHash3 x86_32 test vectors of the empty
  input (the hash of an empty input is the finalizer of the seed), and as a
  bijection.
- The uniforms: on their 2^-23 grid in [-1, 1), mean and variance of a uniform
  law, decorrelated across steps.
- The bf16 rounding against torch's float32 -> bfloat16 conversion.
- drift_queries against torch's fp32 addition plus that conversion.
- The denoising loop with drift: amplitude 0 is the loop without drift, and the
  last step is masked attention over that step's queries with the last
  selection's pattern.
"""
import math

import numpy as np
import torch

import oracle as O


def test_fmix32_published_vectors():
    # MurmurHash3_x86_32(key="", len=0, seed) = fmix32(seed ^ 0)
    assert int(O.fmix32(0)) == 0
    assert int(O.fmix32(1)) == 0x514E28B7
    assert int(O.fmix32(0xFFFFFFFF)) == 0x81F16F39


def test_fmix32_is_a_bijection_on_a_sample():
    rng = np.random.default_rng(0)
    x = np.unique(rng.integers(0, 2 ** 32, 1 << 20, dtype=np.uint64))
    h = O.fmix32(x)
    assert len(np.unique(h)) == len(x)
    assert h.max() < 2 ** 32


def test_drift_uniform_grid_and_moments():
    n = 1 << 18
    u = O.drift_uniform(1234, 7, n)
    k = (u + 1.0) * 2.0 ** 23
    assert np.all(k == np.floor(k)) and k.min() >= 0 and k.max() < 2 ** 24
    assert u.min() >= -1.0 and u.max() < 1.0
    assert abs(u.mean()) < 5 * math.sqrt(1 / 3 / n)
    assert abs(u.var() - 1 / 3) < 0.01
    v = O.drift_uniform(1234, 8, n)
    assert abs(np.corrcoef(u, v)[0, 1]) < 0.02
    assert np.array_equal(u, O.drift_uniform(1234, 7, n))
    assert not np.array_equal(u, O.drift_uniform(1235, 7, n))


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(1 << 16) * rng.choice([1e-3, 1.0, 1e3], 1 << 16)).astype(np.float32)
    # exact ties: the discarded half is 0x8000, with both parities of the kept part
    mant = rng.integers(0, 1 << 7, 4096, dtype=np.uint32)
    tb = ((np.uint32(0x3F80) | mant) << np.uint32(16)) | np.uint32(0x8000)  # values in [1, 2)
    x = np.concatenate([x, tb.view(np.float32), -tb.view(np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.bf16_round(x), ref)


def test_drift_queries_against_torch_arithmetic():
    q = torch.randn(3, 40, 16, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16)
    q64 = q.to(torch.float64).numpy()
    for seed, t in [(0, 0), (17, 5), (2 ** 31 + 3, 1000)]:
        got = O.drift_queries(q64, seed, t)
        u = O.drift_uniform(seed, t, q64.size).reshape(q64.shape)
        d = torch.from_numpy(u * O.DRIFT_AMPLITUDE).to(torch.float32)
        ref = (q.to(torch.float32) + d).to(torch.bfloat16).to(torch.float64).numpy()
        assert np.array_equal(got, ref)
        # a perturbation of at most the amplitude plus half a bf16 step of the
        # sum: half an ulp of x is at most |x| * 2^-8, and |q + u*amp| <= |q| + amp
        bound = O.DRIFT_AMPLITUDE + (np.abs(q64) + O.DRIFT_AMPLITUDE) * 2.0 ** -8
        assert np.all(np.abs(got - q64) <= bound)
    assert np.array_equal(O.drift_queries(q64, 9, 3, amplitude=0.0), q64)
    assert not np.array_equal(O.drift_queries(q64, 9, 3), O.drift_queries(q64, 9, 4))


def _bf16(x):
    return torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()


def test_loop_with_drift():
    rng = np.random.default_rng(3)
    H, L, d, b = 2, 96, 8, 16
    q, k, v = (_bf16(rng.standard_normal((H, L, d))) for _ in range(3))
    T, w, R = 8, 0.3, 2   # D D S P S P S P
    o0, l0, kinds0, _ = O.run_steps(q, k, v, 0.35, b, b, 0.3, "uniform", T, w, R)
    o1, l1, kinds1, _ = O.run_steps(q, k, v, 0.35, b, b, 0.3, "uniform", T, w, R, drift_seed=5,
                                    drift_amplitude=0.0)
    assert kinds0 == kinds1 and np.array_equal(o0, o1) and np.array_equal(l0, l1)
    sels = []
    o2, l2, kinds2, pat = O.run_steps(q, k, v, 0.35, b, b, 0.3, "uniform", T, w, R, drift_seed=5,
                                      patterns=sels)
    assert [t for t, _ in sels] == [t for t, kd in enumerate(kinds2) if kd == O.SELECT]
    assert kinds2[-1] == O.SPARSE and pat is sels[-1][1]
    # the last step: masked attention over step T-1's queries with the last pattern
    qT = O.drift_queries(q, 5, T - 1)
    for h in range(H):
        om, lm = O.masked_attention(qT[h], k[h], v[h], 0.35, pat["kv_idx"][h], pat["kv_count"][h], b, b)
        assert np.array_equal(om, o2[h]) and np.array_equal(lm, l2[h])
    # each selection was taken on its own step's queries
    t_sel, p_sel = sels[-1]
    ref = O.select_pattern(O.drift_queries(q, 5, t_sel), k, v, 0.35, b, b, 0.3)
    assert all(np.array_equal(a, b_) for a, b_ in zip(ref["kv_count"], p_sel["kv_count"]))
    assert not np.array_equal(o2, o0)

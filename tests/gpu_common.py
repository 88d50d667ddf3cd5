"""Shared helpers of the GPU parity tests: tolerances, comparisons against the
fp64 oracle, and the selection-margin rule."""
import math

import numpy as np
import torch

import oracle as O
from block_sparse_bidirectional_select_b200.inputs import to_f64

# Tolerances fixed for this path: bf16 inputs and bf16 P/O with fp32
# accumulation against an fp64 reference.
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-3
SELECT_MARGIN = 1e-4      # relative gap between the k-th and (k+1)-th mass
MASS_RTOL = 1e-4          # fp32 scores and exp against fp64


def assert_o_lse(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    o = o_gpu.float().cpu().numpy().astype(np.float64) if isinstance(o_gpu, torch.Tensor) else o_gpu
    lse = lse_gpu.cpu().numpy().astype(np.float64) if isinstance(lse_gpu, torch.Tensor) else lse_gpu
    finite = np.isfinite(lse_ref)
    assert (np.isneginf(lse) == np.isneginf(lse_ref)).all(), f"{what}: -inf rows differ"
    err = np.abs(o - o_ref)
    assert err.max() <= O_MAX_ABS, f"{what}: O max-abs {err.max():.3e}"
    assert err.mean() <= O_MEAN_ABS, f"{what}: O mean-abs {err.mean():.3e}"
    if finite.any():
        lerr = np.abs(lse[finite] - lse_ref[finite]).max()
        assert lerr <= LSE_MAX_ABS, f"{what}: LSE max-abs {lerr:.3e}"


def check_selection(gpu_row, gpu_count, mass_ref_row, k, what=""):
    """kv_idx must be bit-exact where the oracle's selection margin exceeds
    SELECT_MARGIN; otherwise every chosen block must be within the margin of
    the k-th largest oracle mass. Always: k entries, strictly ascending, in range."""
    n = len(mass_ref_row)
    assert int(gpu_count) == k, f"{what}: count {gpu_count} != {k}"
    sel = [int(x) for x in gpu_row[:k]]
    assert all(0 <= j < n for j in sel), f"{what}: index out of range {sel}"
    assert all(a < b for a, b in zip(sel, sel[1:])), f"{what}: not ascending {sel}"
    srt = np.sort(mass_ref_row)[::-1]
    mk = srt[k - 1]
    mk1 = srt[k] if k < n else -math.inf
    margin = (mk - mk1) / mk if mk > 0 else 0.0
    if margin > SELECT_MARGIN:
        ref = [int(x) for x in O.topk_blocks(mass_ref_row, k)]
        assert sel == ref, f"{what}: selection {sel} != oracle {ref} (margin {margin:.2e})"
        return True
    assert all(mass_ref_row[j] >= mk * (1 - SELECT_MARGIN) for j in sel), f"{what}: low-mass pick"
    return False


def f64(t):
    return to_f64(t)


def oracle_dense_heads(q, k, v, scale, heads=None):
    qh, kh, vh = f64(q), f64(k), f64(v)
    heads = range(qh.shape[0]) if heads is None else heads
    os_, ls_ = [], []
    for h in heads:
        o, l = O.dense_attention(qh[h], kh[h], vh[h], scale)
        os_.append(o)
        ls_.append(l)
    return np.stack(os_), np.stack(ls_)


def pattern_lists(kv_idx, kv_count):
    """[H,nqb,stride] / [H,nqb] tensors -> per-head python lists for the oracle."""
    idx = kv_idx.cpu().numpy()
    cnt = kv_count.cpu().numpy()
    return [[idx[h, i, :cnt[h, i]] for i in range(idx.shape[1])] for h in range(idx.shape[0])], cnt

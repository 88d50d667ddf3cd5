"""fp64 CPU oracle for block-sparse bidirectional attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, calls or links
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it. It shares no code, constant or helper with the CUDA
library; both sides only consume the same seeded bf16 inputs.

It is a plain, slow, obviously correct restatement, in float64 numpy, of what
the pages define (citations name the page title and the part of the page):

* SparseD: Sparse Attention for Diffusion Language Models, abstract -- DLM
  attention covers all query-key pairs (bidirectional); patterns differ per
  head, stay similar across denoising steps, and early steps are critical; so
  head-specific sparse patterns are computed once from full attention and
  reused, with full attention in the early steps.
* Step-dLLM: Adaptive Step-aware Sparse Attention for Efficient Diffusion LLM
  Inference, abstract -- bidirectional attention recomputes the full map every
  step; a block-sparse mask is refreshed at anchor steps and reused in between;
  a head-adaptive global budget compresses concentrated heads harder;
  "90% sparsity" means a keep ratio of 0.10.
* PulseCol: Periodically Refreshed Column-Sparse Attention for Accelerating
  Diffusion Language Models, abstract -- the same periodic-refresh schedule,
  and column-level (per key position) instead of block-level sparsity.

Where the pages leave a step open, the reading taken is stated in the function
docstring (rule for what is scored, rounding of k, tie-break, list order, the
budget formula, the schedule).

Every function here is pinned by ``tests/test_oracle_pins.py`` against closed
forms, brute force, library routines (torch float64 softmax/logsumexp) and
hand-computed fixtures in ``tests/golden/``.

Conventions: arrays are float64 numpy; one head is [L, d]; block j of a
length-L axis with block size b is the index range [j*b, min((j+1)*b, L)).
"""
from __future__ import annotations

import math

import numpy as np

DENSE, SELECT, SPARSE = 0, 1, 2
ROUND_EPS = 1e-6  # guards ceil() against products like 0.1*30 = 3.0000000000000004

# --------------------------------------------------------------------------
# O1  dense bidirectional attention
# --------------------------------------------------------------------------


def softmax_attention(q, k, v, scale):
    """Softmax attention of every row of ``q`` over every row of ``k``/``v``.

    Follows the SparseD abstract (attention over all query-key pairs, no causal
    mask) and the Step-dLLM abstract (bidirectional attention, full map every
    step). For row r:  s_c = scale * <q_r, k_c>,  m = max_c s_c,
    Z = sum_c exp(s_c - m),  o_r = sum_c exp(s_c - m)/Z * v_c,
    lse_r = m + ln Z  (natural log).

    An empty key set gives o_r = 0 and lse_r = -inf (reading: the pages never
    form an empty set; this is the limit of an empty sum).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    R = q.shape[0]
    if k.shape[0] == 0:
        return np.zeros((R, v.shape[1])), np.full(R, -np.inf)
    s = float(scale) * (q @ k.T)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(axis=1, keepdims=True)
    p = e / z
    o = p @ v
    lse = m[:, 0] + np.log(z[:, 0])
    return o, lse


def dense_attention(q, k, v, scale, rows=None, chunk=1024):
    """O1 for one head: full bidirectional attention, row by row.

    ``rows`` optionally restricts the query rows computed (rows are independent,
    so a sample of rows equals the same rows of the full result). Rows are
    processed in chunks only to bound memory; each row's arithmetic is the same.
    """
    q = np.asarray(q, dtype=np.float64)
    rows = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    o = np.empty((len(rows), v.shape[1]))
    lse = np.empty(len(rows))
    for s0 in range(0, len(rows), chunk):
        sel = rows[s0:s0 + chunk]
        o[s0:s0 + chunk], lse[s0:s0 + chunk] = softmax_attention(q[sel], k, v, scale)
    return o, lse


# --------------------------------------------------------------------------
# O2  block probability mass
# --------------------------------------------------------------------------


def n_blocks(L, b):
    return (L + b - 1) // b


def block_mass(q, k, scale, lse, bq, bk, qblocks=None):
    """Softmax probability mass of one head summed over each (query block,
    key block) tile.

    SparseD abstract: the head-specific sparse pattern is computed once from a
    full-attention pass. Reading taken for "what is scored": the post-softmax
    probability p_rc = exp(scale*<q_r,k_c> - lse_r) of the full (non-causal)
    row, summed over rows r of query block i and columns c of key block j:
        M[i, j] = sum_{r in qblk i} sum_{c in kblk j} p_rc.
    ``lse`` is the per-row log-sum-exp of that same head (from O1).
    Returns an array [len(qblocks), nkb].
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    L = q.shape[0]
    nqb, nkb = n_blocks(L, bq), n_blocks(k.shape[0], bk)
    qblocks = range(nqb) if qblocks is None else qblocks
    out = np.zeros((len(qblocks), nkb))
    for a, i in enumerate(qblocks):
        r0, r1 = i * bq, min((i + 1) * bq, L)
        s = float(scale) * (q[r0:r1] @ k.T)
        p = np.exp(s - np.asarray(lse)[r0:r1, None])
        for j in range(nkb):
            c0, c1 = j * bk, min((j + 1) * bk, k.shape[0])
            out[a, j] = p[:, c0:c1].sum()
    return out


# --------------------------------------------------------------------------
# O3  budgets
# --------------------------------------------------------------------------


def uniform_keep(nkb, keep_ratio):
    """Kept key blocks per query block when the budget is uniform over heads.

    Step-dLLM abstract: prior methods spread the sparsity budget uniformly
    across heads, and "90% sparsity" keeps 10%. Reading: k = ceil(rho * nkb)
    (with a 1e-6 guard against floating-point excess), at least 1 and at most
    nkb. ``keep_ratio`` is the fp32 value the C ABI receives, widened.
    """
    rho = float(np.float32(keep_ratio))
    k = math.ceil(rho * nkb - ROUND_EPS)
    return int(min(max(k, 1), nkb))


def head_entropy(M):
    """Mean over query blocks of the natural-log entropy of the row-normalised
    block mass, for one head. M is [nqb, nkb]; 0*ln 0 = 0.

    Step-dLLM abstract: heads concentrate their attention mass to very
    different extents. Reading: concentration is measured by this entropy
    (low entropy = concentrated).
    """
    total = 0.0
    for row in np.asarray(M, dtype=np.float64):
        z = row.sum()
        ent = 0.0
        for x in row:
            if x > 0.0:
                pj = x / z
                ent -= pj * math.log(pj)
        total += ent
    return total / M.shape[0]


def largest_remainder(total, weights):
    """Split integer ``total`` in proportion to ``weights``: floor of each quota,
    then one more unit to the largest fractional parts (ties: lower position).
    All-zero weights split evenly by the same rule."""
    w = [float(x) for x in weights]
    sw = sum(w)
    if sw <= 0.0:
        w = [1.0] * len(w)
        sw = float(len(w))
    quota = [total * x / sw for x in w]
    base = [math.floor(x) for x in quota]
    rem = total - sum(base)
    if rem >= 0:
        order = sorted(range(len(w)), key=lambda a: (-(quota[a] - base[a]), a))
        for a in order[:rem]:
            base[a] += 1
    else:
        # only reachable when fp64 rounding pushes a quota across an integer:
        # take units back from the smallest fractions (ties: higher position)
        order = sorted((a for a in range(len(w)) if base[a] > 0),
                       key=lambda a: (quota[a] - base[a], -a))
        for a in order[:-rem]:
            base[a] -= 1
    return base, quota


def entropy_budget(entropies, nkb, keep_ratio):
    """Head-adaptive global budget: per-head kept-block counts k_h.

    Step-dLLM abstract: a head-adaptive global budget compresses heads with
    concentrated attention more. Reading taken (the pages give only the
    direction):
      B = ceil(rho * H * nkb) blocks per query-block index, summed over heads
          (clamped to [H, H*nkb]);
      every head keeps at least one block; the extra budget X = B - H is split
      in proportion to E_h (evenly when the entropies of the heads being split
      sum to 0);
      a head whose extra share is above nkb - 1 is capped there and the rest
      of X is re-split over the uncapped heads, until no share is above the
      cap; the shares are then rounded by largest remainder (ties to the lower
      head index). k_h = 1 + extra_h, the same for every query block of head h.
    Returns (k [H], B).
    """
    H = len(entropies)
    rho = float(np.float32(keep_ratio))
    B = math.ceil(rho * H * nkb - ROUND_EPS)
    B = min(max(B, H), H * nkb)
    cap = nkb - 1
    extra = [None] * H
    while True:
        free = [h for h in range(H) if extra[h] is None]
        if not free:
            break
        Xf = (B - H) - sum(x for x in extra if x is not None)
        E = [float(entropies[h]) for h in free]
        sE = sum(E)
        weights = E if sE > 0.0 else [1.0] * len(free)
        sw = sum(weights)
        over = [h for h, w in zip(free, weights) if Xf * w / sw > cap]
        if over:
            for h in over:
                extra[h] = cap
            continue
        shares, _ = largest_remainder(Xf, weights)
        for h, x in zip(free, shares):
            extra[h] = x
        break
    return [1 + int(x) for x in extra], B


# --------------------------------------------------------------------------
# O4  top-k selection
# --------------------------------------------------------------------------


def topk_blocks(mass_row, k):
    """The k key blocks of largest mass for one (head, query block).

    Reading (pages do not state the rule): fixed-count top-k by mass, ties go
    to the lower block index, and the kept list is emitted in ascending index
    order.
    """
    m = np.asarray(mass_row, dtype=np.float64)
    order = np.lexsort((np.arange(len(m)), -m))
    return np.sort(order[:k]).astype(np.int32)


# --------------------------------------------------------------------------
# O5  block-sparse (masked) attention
# --------------------------------------------------------------------------


def kept_keys(blocks, bk, L):
    """Key positions covered by the listed key blocks, in ascending order."""
    idx = []
    for j in sorted(int(x) for x in blocks):
        idx.extend(range(j * bk, min((j + 1) * bk, L)))
    return np.asarray(idx, dtype=np.int64)


def masked_attention(q, k, v, scale, kv_idx, kv_count, bq, bk, qblocks=None):
    """O1 restricted, per query block i, to the keys of its kept blocks.

    Step-dLLM abstract (block-sparse mask reused between anchors) and SparseD
    abstract (the precomputed pattern reused at later steps). For query block
    i the key set is the union of blocks kv_idx[i, :kv_count[i]], visited in
    ascending key order, and the output is softmax attention over that set
    (LSE over the kept keys). With every block kept this performs exactly the
    operations of ``dense_attention`` on the same rows.
    Returns (o [rows, d], lse [rows]) for the rows of ``qblocks`` (all by
    default), in order.
    """
    q = np.asarray(q, dtype=np.float64)
    L = q.shape[0]
    nqb = n_blocks(L, bq)
    qblocks = range(nqb) if qblocks is None else qblocks
    os, ls = [], []
    for i in qblocks:
        r0, r1 = i * bq, min((i + 1) * bq, L)
        keys = kept_keys(kv_idx[i][: int(kv_count[i])], bk, k.shape[0])
        o, lse = softmax_attention(q[r0:r1], np.asarray(k)[keys], np.asarray(v)[keys], scale)
        os.append(o)
        ls.append(lse)
    return np.concatenate(os), np.concatenate(ls)


# --------------------------------------------------------------------------
# Pattern selection (O1 -> O2 -> O3 -> O4) for all heads
# --------------------------------------------------------------------------


def select_pattern(q, k, v, scale, bq, bk, keep_ratio, budget="uniform"):
    """One full-attention pass that also yields the block-sparse pattern.

    SparseD abstract: the pattern is computed from full attention (once); the
    full pass's own output is that step's output. q, k, v are [H, L, d].
    Returns dict with o [H,L,d], lse [H,L], mass [H,nqb,nkb], head_k [H],
    kv_idx (list over heads of lists over query blocks of int arrays),
    kv_count [H, nqb], entropies [H] (entropy budget only).
    """
    H, L, _ = q.shape
    nkb = n_blocks(L, bk)
    o = np.empty(q.shape)
    lse = np.empty((H, L))
    mass = []
    for h in range(H):
        o[h], lse[h] = dense_attention(q[h], k[h], v[h], scale)
        mass.append(block_mass(q[h], k[h], scale, lse[h], bq, bk))
    mass = np.stack(mass)
    ent = None
    if budget == "uniform":
        head_k = [uniform_keep(nkb, keep_ratio)] * H
    elif budget == "entropy":
        ent = [head_entropy(mass[h]) for h in range(H)]
        head_k, _ = entropy_budget(ent, nkb, keep_ratio)
    else:
        raise ValueError(budget)
    kv_idx = [[topk_blocks(mass[h, i], head_k[h]) for i in range(mass.shape[1])]
              for h in range(H)]
    kv_count = np.array([[head_k[h]] * mass.shape[1] for h in range(H)], dtype=np.int32)
    return dict(o=o, lse=lse, mass=mass, head_k=np.array(head_k, dtype=np.int32),
                kv_idx=kv_idx, kv_count=kv_count, entropies=ent)


# --------------------------------------------------------------------------
# O6  step schedule and the denoising loop
# --------------------------------------------------------------------------


def schedule(T, warmup_frac, refresh_every=0):
    """Kind of each denoising step t in [0, T).

    SparseD abstract: full attention in the early steps, then sparse attention
    with the pattern computed once. Step-dLLM / PulseCol abstracts: the pattern
    is refreshed at anchor steps and reused in between. Readings taken:
    n_dense = clamp(ceil(w*T), 1, T) (w is the fp32 ABI value widened); steps
    t < n_dense-1 are DENSE; the last warm-up step t = n_dense-1 is SELECT (its
    full pass is that step's output and yields the pattern); a later step t is
    SELECT when refresh_every R > 0 and (t - (n_dense-1)) is a multiple of R,
    else SPARSE. When n_dense = T no sparse step follows, so every step is
    DENSE and no pattern is selected.
    """
    w = float(np.float32(warmup_frac))
    n_dense = min(max(math.ceil(w * T - ROUND_EPS), 1), T)
    if n_dense == T:
        return [DENSE] * T
    kinds = []
    for t in range(T):
        if t < n_dense - 1:
            kinds.append(DENSE)
        elif t == n_dense - 1:
            kinds.append(SELECT)
        elif refresh_every > 0 and (t - (n_dense - 1)) % refresh_every == 0:
            kinds.append(SELECT)
        else:
            kinds.append(SPARSE)
    return kinds


def run_steps(q, k, v, scale, bq, bk, keep_ratio, budget, T, warmup_frac,
              refresh_every=0):
    """The denoising loop over one layer with fixed inputs: each step runs the
    kind ``schedule`` gives; SELECT refreshes the cached pattern; SPARSE uses
    the cached pattern. Returns (o, lse, kinds, pattern) of the last step."""
    kinds = schedule(T, warmup_frac, refresh_every)
    H, L, _ = q.shape
    pattern = None
    o = lse = None
    for t in range(T):
        if kinds[t] == DENSE:
            o = np.empty(q.shape)
            lse = np.empty((H, L))
            for h in range(H):
                o[h], lse[h] = dense_attention(q[h], k[h], v[h], scale)
        elif kinds[t] == SELECT:
            pattern = select_pattern(q, k, v, scale, bq, bk, keep_ratio, budget)
            o, lse = pattern["o"], pattern["lse"]
        else:
            o = np.empty(q.shape)
            lse = np.empty((H, L))
            for h in range(H):
                o[h], lse[h] = masked_attention(q[h], k[h], v[h], scale,
                                                pattern["kv_idx"][h],
                                                pattern["kv_count"][h], bq, bk)
    return o, lse, kinds, pattern


# --------------------------------------------------------------------------
# O7  column-sparse attention (PulseCol)
# --------------------------------------------------------------------------


def column_keep(L, keep_ratio):
    """Number of key columns kept per head: clamp(ceil(rho*L), 1, L).

    PulseCol abstract: column-level sparsity instead of block-level. Reading
    taken (the page gives no count rule): the keep ratio rho applies to the
    L key columns of a head, rounded up as for blocks (``uniform_keep``)."""
    rho = float(np.float32(keep_ratio))
    return min(max(math.ceil(rho * L - ROUND_EPS), 1), L)


def column_mass(q, k, scale, lse, chunk=1024):
    """Full-attention probability mass of every key column of one head:
        A[c] = sum over all rows r of p_rc,  p_rc = exp(scale*<q_r,k_c> - lse_r).

    PulseCol abstract: important attention interactions are kept at column
    granularity, identified from an early full pass. Reading taken for what is
    scored: the column analogue of the block mass, i.e. the post-softmax mass a
    key receives from all queries of the head. Rows are summed in ascending
    order, ``chunk`` rows at a time. Returns [Lk]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    out = np.zeros(k.shape[0])
    for r0 in range(0, q.shape[0], chunk):
        r1 = min(r0 + chunk, q.shape[0])
        s = float(scale) * (q[r0:r1] @ k.T)
        out += np.exp(s - lse[r0:r1, None]).sum(axis=0)
    return out


def topk_columns(col_mass, k):
    """The k key columns of largest mass of one head, ties to the lower
    column index, emitted in ascending index order (the block rule of
    ``topk_blocks`` at column granularity)."""
    m = np.asarray(col_mass, dtype=np.float64)
    order = np.lexsort((np.arange(len(m)), -m))
    return np.sort(order[:k]).astype(np.int32)


def column_sparse_attention(q, k, v, scale, cols):
    """Every query row of one head attends to the kept key columns only, in
    ascending column order: softmax attention over k[cols], v[cols]."""
    cols = np.asarray(cols, dtype=np.int64)
    return softmax_attention(q, np.asarray(k)[cols], np.asarray(v)[cols], scale)


def select_columns(q, k, v, scale, keep_ratio):
    """One full-attention pass that also yields the per-head column pattern
    (PulseCol abstract: the sparse pattern is identified at an early denoising
    step). q, k, v are [H, L, d]. Returns dict with o [H,L,d], lse [H,L],
    col_mass [H,L], cols [H, kc] (ascending per head)."""
    H, L, _ = q.shape
    kc = column_keep(L, keep_ratio)
    o = np.empty(q.shape)
    lse = np.empty((H, L))
    mass = np.empty((H, L))
    cols = np.empty((H, kc), dtype=np.int32)
    for h in range(H):
        o[h], lse[h] = dense_attention(q[h], k[h], v[h], scale)
        mass[h] = column_mass(q[h], k[h], scale, lse[h])
        cols[h] = topk_columns(mass[h], kc)
    return dict(o=o, lse=lse, col_mass=mass, cols=cols)


def run_steps_columns(q, k, v, scale, keep_ratio, T, warmup_frac, refresh_every=0):
    """The denoising loop with the column-sparse pattern (PulseCol abstract:
    the pattern is identified early, reused, and refreshed at a few
    intermediate steps): the step kinds of ``schedule``; SELECT runs
    ``select_columns``, SPARSE ``column_sparse_attention`` with the cached
    columns. Returns (o, lse, kinds, pattern) of the last step."""
    kinds = schedule(T, warmup_frac, refresh_every)
    H, L, _ = q.shape
    pattern = None
    o = lse = None
    for t in range(T):
        if kinds[t] == DENSE:
            o = np.empty(q.shape)
            lse = np.empty((H, L))
            for h in range(H):
                o[h], lse[h] = dense_attention(q[h], k[h], v[h], scale)
        elif kinds[t] == SELECT:
            pattern = select_columns(q, k, v, scale, keep_ratio)
            o, lse = pattern["o"], pattern["lse"]
        else:
            o = np.empty(q.shape)
            lse = np.empty((H, L))
            for h in range(H):
                o[h], lse[h] = column_sparse_attention(q[h], k[h], v[h], scale, pattern["cols"][h])
    return o, lse, kinds, pattern


def effective_flops(bq, bk, d, kept_blocks):
    """Flops of QK^T plus PV over the kept blocks: 4 * bq * bk * d per block."""
    return 4.0 * bq * bk * d * float(kept_blocks)

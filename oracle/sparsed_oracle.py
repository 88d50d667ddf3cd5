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
* LoSA: Locality Aware Sparse Attention for Block-Wise Diffusion Language
  Models (a Dutch summary page) -- block-wise generation over a prefix KV
  cache: per step, tokens whose query changed are "active" and get sparse
  prefix attention over the union of their selections; "stable" tokens reuse
  their cached prefix output; prefix and in-block parts are merged by their
  log-sum-exp (section 1, the union cost; section 2, locality of the query
  change; section 3, the method and its workflow).

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
DRIFT_AMPLITUDE = 2.0 ** -6  # default size of the per-step query drift (O6b)

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
    All-zero weights split evenly by the same rule.

    The floors never sum above ``total``: the quotas sum to ``total`` up to a
    relative error of a few ulps, so the fractional parts sum to an integer m
    (up to that error), and a computed quota can cross an integer from below
    only when its exact fractional part is within an ulp of 1; m + 1 such
    crossings would need fractional parts summing to about m + 1 > m. The
    remainder is therefore never negative (asserted)."""
    w = [float(x) for x in weights]
    sw = sum(w)
    if sw <= 0.0:
        w = [1.0] * len(w)
        sw = float(len(w))
    quota = [total * x / sw for x in w]
    base = [math.floor(x) for x in quota]
    rem = total - sum(base)
    assert rem >= 0, "floors of the quotas exceed the total"
    order = sorted(range(len(w)), key=lambda a: (-(quota[a] - base[a]), a))
    for a in order[:rem]:
        base[a] += 1
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
              refresh_every=0, drift_seed=None, drift_amplitude=DRIFT_AMPLITUDE, patterns=None):
    """The denoising loop over one layer: each step runs the kind ``schedule``
    gives; SELECT refreshes the cached pattern; SPARSE uses the cached pattern.
    With ``drift_seed`` the queries of step t are drift_queries(q, drift_seed,
    t) (K and V fixed), otherwise q at every step. ``patterns`` (a list), when
    given, receives every SELECT step's (t, pattern). Returns (o, lse, kinds,
    pattern) of the last step."""
    kinds = schedule(T, warmup_frac, refresh_every)
    H, L, _ = q.shape
    pattern = None
    o = lse = None
    q_fixed = q
    for t in range(T):
        q = q_fixed if drift_seed is None else drift_queries(q_fixed, drift_seed, t, drift_amplitude)
        if kinds[t] == DENSE:
            o = np.empty(q.shape)
            lse = np.empty((H, L))
            for h in range(H):
                o[h], lse[h] = dense_attention(q[h], k[h], v[h], scale)
        elif kinds[t] == SELECT:
            pattern = select_pattern(q, k, v, scale, bq, bk, keep_ratio, budget)
            o, lse = pattern["o"], pattern["lse"]
            if patterns is not None:
                patterns.append((t, pattern))
        else:
            o = np.empty(q.shape)
            lse = np.empty((H, L))
            for h in range(H):
                o[h], lse[h] = masked_attention(q[h], k[h], v[h], scale,
                                                pattern["kv_idx"][h],
                                                pattern["kv_count"][h], bq, bk)
    return o, lse, kinds, pattern


# --------------------------------------------------------------------------
# O6b  queries that change across the denoising steps
# --------------------------------------------------------------------------


def fmix32(x):
    """MurmurHash3's 32-bit finalizer (Austin Appleby's published definition):
    h ^= h >> 16; h *= 0x85ebca6b; h ^= h >> 13; h *= 0xc2b2ae35; h ^= h >> 16,
    all modulo 2^32. Elementwise on an integer array."""
    h = np.asarray(x, dtype=np.uint64) & 0xFFFFFFFF
    h = h ^ (h >> 16)
    h = (h * 0x85EBCA6B) & 0xFFFFFFFF
    h = h ^ (h >> 13)
    h = (h * 0xC2B2AE35) & 0xFFFFFFFF
    h = h ^ (h >> 16)
    return h


def drift_uniform(seed, t, n):
    """The counter-based uniforms of step t: for element i of a tensor of n
    elements, key = fmix32(fmix32(seed) ^ t) and u = (fmix32(i ^ key) >> 8) *
    2^-23 - 1, on a 2^-23 grid in [-1, 1). Returned in float64 (exact)."""
    key = int(fmix32(int(fmix32(seed)) ^ (int(t) & 0xFFFFFFFF)))
    i = np.arange(n, dtype=np.uint64)
    h = fmix32(i ^ key)
    return (h >> 8).astype(np.float64) * 2.0 ** -23 - 1.0


def bf16_round(x32):
    """Round float32 values to bf16, nearest even (finite inputs), returned as
    float64."""
    b = np.asarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def drift_queries(q, seed, t, amplitude=DRIFT_AMPLITUDE):
    """Q of denoising step t: Q_t = bf16(fp32(Q) + fp32(amplitude * u)) elementwise,
    u = drift_uniform(seed, t, Q.size) in the row-major order of Q [H, L, d].

    The pages give no per-step activations. They say that attention patterns
    stay similar across steps (SparseD abstract) and are only locally
    consistent, shifting at some transitions (Step-dLLM abstract). The reading
    taken: a small seeded perturbation of the queries at every step, the same
    bits on any machine (integer hash, one fp32 addition and one bf16
    rounding). ``q`` holds bf16 values (float64 or float32); amplitude a power
    of two keeps amplitude * u exact in fp32."""
    q32 = np.asarray(q, dtype=np.float32)
    u = drift_uniform(seed, t, q32.size).reshape(q32.shape)
    d32 = (u * float(amplitude)).astype(np.float32)
    return bf16_round(q32 + d32)


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


# --------------------------------------------------------------------------
# O8  block-wise generation with active-token reuse (LoSA)
# --------------------------------------------------------------------------
#
# Setting (LoSA page, section 1): a block of B tokens is denoised over several
# steps on top of a prefix of P tokens whose keys and values are cached and
# fixed while the block is generated. At every step each block token attends
# bidirectionally to the whole block (the "suffix": the block's own current
# keys and values) and to the prefix. Arrays: one head is [rows, d]; all heads
# are [H, rows, d]; prefix key block j covers positions [j*bk, min((j+1)*bk, P)).


def merge_partials(o1, lse1, o2, lse2):
    """Attention over the union of two disjoint key sets from the attention
    over each set: with m = max(lse1, lse2) and w_i = exp(lse_i - m),
        o = (w1*o1 + w2*o2) / (w1 + w2),   lse = m + ln(w1 + w2).

    LoSA page, section 3 (methodology), workflow: the prefix and suffix
    contributions are combined by online softmax; this is that identity
    applied once. A part over no keys (lse = -inf) contributes nothing; two
    empty parts give o = 0, lse = -inf."""
    o1, o2 = np.asarray(o1, dtype=np.float64), np.asarray(o2, dtype=np.float64)
    lse1, lse2 = np.asarray(lse1, dtype=np.float64), np.asarray(lse2, dtype=np.float64)
    m = np.maximum(lse1, lse2)
    both_empty = np.isneginf(m)
    msafe = np.where(both_empty, 0.0, m)
    w1 = np.where(np.isneginf(lse1), 0.0, np.exp(lse1 - msafe))
    w2 = np.where(np.isneginf(lse2), 0.0, np.exp(lse2 - msafe))
    z = w1 + w2
    zsafe = np.where(both_empty, 1.0, z)
    o = (w1[..., None] * o1 + w2[..., None] * o2) / zsafe[..., None]
    o = np.where(both_empty[..., None], 0.0, o)
    lse = np.where(both_empty, -np.inf, msafe + np.log(zsafe))
    return o, lse


def query_mse(q_t, q_prev):
    """Locality score of every block token: the mean squared change of its
    query between two consecutive denoising steps,
        mse_b = 1/(H*d) * sum_h sum_c (q_t[h,b,c] - q_prev[h,b,c])^2.

    LoSA page, section 2 (only a few tokens change much between steps t-1 and
    t, shown by MSE measurements) and section 3 (locality pruning measures the
    query change of every token by MSE at the start of a step). Reading taken:
    one score per token over its whole query vector (every head), so all heads
    share one active set. q_t, q_prev are [H, B, d]; returns [B]."""
    diff = np.asarray(q_t, dtype=np.float64) - np.asarray(q_prev, dtype=np.float64)
    return (diff * diff).mean(axis=(0, 2))


def active_tokens(mse, tau):
    """Active tokens: mse_b > tau, strictly (LoSA page, section 3: tokens with
    a high change are active, the rest stable). Reading taken: "high" is a
    caller-given threshold tau, an fp32 value widened to double."""
    return np.asarray(mse, dtype=np.float64) > float(np.float32(tau))


def token_block_mass(q, k_pre, scale, lse, bk):
    """Per-token prefix block mass of one head,
        M[b, j] = sum over prefix keys c in block j of exp(scale*<q_b,k_c> - lse_b),
    i.e. the block mass of O2 with query blocks of a single row.

    The selector of the active tokens (LoSA page, section 3: the method works
    with any sparse selector; the page names QUEST only by name). Reading
    taken: the selector of the SparseD abstract -- the pattern is computed once
    from full attention and reused -- at token granularity: each block token's
    prefix blocks are scored by its post-softmax mass in the block's first,
    dense step, with ``lse`` that step's prefix LSE of the token."""
    return block_mass(q, k_pre, scale, lse, 1, bk)


def token_select(M, n_sel):
    """Per token, its ``n_sel`` prefix blocks of largest mass (``topk_blocks``:
    ties to the lower block, ascending). n_sel is clamped to [1, nkb].
    Returns [B, n_sel'] int32."""
    M = np.asarray(M, dtype=np.float64)
    k = min(max(int(n_sel), 1), M.shape[1])
    return np.stack([topk_blocks(M[b], k) for b in range(M.shape[0])]).astype(np.int32)


def kv_union(sel, active):
    """The prefix blocks one head loads in a step: the union, over the active
    tokens, of their selected blocks, ascending (LoSA page, section 1: the cost
    of a block's sparse attention is set by the union of the positions its
    queries select; section 3: the selector's output for the active tokens only
    forms the union that is loaded). Returns int32 [u]."""
    rows = np.nonzero(np.asarray(active))[0]
    if rows.size == 0:
        return np.zeros(0, dtype=np.int32)
    return np.unique(np.asarray(sel)[rows].ravel()).astype(np.int32)


def prefix_attention(q_rows, k_pre, v_pre, scale, blocks, bk):
    """Attention of the given query rows over every prefix key of the listed
    blocks, in ascending key order (LoSA page, section 3: only the union's
    positions are loaded and the active tokens' prefix attention is computed
    over them). Reading taken: each active token attends to the whole loaded
    union, not only to its own selection."""
    keys = kept_keys(blocks, bk, np.asarray(k_pre).shape[0])
    return softmax_attention(q_rows, np.asarray(k_pre)[keys], np.asarray(v_pre)[keys], scale)


def losa_init(q, k, v, k_pre, v_pre, scale, bk, n_sel, sel=None):
    """First denoising step of a block (LoSA page, section 3, workflow,
    initialisation: dense attention fills the cache).

    For every head and block token: the prefix attention over all P prefix
    keys is the cached prefix output and LSE; its per-token block mass gives
    the token's ``n_sel`` blocks (``token_block_mass``); the suffix attention
    is dense over the block; the step's output merges the two.
    q, k, v: [H, B, d]; k_pre, v_pre: [H, P, d]. ``sel`` (optional, [H, B,
    n_sel']) replaces the selection, so that the later steps can be followed
    from a selection made elsewhere. Returns dict with o [H,B,d], lse [H,B],
    mass [H,B,nkb] and state = {o_pre, lse_pre, sel [H,B,n_sel']}."""
    H, B, d = np.asarray(q).shape
    o = np.empty((H, B, d))
    lse = np.empty((H, B))
    o_pre = np.empty((H, B, d))
    lse_pre = np.empty((H, B))
    nkb = n_blocks(np.asarray(k_pre).shape[1], bk)
    mass = np.empty((H, B, nkb))
    sels = []
    for h in range(H):
        o_pre[h], lse_pre[h] = dense_attention(q[h], k_pre[h], v_pre[h], scale)
        mass[h] = token_block_mass(q[h], k_pre[h], scale, lse_pre[h], bk)
        sels.append(token_select(mass[h], n_sel) if sel is None else np.asarray(sel[h], dtype=np.int32))
        o_suf, lse_suf = dense_attention(q[h], k[h], v[h], scale)
        o[h], lse[h] = merge_partials(o_pre[h], lse_pre[h], o_suf, lse_suf)
    state = dict(o_pre=o_pre, lse_pre=lse_pre, sel=np.stack(sels))
    return dict(o=o, lse=lse, mass=mass, state=state)


def losa_step(q, k, v, q_prev, k_pre, v_pre, scale, bk, tau, state):
    """A later denoising step of the block (LoSA page, section 3, workflow,
    iteration), in the page's order:
      1. locality scores (``query_mse``) against the previous step's queries,
         active tokens (``active_tokens``);
      2. per head, the union of the active tokens' selected blocks
         (``kv_union``);
      3. only those blocks are read;
      4. the active tokens' prefix attention over the union replaces their
         cached prefix output and LSE; stable tokens keep theirs (section 3,
         reuse for stable tokens);
      5. every token's suffix attention (dense over the block) is merged with
         its prefix part (``merge_partials``).
    ``state`` (from ``losa_init`` or an earlier step) is updated in place.
    Returns dict with o, lse, mse [B], active [B] bool, union (list of H
    int32 arrays)."""
    H, B, d = np.asarray(q).shape
    mse = query_mse(q, q_prev)
    act = active_tokens(mse, tau)
    rows = np.nonzero(act)[0]
    o = np.empty((H, B, d))
    lse = np.empty((H, B))
    unions = []
    for h in range(H):
        u = kv_union(state["sel"][h], act)
        unions.append(u)
        if rows.size:
            o_a, l_a = prefix_attention(np.asarray(q[h])[rows], k_pre[h], v_pre[h], scale, u, bk)
            state["o_pre"][h][rows] = o_a
            state["lse_pre"][h][rows] = l_a
        o_suf, lse_suf = dense_attention(q[h], k[h], v[h], scale)
        o[h], lse[h] = merge_partials(state["o_pre"][h], state["lse_pre"][h], o_suf, lse_suf)
    return dict(o=o, lse=lse, mse=mse, active=act, union=unions)


def losa_block(qs, ks, vs, k_pre, v_pre, scale, bk, n_sel, tau, sel=None):
    """All T denoising steps of one block: ``losa_init`` at step 0, then
    ``losa_step`` with the previous step's queries. qs, ks, vs: [T, H, B, d].
    Returns dict with o [T,H,B,d], lse [T,H,B], active [T,B] (step 0: all),
    union_count [T,H] (step 0: every prefix block), state. ``sel`` as in
    ``losa_init``."""
    T, H, B, d = np.asarray(qs).shape
    nkb = n_blocks(np.asarray(k_pre).shape[1], bk)
    o = np.empty((T, H, B, d))
    lse = np.empty((T, H, B))
    active = np.ones((T, B), dtype=bool)
    ucount = np.full((T, H), nkb, dtype=np.int64)
    first = losa_init(qs[0], ks[0], vs[0], k_pre, v_pre, scale, bk, n_sel, sel)
    o[0], lse[0] = first["o"], first["lse"]
    state = first["state"]
    for t in range(1, T):
        r = losa_step(qs[t], ks[t], vs[t], qs[t - 1], k_pre, v_pre, scale, bk, tau, state)
        o[t], lse[t] = r["o"], r["lse"]
        active[t] = r["active"]
        ucount[t] = [len(u) for u in r["union"]]
    return dict(o=o, lse=lse, active=active, union_count=ucount, state=state)

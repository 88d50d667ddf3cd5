"""Seeded synthetic inputs for the benchmark workloads.

This module holds no attention arithmetic. It only draws Q, K, V (and the
structure terms each workload describes) from a seeded torch CPU generator in
fp32, adds the structure in fp32 and rounds once to bf16 (round to nearest
even). The CUDA path and the fp64 oracle both consume exactly these bf16 bits;
nothing here is shared with either implementation of the method.

Workloads (shapes from the SparseD / Step-dLLM setting: bidirectional
attention of a diffusion LM, one layer, every head over all query-key pairs):

* ``tiny``      H=4,  L=1024,  d=64,  bq=bk=64,  keep 0.25, i.i.d. N(0,1)
* ``c2_8k``     H=32, L=8192,  d=128, keep 0.10, 10% of key positions per head
                get +2.0 on every component (distinct hot columns per head)
* ``c3_16k``    H=32, L=16384, keep 0.15, Q/K = rank-8 signal + N(0, 0.5^2)
                noise, per-head seeded factors, anchor refresh every 64 steps
* ``c4_64k``    H=32, L=65536, keep 0.10, i.i.d. N(0,1) plus a banded local
                term on a seeded half of the heads
* ``c5_32k_entropy``  as c4 at L=32768, head-adaptive (entropy) budget

The banded term: seeded N(0,1) anchor vectors every 512 positions, linearly
interpolated to every position p as z(p); z(p) is added to both Q[p] and K[p],
so scores are raised for |i-j| within a few hundred positions and fall off by
about 1024.

Block-wise workloads (the LoSA setting: a block of B tokens denoised over T
steps on a prefix of P cached tokens), ``BLOCK_WORKLOADS``:

* ``losa_tiny``  H=2,  P=1000,  B=48, d=64,  bq=bk=64, 3 blocks per token, T=4
* ``losa_32k``   H=32, P=32768, B=64, d=128, bq=bk=64, 2 blocks per token
                 (128 prefix positions, the page's tightest budget), T=16

Prefix K, V ~ N(0,1) with 10% of the prefix positions of every head raised by
+2.0 on every key component (as c2_8k). The block's Q, K, V start from N(0,1)
and evolve in fp32: at every step t >= 1 a seeded round(0.25*B) tokens change
by N(0, 0.5^2) per element (active), every other token by N(0, 0.02^2)
(stable); each step's tensors are the fp32 state rounded to bf16. The query
MSE of an active token is then about 0.25 and of a stable one about 4e-4, on
either side of the threshold tau = 0.01.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

BAND_PERIOD = 512
LOW_RANK = 8


@dataclass(frozen=True)
class Workload:
    name: str
    H: int
    L: int
    d: int
    bq: int
    bk: int
    keep: float
    T: int
    warmup_frac: float
    refresh_every: int
    budget: str          # "uniform" | "entropy"
    structure: str       # "iid" | "key_bias" | "low_rank" | "band"
    seed: int

    @property
    def scale(self) -> float:
        """1/sqrt(d) rounded to fp32, the value passed through the C ABI."""
        return float(torch.tensor(1.0 / math.sqrt(self.d), dtype=torch.float32))

    def scaled(self, **kw) -> "Workload":
        """Same recipe with some fields overridden (smaller H or L for tests)."""
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 4, 1024, 64, 64, 64, 0.25, 2, 0.5, 0,
                     "uniform", "iid", 1001),
    "c2_8k": Workload("c2_8k", 32, 8192, 128, 128, 128, 0.10, 256, 0.2, 0,
                      "uniform", "key_bias", 1002),
    "c3_16k": Workload("c3_16k", 32, 16384, 128, 128, 128, 0.15, 512, 0.2, 64,
                       "uniform", "low_rank", 1003),
    "c4_64k": Workload("c4_64k", 32, 65536, 128, 128, 128, 0.10, 1024, 0.2, 0,
                       "uniform", "band", 1004),
    "c5_32k_entropy": Workload("c5_32k_entropy", 32, 32768, 128, 128, 128, 0.10,
                               256, 0.2, 0, "entropy", "band", 1005),
}


def _band_term(L: int, d: int, g: torch.Generator) -> torch.Tensor:
    n_anchor = L // BAND_PERIOD + 2
    anchors = torch.randn(n_anchor, d, generator=g)
    p = torch.arange(L)
    a = p // BAND_PERIOD
    t = ((p % BAND_PERIOD).to(torch.float32) / BAND_PERIOD).unsqueeze(1)
    return (1.0 - t) * anchors[a] + t * anchors[a + 1]


def make_inputs(wl: Workload, device: str | torch.device = "cpu"):
    """Return (q, k, v) as bf16 tensors of shape [H, L, d] on ``device``.

    Draw order is fixed: Q, K, V, then the structure terms, all from one
    ``torch.Generator('cpu').manual_seed(wl.seed)``.
    """
    H, L, d = wl.H, wl.L, wl.d
    g = torch.Generator("cpu").manual_seed(wl.seed)
    shape = (H, L, d)
    if wl.structure == "low_rank":
        q = torch.randn(shape, generator=g).mul_(0.5)
        k = torch.randn(shape, generator=g).mul_(0.5)
    else:
        q = torch.randn(shape, generator=g)
        k = torch.randn(shape, generator=g)
    v = torch.randn(shape, generator=g)

    if wl.structure == "key_bias":
        n_hot = int(round(0.1 * L))
        for h in range(H):
            pos = torch.randperm(L, generator=g)[:n_hot]
            k[h, pos, :] += 2.0
    elif wl.structure == "low_rank":
        for h in range(H):
            u = torch.randn(L, LOW_RANK, generator=g)
            w = torch.randn(LOW_RANK, d, generator=g).mul_(1.0 / math.sqrt(LOW_RANK))
            sig = u @ w
            q[h] += sig
            k[h] += sig
    elif wl.structure == "band":
        heads = torch.randperm(H, generator=g)[: H // 2].sort().values
        for h in heads.tolist():
            z = _band_term(L, d, g)
            q[h] += z
            k[h] += z
    elif wl.structure != "iid":
        raise ValueError(f"unknown structure {wl.structure!r}")

    out = []
    for t in (q, k, v):
        b = t.to(torch.bfloat16)
        out.append(b.to(device) if str(device) != "cpu" else b)
    return tuple(out)


def zero_q(wl: Workload):
    """Degenerate input: Q = 0 (all scores exactly 0), K and V from the recipe."""
    q, k, v = make_inputs(wl)
    return torch.zeros_like(q), k, v


def to_f64(t: torch.Tensor):
    """Exact widening of bf16 bits to a float64 numpy array (no arithmetic)."""
    return t.detach().to("cpu").to(torch.float64).numpy()


@dataclass(frozen=True)
class BlockWorkload:
    name: str
    H: int
    P: int            # prefix tokens (cached keys and values)
    B: int            # block tokens
    d: int
    bq: int
    bk: int
    n_sel: int        # prefix blocks selected per token
    T: int            # denoising steps of the block
    active_frac: float
    tau: float
    seed: int

    @property
    def scale(self) -> float:
        return float(torch.tensor(1.0 / math.sqrt(self.d), dtype=torch.float32))

    def scaled(self, **kw) -> "BlockWorkload":
        return replace(self, **kw)


BLOCK_WORKLOADS = {
    "losa_tiny": BlockWorkload("losa_tiny", 2, 1000, 48, 64, 64, 64, 3, 4, 0.25, 0.01, 2001),
    "losa_32k": BlockWorkload("losa_32k", 32, 32768, 64, 128, 64, 64, 2, 16, 0.25, 0.01, 2002),
}

ACTIVE_STD = 0.5
STABLE_STD = 0.02


def make_block_inputs(wl: BlockWorkload, device: str | torch.device = "cpu"):
    """Return (k_pre, v_pre, qs, ks, vs): the prefix [H, P, d] and the block's
    per-step tensors [T, H, B, d], all bf16 on ``device``.

    Draw order: prefix K, prefix V, the hot positions of each head, block Q,
    K, V at step 0, then per step the active set and the changes of Q, K, V.
    """
    H, P, B, d, T = wl.H, wl.P, wl.B, wl.d, wl.T
    g = torch.Generator("cpu").manual_seed(wl.seed)
    k_pre = torch.randn((H, P, d), generator=g)
    v_pre = torch.randn((H, P, d), generator=g)
    n_hot = int(round(0.1 * P))
    for h in range(H):
        pos = torch.randperm(P, generator=g)[:n_hot]
        k_pre[h, pos, :] += 2.0
    state = [torch.randn((H, B, d), generator=g) for _ in range(3)]
    n_act = int(round(wl.active_frac * B))
    steps = [[t.to(torch.bfloat16) for t in state]]
    for _ in range(1, T):
        act = torch.randperm(B, generator=g)[:n_act]
        std = torch.full((B,), STABLE_STD)
        std[act] = ACTIVE_STD
        for i in range(3):
            state[i] = state[i] + torch.randn((H, B, d), generator=g) * std[None, :, None]
        steps.append([t.to(torch.bfloat16) for t in state])
    qs, ks, vs = (torch.stack([s[i] for s in steps]) for i in range(3))
    out = [k_pre.to(torch.bfloat16), v_pre.to(torch.bfloat16), qs, ks, vs]
    if str(device) != "cpu":
        out = [t.to(device) for t in out]
    return tuple(out)

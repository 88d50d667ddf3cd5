"""Block-sparse bidirectional attention for diffusion-LM denoising on B200.

Thin Python binding over the C ABI of libsparsed.so (include/sparsed.h). Each
function checks and marshals torch tensors (device memory, dtype, contiguity)
and passes raw pointers plus the current CUDA stream; every step of the
computation runs in the library's sm_100a kernels. torch is used only for
device memory and streams.

    dense_attn(q, k, v)                      -> (o, lse)
    select_pattern(q, k, v, keep, budget)    -> Pattern (o, lse, kv_idx, kv_count, ...)
    block_sparse_attn(q, k, v, kv_idx, kv_count) -> (o, lse)
    run_steps(q, k, v, T, warmup_frac, ...)  -> RunResult (o, lse, kinds, step_ms, pattern)

Head-sharded selection (the heads of one layer over several ranks; only the
per-head entropies cross ranks):

    select_pattern_sharded(q, k, v, keep, group) -> Pattern for this rank's heads

Column-sparse path (per-head kept key columns shared by all queries):

    select_columns(q, k, v, keep)            -> ColumnPattern (o, lse, cols, col_mass)
    column_sparse_attn(q, k, v, cols)        -> (o, lse)
    run_steps_columns(q, k, v, T, warmup_frac, ...) -> RunResult (kv_idx holds cols [H, kc])

Block-wise generation over a prefix cache with active-token reuse (a block
of B tokens denoised over T steps; q, k, v of the block are [H, B, d]):

    losa_init(q, k, v, k_pre, v_pre, n_sel)  -> (o, lse, BlockState)
    losa_step(q, k, v, q_prev, k_pre, v_pre, state, tau) -> LosaStep
    losa_block(qs, ks, vs, k_pre, v_pre, n_sel, tau) -> LosaBlock (all T steps)

q, k, v are [H, L, d] bf16 CUDA tensors (d in {64, 128}); o is [H, L, d] bf16,
lse [H, L] fp32 natural log; kv_idx [H, nqb, kv_stride] int32 and kv_count
[H, nqb] int32 hold the per-(head, query block) kept key blocks, ascending.
"""
from __future__ import annotations

import ctypes
import math
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import (BUDGET_ENTROPY, BUDGET_UNIFORM, STEP_DENSE, STEP_SELECT,  # noqa: F401
                   STEP_SPARSE, SparsedError, check)

__all__ = ["dense_attn", "select_pattern", "block_sparse_attn", "run_steps", "workspace_bytes",
           "run_steps_workspace_bytes", "drift_queries", "DRIFT_AMPLITUDE",
           "uniform_keep", "schedule", "device_check", "version", "SparsedError", "Pattern",
           "RunResult", "default_scale", "column_keep", "column_workspace_bytes", "select_columns",
           "column_sparse_attn", "run_steps_columns", "ColumnPattern", "select_head_entropy",
           "entropy_budget", "select_with_head_k", "select_pattern_sharded", "gather_head_entropies",
           "run_steps_sharded",
           "losa_splits", "losa_workspace_bytes", "losa_init", "losa_step", "losa_block", "BlockState",
           "LosaStep", "LosaBlock"]


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check_qkv(q, k, v):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor")
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
        if t.device.type != "cuda":
            raise ValueError(f"{name} must be a CUDA tensor")
        if t.dim() != 3 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous [H, L, d] tensor")
    if not (q.shape == k.shape == v.shape):
        raise ValueError(f"q, k, v shapes differ: {tuple(q.shape)} {tuple(k.shape)} {tuple(v.shape)}")
    if not (q.device == k.device == v.device):
        raise ValueError("q, k, v must be on the same device")
    return q.shape


def default_scale(d: int) -> float:
    """1/sqrt(d) rounded to fp32 (the value the C ABI receives)."""
    return float(torch.tensor(1.0 / math.sqrt(d), dtype=torch.float32))


def version() -> int:
    return _lib.load().sparsed_version()


def uniform_keep(L: int, bk: int, keep: float) -> int:
    k = ctypes.c_int()
    check(_lib.load().sparsed_uniform_keep(L, bk, keep, ctypes.byref(k)), "sparsed_uniform_keep")
    return k.value


def schedule(T: int, warmup_frac: float, refresh_every: int = 0) -> list[int]:
    buf = (ctypes.c_int8 * max(T, 1))()
    check(_lib.load().sparsed_schedule(T, warmup_frac, refresh_every, ctypes.cast(buf, ctypes.c_void_p)),
          "sparsed_schedule")
    return list(buf[:T])


def workspace_bytes(H: int, L: int, bq: int = 128, bk: int = 128) -> int:
    n = ctypes.c_size_t()
    check(_lib.load().sparsed_workspace_bytes(H, L, bq, bk, ctypes.byref(n)), "sparsed_workspace_bytes")
    return n.value


def run_steps_workspace_bytes(H: int, L: int, bq: int = 128, bk: int = 128) -> int:
    """Workspace with which run_steps fuses the block mass into its selecting passes."""
    n = ctypes.c_size_t()
    check(_lib.load().sparsed_run_steps_workspace_bytes(H, L, bq, bk, ctypes.byref(n)),
          "sparsed_run_steps_workspace_bytes")
    return n.value


def device_check(stream=None) -> None:
    """Synchronise the stream and raise if a kernel recorded a device-side fault."""
    check(_lib.load().sparsed_check(_stream(stream)), "sparsed_check")


def _alloc_out(q, out, lse):
    H, L, _ = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((H, L), dtype=torch.float32, device=q.device)
    return out, lse


def _workspace(q, bq, bk, workspace):
    H, L, _ = q.shape
    need = workspace_bytes(H, L, bq, bk)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    return workspace


def dense_attn(q, k, v, scale=None, bq=128, bk=128, out=None, lse=None, stream=None):
    """Dense bidirectional attention: returns (o [H,L,d] bf16, lse [H,L] fp32)."""
    H, L, d = _check_qkv(q, k, v)
    scale = default_scale(d) if scale is None else scale
    out, lse = _alloc_out(q, out, lse)
    rc = _lib.load().sparsed_dense_attn(_ptr(q), _ptr(k), _ptr(v), H, L, d, scale, bq, bk, _ptr(out),
                                        _ptr(lse), _stream(stream))
    check(rc, "sparsed_dense_attn")
    return out, lse


@dataclass
class Pattern:
    o: torch.Tensor
    lse: torch.Tensor
    kv_idx: torch.Tensor       # [H, nqb, kv_stride] int32
    kv_count: torch.Tensor     # [H, nqb] int32
    block_mass: torch.Tensor | None
    head_k: torch.Tensor       # [H] int32


def select_pattern(q, k, v, keep=0.1, budget="uniform", scale=None, bq=128, bk=128, kv_stride=None,
                   return_mass=False, workspace=None, stream=None) -> Pattern:
    """Full-attention pass plus block-sparse pattern selection."""
    H, L, d = _check_qkv(q, k, v)
    scale = default_scale(d) if scale is None else scale
    mode = {"uniform": BUDGET_UNIFORM, "entropy": BUDGET_ENTROPY}[budget]
    nqb, nkb = -(-L // bq), -(-L // bk)
    if kv_stride is None:
        kv_stride = uniform_keep(L, bk, keep) if (mode == BUDGET_UNIFORM and L > 0) else max(nkb, 1)
    dev = q.device
    out, lse = _alloc_out(q, None, None)
    kv_idx = torch.full((H, nqb, kv_stride), -1, dtype=torch.int32, device=dev)
    kv_count = torch.zeros((H, nqb), dtype=torch.int32, device=dev)
    mass = torch.empty((H, nqb, nkb), dtype=torch.float32, device=dev) if return_mass else None
    head_k = torch.zeros(H, dtype=torch.int32, device=dev)
    ws = _workspace(q, bq, bk, workspace)
    rc = _lib.load().sparsed_select_pattern(
        _ptr(q), _ptr(k), _ptr(v), H, L, d, scale, bq, bk, keep, mode, _ptr(out), _ptr(lse),
        _ptr(kv_idx), _ptr(kv_count), kv_stride, _ptr(mass), _ptr(head_k), _ptr(ws), ws.numel(),
        _stream(stream))
    check(rc, "sparsed_select_pattern")
    return Pattern(out, lse, kv_idx, kv_count, mass, head_k)


def block_sparse_attn(q, k, v, kv_idx, kv_count, scale=None, bq=128, bk=128, out=None, lse=None,
                      stream=None):
    """Block-sparse attention over a cached pattern: returns (o, lse)."""
    H, L, d = _check_qkv(q, k, v)
    scale = default_scale(d) if scale is None else scale
    for name, t in (("kv_idx", kv_idx), ("kv_count", kv_count)):
        if t.dtype != torch.int32 or not t.is_contiguous() or t.device != q.device:
            raise ValueError(f"{name} must be a contiguous int32 tensor on {q.device}")
    nqb = -(-L // bq)
    if kv_idx.dim() != 3 or kv_idx.shape[:2] != (H, nqb) or kv_count.shape != (H, nqb):
        raise ValueError(f"pattern shapes must be [H, nqb, stride] and [H, nqb] with nqb={nqb}")
    out, lse = _alloc_out(q, out, lse)
    rc = _lib.load().sparsed_block_sparse_attn(
        _ptr(q), _ptr(k), _ptr(v), H, L, d, scale, bq, bk, _ptr(kv_idx), _ptr(kv_count),
        kv_idx.shape[2], _ptr(out), _ptr(lse), _stream(stream))
    check(rc, "sparsed_block_sparse_attn")
    return out, lse


@dataclass
class RunResult:
    o: torch.Tensor
    lse: torch.Tensor
    kinds: list
    step_ms: list | None
    kv_idx: torch.Tensor
    kv_count: torch.Tensor


DRIFT_AMPLITUDE = 2.0 ** -6


def drift_queries(q, seed: int, t: int, amplitude: float = DRIFT_AMPLITUDE, out=None, stream=None):
    """The queries of denoising step t (sparsed_drift_queries): a seeded
    perturbation of q, the same bits on any machine."""
    H, L, d = q.shape
    if q.dtype != torch.bfloat16 or not q.is_cuda or not q.is_contiguous():
        raise ValueError("q must be a contiguous bfloat16 CUDA tensor [H, L, d]")
    out = torch.empty_like(q) if out is None else out
    check(_lib.load().sparsed_drift_queries(_ptr(q), H, L, d, seed & 0xFFFFFFFF, t, amplitude, _ptr(out),
                                            _stream(stream)), "sparsed_drift_queries")
    return out


def run_steps(q, k, v, T, warmup_frac=0.2, keep=0.1, budget="uniform", refresh_every=0, scale=None,
              bq=128, bk=128, start_step=0, pattern=None, time_steps=False, out=None, lse=None,
              workspace=None, stream=None, end_step=None, drift_seed=None,
              drift_amplitude=DRIFT_AMPLITUDE) -> RunResult:
    """The denoising loop over one layer: dense warm-up, pattern selection at
    the switch (and at anchors), block-sparse attention afterwards. With
    ``end_step`` only steps start_step .. end_step-1 of the T-step schedule run.
    With ``drift_seed`` every step t attends with its own queries,
    drift_queries(q, drift_seed, t, drift_amplitude) (K and V fixed)."""
    H, L, d = _check_qkv(q, k, v)
    scale = default_scale(d) if scale is None else scale
    mode = {"uniform": BUDGET_UNIFORM, "entropy": BUDGET_ENTROPY}[budget]
    nqb, nkb = -(-L // bq), -(-L // bk)
    if pattern is not None:
        kv_idx, kv_count = pattern
        have = 1
    else:
        stride = uniform_keep(L, bk, keep) if (mode == BUDGET_UNIFORM and L > 0) else max(nkb, 1)
        kv_idx = torch.full((H, nqb, stride), -1, dtype=torch.int32, device=q.device)
        kv_count = torch.zeros((H, nqb), dtype=torch.int32, device=q.device)
        have = 0
    out, lse = _alloc_out(q, out, lse)
    if workspace is None:
        workspace = torch.empty(run_steps_workspace_bytes(H, L, bq, bk), dtype=torch.uint8, device=q.device)
    ws = workspace
    kinds = (ctypes.c_int8 * max(T, 1))()
    ms = (ctypes.c_float * max(T, 1))() if time_steps else None
    tail = (_ptr(kv_idx), _ptr(kv_count), kv_idx.shape[2], _ptr(out), _ptr(lse),
            ctypes.cast(kinds, ctypes.c_void_p), None if ms is None else ctypes.cast(ms, ctypes.c_void_p),
            _ptr(ws), ws.numel(), _stream(stream))
    if drift_seed is not None:
        q_step = torch.empty_like(q)
        rc = _lib.load().sparsed_run_steps_drift(_ptr(q), _ptr(k), _ptr(v), H, L, d, scale, bq, bk, keep, mode,
                                                 T, warmup_frac, refresh_every, start_step,
                                                 T if end_step is None else end_step, have,
                                                 drift_seed & 0xFFFFFFFF, drift_amplitude, _ptr(q_step), *tail)
        check(rc, "sparsed_run_steps_drift")
    elif end_step is None:
        rc = _lib.load().sparsed_run_steps(_ptr(q), _ptr(k), _ptr(v), H, L, d, scale, bq, bk, keep, mode, T,
                                           warmup_frac, refresh_every, start_step, have, *tail)
        check(rc, "sparsed_run_steps")
    else:
        rc = _lib.load().sparsed_run_steps_span(_ptr(q), _ptr(k), _ptr(v), H, L, d, scale, bq, bk, keep, mode,
                                                T, warmup_frac, refresh_every, start_step, end_step, have,
                                                *tail)
        check(rc, "sparsed_run_steps_span")
    return RunResult(out, lse, list(kinds[:T]), None if ms is None else list(ms[:T]), kv_idx, kv_count)


# ---------------------------------------------------------------- column path

def column_keep(L: int, keep: float) -> int:
    kc = ctypes.c_int()
    check(_lib.load().sparsed_column_keep(L, keep, ctypes.byref(kc)), "sparsed_column_keep")
    return kc.value


def column_workspace_bytes(H: int, L: int, d: int, kc: int) -> int:
    n = ctypes.c_size_t()
    check(_lib.load().sparsed_column_workspace_bytes(H, L, d, kc, ctypes.byref(n)),
          "sparsed_column_workspace_bytes")
    return n.value


def _col_workspace(q, kc, workspace):
    H, L, d = q.shape
    need = column_workspace_bytes(H, L, d, kc)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    return workspace


@dataclass
class ColumnPattern:
    o: torch.Tensor
    lse: torch.Tensor
    cols: torch.Tensor              # [H, kc] int32, ascending per head
    col_mass: torch.Tensor | None   # [H, L] fp32


def select_columns(q, k, v, keep=0.1, scale=None, bq=128, bk=128, return_mass=False, workspace=None,
                   stream=None) -> ColumnPattern:
    """Full-attention pass plus per-head column selection (column mass, top-k)."""
    H, L, d = _check_qkv(q, k, v)
    scale = default_scale(d) if scale is None else scale
    kc = column_keep(L, keep) if L > 0 else 1
    out, lse = _alloc_out(q, None, None)
    cols = torch.full((H, kc), -1, dtype=torch.int32, device=q.device)
    mass = torch.empty((H, L), dtype=torch.float32, device=q.device) if return_mass else None
    ws = _col_workspace(q, kc, workspace)
    rc = _lib.load().sparsed_select_columns(
        _ptr(q), _ptr(k), _ptr(v), H, L, d, scale, bq, bk, keep, _ptr(out), _ptr(lse), _ptr(cols), kc,
        _ptr(mass), _ptr(ws), ws.numel(), _stream(stream))
    check(rc, "sparsed_select_columns")
    return ColumnPattern(out, lse, cols, mass)


def column_sparse_attn(q, k, v, cols, scale=None, bq=128, bk=128, out=None, lse=None, workspace=None,
                       stream=None):
    """Attention of every query over its head's kept columns: returns (o, lse)."""
    H, L, d = _check_qkv(q, k, v)
    scale = default_scale(d) if scale is None else scale
    if cols.dtype != torch.int32 or not cols.is_contiguous() or cols.device != q.device or cols.dim() != 2 \
            or cols.shape[0] != H:
        raise ValueError(f"cols must be a contiguous [H, kc] int32 tensor on {q.device}")
    kc = cols.shape[1]
    out, lse = _alloc_out(q, out, lse)
    ws = _col_workspace(q, kc, workspace)
    rc = _lib.load().sparsed_column_sparse_attn(
        _ptr(q), _ptr(k), _ptr(v), H, L, d, scale, bq, bk, _ptr(cols), kc, kc, _ptr(out), _ptr(lse),
        _ptr(ws), ws.numel(), _stream(stream))
    check(rc, "sparsed_column_sparse_attn")
    return out, lse


def run_steps_columns(q, k, v, T, warmup_frac=0.2, keep=0.1, refresh_every=0, scale=None, bq=128, bk=128,
                      start_step=0, cols=None, time_steps=False, out=None, lse=None, workspace=None,
                      stream=None) -> RunResult:
    """The denoising loop with the column pattern: dense warm-up, column
    selection at the switch (and at refreshes), column-sparse attention
    afterwards. The result's kv_idx holds the columns [H, kc]."""
    H, L, d = _check_qkv(q, k, v)
    scale = default_scale(d) if scale is None else scale
    kc = column_keep(L, keep) if L > 0 else 1
    have = 1 if cols is not None else 0
    if cols is None:
        cols = torch.full((H, kc), -1, dtype=torch.int32, device=q.device)
    out, lse = _alloc_out(q, out, lse)
    ws = _col_workspace(q, kc, workspace)
    kinds = (ctypes.c_int8 * max(T, 1))()
    ms = (ctypes.c_float * max(T, 1))() if time_steps else None
    rc = _lib.load().sparsed_run_steps_columns(
        _ptr(q), _ptr(k), _ptr(v), H, L, d, scale, bq, bk, keep, T, warmup_frac, refresh_every, start_step,
        have, _ptr(cols), cols.shape[1], _ptr(out), _ptr(lse), ctypes.cast(kinds, ctypes.c_void_p),
        None if ms is None else ctypes.cast(ms, ctypes.c_void_p), _ptr(ws), ws.numel(), _stream(stream))
    check(rc, "sparsed_run_steps_columns")
    return RunResult(out, lse, list(kinds[:T]), None if ms is None else list(ms[:T]), cols, None)


# ---------------------------------------------------------------- head-sharded selection

def select_head_entropy(q, k, v, scale=None, bq=128, bk=128, workspace=None, stream=None, out=None, lse=None):
    """Full pass, block mass and the mean row entropy of every head:
    returns (o, lse, head_entropy [H] fp64 on the device, workspace). The
    workspace keeps the block mass for select_with_head_k."""
    H, L, d = _check_qkv(q, k, v)
    scale = default_scale(d) if scale is None else scale
    out, lse = _alloc_out(q, out, lse)
    ent = torch.empty(H, dtype=torch.float64, device=q.device)
    ws = _workspace(q, bq, bk, workspace)
    rc = _lib.load().sparsed_select_head_entropy(_ptr(q), _ptr(k), _ptr(v), H, L, d, scale, bq, bk, _ptr(out),
                                                 _ptr(lse), _ptr(ent), _ptr(ws), ws.numel(), _stream(stream))
    check(rc, "sparsed_select_head_entropy")
    return out, lse, ent, ws


def entropy_budget(head_entropy, nkb: int, keep: float) -> list[int]:
    """The head-adaptive allocation on the host, from the entropies of all
    heads of a layer (any float sequence) to k_h per head."""
    vals = [float(x) for x in head_entropy]
    H = len(vals)
    src = (ctypes.c_double * max(H, 1))(*vals)
    dst = (ctypes.c_int32 * max(H, 1))()
    check(_lib.load().sparsed_entropy_budget(ctypes.cast(src, ctypes.c_void_p), H, nkb, keep,
                                             ctypes.cast(dst, ctypes.c_void_p)), "sparsed_entropy_budget")
    return list(dst[:H])


def select_with_head_k(H, L, head_k, workspace, bq=128, bk=128, stream=None):
    """Top-k per (head, query block) with given k_h over the block mass a
    preceding select_head_entropy left in ``workspace``: (kv_idx, kv_count)."""
    dev = workspace.device
    nqb, nkb = -(-L // bq), -(-L // bk)
    hk = torch.as_tensor(head_k, dtype=torch.int32).to(dev).contiguous()
    kv_idx = torch.full((H, nqb, max(nkb, 1)), -1, dtype=torch.int32, device=dev)
    kv_count = torch.zeros((H, nqb), dtype=torch.int32, device=dev)
    rc = _lib.load().sparsed_select_with_head_k(H, L, bq, bk, _ptr(hk), _ptr(kv_idx), _ptr(kv_count),
                                                kv_idx.shape[2], _ptr(workspace), workspace.numel(),
                                                _stream(stream))
    check(rc, "sparsed_select_with_head_k")
    return kv_idx, kv_count, hk


def gather_head_entropies(ent, group=None):
    """All ranks' per-head entropies in rank order (a CPU fp64 tensor) and
    this rank's index; the identity without a group. NCCL gathers device
    tensors, other backends host tensors."""
    if group is None:
        return ent.cpu(), 0
    import torch.distributed as dist
    world = dist.get_world_size(group)
    mine = ent if dist.get_backend(group) == "nccl" else ent.cpu()
    parts = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(parts, mine, group=group)
    return torch.cat([t.cpu() for t in parts]), dist.get_rank(group)


def select_pattern_sharded(q, k, v, keep=0.1, group=None, scale=None, bq=128, bk=128, workspace=None,
                           stream=None, out=None, lse=None, gather=None) -> Pattern:
    """Entropy-budget pattern selection for this rank's heads of a layer whose
    heads are split evenly over the ranks of ``group`` (in rank order). The
    per-head entropies are all-gathered, every rank runs the same host
    allocation over all heads, and keeps its own heads' k_h. Without a group
    the local heads are the whole layer. ``gather`` (optional) replaces the
    all-gather: a function from this rank's entropies to (all entropies in
    head order as a CPU tensor, this rank's index)."""
    H, L, d = _check_qkv(q, k, v)
    out, lse, ent, ws = select_head_entropy(q, k, v, scale, bq, bk, workspace, stream, out, lse)
    ent_all, rank = gather(ent) if gather is not None else gather_head_entropies(ent, group)
    nkb = -(-L // bk)
    head_k_all = entropy_budget(ent_all.tolist(), nkb, keep)
    kv_idx, kv_count, hk = select_with_head_k(H, L, head_k_all[rank * H:(rank + 1) * H], ws, bq, bk, stream)
    return Pattern(out, lse, kv_idx, kv_count, None, hk)


# ---------------------------------------------------------------- block-wise generation with active-token reuse

def losa_splits(H: int, B: int, P: int, bq: int = 64, bk: int = 64, sm_count: int | None = None) -> int:
    """Splits of a head's block list for a step of these sizes (sm_count: the
    current device's SM count by default)."""
    if sm_count is None:
        sm_count = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    s = ctypes.c_int()
    check(_lib.load().sparsed_losa_splits(H, B, bq, P, bk, sm_count, ctypes.byref(s)), "sparsed_losa_splits")
    return s.value


def losa_workspace_bytes(H: int, B: int, P: int, d: int, bq: int = 64, bk: int = 64, splits: int = 1) -> int:
    n = ctypes.c_size_t()
    check(_lib.load().sparsed_losa_workspace_bytes(H, B, P, d, bq, bk, splits, ctypes.byref(n)),
          "sparsed_losa_workspace_bytes")
    return n.value


@dataclass
class BlockState:
    """What a block carries across its denoising steps (caller memory)."""
    o_cache: torch.Tensor    # [H, B, d] bf16: every token's prefix attention output
    lse_cache: torch.Tensor  # [H, B] fp32: its LSE over the prefix keys it attended
    sel: torch.Tensor        # [H, B, n_sel] int32: each token's prefix blocks, ascending
    scale: float
    bq: int
    bk: int
    splits: int
    workspace: torch.Tensor


@dataclass
class LosaStep:
    o: torch.Tensor
    lse: torch.Tensor
    active: torch.Tensor            # [B] int32 0/1
    union_count: torch.Tensor       # [H] int32
    union_idx: torch.Tensor | None  # [H, nkb] int32, first union_count[h] entries


@dataclass
class LosaBlock:
    o: torch.Tensor            # [T, H, B, d]
    lse: torch.Tensor          # [T, H, B]
    active: torch.Tensor       # [T, B] int32 (step 0: all 1)
    union_count: torch.Tensor  # [T, H] int32 (step 0: nkb)
    state: BlockState


def _check_prefix(k_pre, v_pre, H, d, device):
    for name, t in (("k_pre", k_pre), ("v_pre", v_pre)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or t.device != device \
                or t.dim() != 3 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous [H, P, d] bf16 tensor on {device}")
    if k_pre.shape != v_pre.shape or k_pre.shape[0] != H or k_pre.shape[2] != d:
        raise ValueError(f"prefix shapes {tuple(k_pre.shape)} / {tuple(v_pre.shape)} do not match H={H}, d={d}")
    return k_pre.shape[1]


def _block_state(q, P, n_sel, scale, bq, bk, splits, workspace):
    H, B, d = q.shape
    splits = losa_splits(H, B, P, bq, bk) if splits is None else splits
    need = losa_workspace_bytes(H, B, P, d, bq, bk, splits)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    return BlockState(torch.empty_like(q), torch.empty((H, B), dtype=torch.float32, device=q.device),
                      torch.empty((H, B, n_sel), dtype=torch.int32, device=q.device), scale, bq, bk, splits,
                      workspace)


def losa_init(q, k, v, k_pre, v_pre, n_sel=2, scale=None, bq=64, bk=64, splits=None, return_mass=False,
              workspace=None, stream=None):
    """First denoising step of a block: dense prefix attention of every token
    (the cache), each token's n_sel prefix blocks, the block's own attention
    and the merged output. Returns (o, lse, state) or (o, lse, state, mass)."""
    H, B, d = _check_qkv(q, k, v)
    P = _check_prefix(k_pre, v_pre, H, d, q.device)
    scale = default_scale(d) if scale is None else scale
    nkb = (P + bk - 1) // bk
    n_sel = max(1, min(n_sel, nkb))  # a token cannot keep more blocks than the prefix has
    st = _block_state(q, P, n_sel, scale, bq, bk, splits, workspace)
    out, lse = _alloc_out(q, None, None)
    mass = torch.empty((H, B, nkb), dtype=torch.float32, device=q.device) if return_mass else None
    rc = _lib.load().sparsed_losa_init(
        _ptr(q), _ptr(k), _ptr(v), _ptr(k_pre), _ptr(v_pre), H, B, P, d, scale, bq, bk, n_sel, st.splits,
        _ptr(st.o_cache), _ptr(st.lse_cache), _ptr(st.sel), _ptr(out), _ptr(lse), _ptr(mass),
        _ptr(st.workspace), st.workspace.numel(), _stream(stream))
    check(rc, "sparsed_losa_init")
    return (out, lse, st, mass) if return_mass else (out, lse, st)


def losa_step(q, k, v, q_prev, k_pre, v_pre, state: BlockState, tau: float, return_union=False,
              stream=None) -> LosaStep:
    """A later step of the block: active tokens by query MSE against q_prev,
    the union of their blocks, their prefix attention over it (cache update),
    the block's own attention, and the merge. Updates ``state`` in place."""
    H, B, d = _check_qkv(q, k, v)
    if not isinstance(q_prev, torch.Tensor) or q_prev.dtype != torch.bfloat16 or q_prev.shape != q.shape \
            or q_prev.device != q.device or not q_prev.is_contiguous():
        raise ValueError(f"q_prev must be a contiguous bf16 tensor shaped like q {tuple(q.shape)} on {q.device}")
    P = _check_prefix(k_pre, v_pre, H, d, q.device)
    n_sel = state.sel.shape[2]
    out, lse = _alloc_out(q, None, None)
    active = torch.empty(B, dtype=torch.int32, device=q.device)
    ucount = torch.empty(H, dtype=torch.int32, device=q.device)
    nkb = (P + state.bk - 1) // state.bk
    uidx = torch.empty((H, nkb), dtype=torch.int32, device=q.device) if return_union else None
    rc = _lib.load().sparsed_losa_step(
        _ptr(q), _ptr(k), _ptr(v), _ptr(q_prev), _ptr(k_pre), _ptr(v_pre), H, B, P, d, state.scale, state.bq,
        state.bk, n_sel, tau, state.splits, _ptr(state.o_cache), _ptr(state.lse_cache), _ptr(state.sel),
        _ptr(out), _ptr(lse), _ptr(active), _ptr(uidx), _ptr(ucount), _ptr(state.workspace),
        state.workspace.numel(), _stream(stream))
    check(rc, "sparsed_losa_step")
    return LosaStep(out, lse, active, ucount, uidx)


def losa_block(qs, ks, vs, k_pre, v_pre, n_sel=2, tau=0.01, scale=None, bq=64, bk=64, splits=None, out=None,
               lse=None, workspace=None, stream=None) -> LosaBlock:
    """All T steps of one block (qs, ks, vs: [T, H, B, d] bf16): the first
    step dense, every later one with active-token reuse."""
    for name, t in (("qs", qs), ("ks", ks), ("vs", vs)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or t.device.type != "cuda" \
                or t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous [T, H, B, d] bf16 CUDA tensor")
    if not (qs.shape == ks.shape == vs.shape):
        raise ValueError("qs, ks, vs shapes differ")
    T, H, B, d = qs.shape
    P = _check_prefix(k_pre, v_pre, H, d, qs.device)
    scale = default_scale(d) if scale is None else scale
    n_sel = max(1, min(n_sel, (P + bk - 1) // bk))
    st = _block_state(qs[0], P, n_sel, scale, bq, bk, splits, workspace)
    if out is None:
        out = torch.empty_like(qs)
    if lse is None:
        lse = torch.empty((T, H, B), dtype=torch.float32, device=qs.device)
    if out.shape != qs.shape or out.dtype != torch.bfloat16 or out.device != qs.device or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous bf16 tensor shaped {tuple(qs.shape)} on {qs.device}")
    if lse.shape != (T, H, B) or lse.dtype != torch.float32 or lse.device != qs.device or not lse.is_contiguous():
        raise ValueError(f"lse must be a contiguous fp32 tensor shaped {(T, H, B)} on {qs.device}")
    active = torch.empty((T, B), dtype=torch.int32, device=qs.device)
    ucount = torch.empty((T, H), dtype=torch.int32, device=qs.device)
    rc = _lib.load().sparsed_losa_block(
        _ptr(qs), _ptr(ks), _ptr(vs), _ptr(k_pre), _ptr(v_pre), T, H, B, P, d, scale, bq, bk, n_sel, tau,
        st.splits, _ptr(st.o_cache), _ptr(st.lse_cache), _ptr(st.sel), _ptr(out), _ptr(lse), _ptr(active),
        _ptr(ucount), _ptr(st.workspace), st.workspace.numel(), _stream(stream))
    check(rc, "sparsed_losa_block")
    return LosaBlock(out, lse, active, ucount, st)


# ---------------------------------------------------------------- head-sharded denoising loop

_EXCHANGE_FN = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.POINTER(ctypes.c_double), ctypes.c_int,
                                ctypes.POINTER(ctypes.c_double), ctypes.c_int, ctypes.c_void_p)


def run_steps_sharded(q, k, v, T, warmup_frac=0.2, keep=0.1, budget="entropy", refresh_every=0, group=None,
                      scale=None, bq=128, bk=128, out=None, lse=None, workspace=None, stream=None,
                      gather=None, rank=None, world=None) -> RunResult:
    """The denoising loop for this rank's heads of a layer whose heads are
    split evenly over the ranks of ``group`` (rank order = head order), run by
    the C driver sparsed_run_steps_sharded.

    A uniform budget is per head, so nothing crosses ranks. The entropy budget
    spans every head of the layer: at each SELECT step the driver calls back
    here with the local per-head entropies, which are all-gathered over
    ``group`` (gather_head_entropies: NCCL for device tensors, other backends
    host tensors). ``gather`` (optional, with ``rank`` and ``world``) replaces
    the all-gather: a function from this rank's entropies (a CPU fp64 tensor)
    to (all entropies in head order as a CPU tensor, this rank's index).
    Without a group or gather the local heads are the whole layer."""
    H, L, d = _check_qkv(q, k, v)
    scale = default_scale(d) if scale is None else scale
    mode = {"uniform": BUDGET_UNIFORM, "entropy": BUDGET_ENTROPY}[budget]
    if group is not None:
        import torch.distributed as dist
        rank, world = dist.get_rank(group), dist.get_world_size(group)
    elif gather is None:
        rank, world = 0, 1
    elif rank is None or world is None:
        raise ValueError("a custom gather needs this rank's index and the number of ranks")
    nqb, nkb = -(-L // bq), -(-L // bk)
    out, lse = _alloc_out(q, out, lse)
    if workspace is None:
        workspace = torch.empty(run_steps_workspace_bytes(H, L, bq, bk), dtype=torch.uint8, device=q.device)
    stride = uniform_keep(L, bk, keep) if (mode == BUDGET_UNIFORM and L > 0) else max(nkb, 1)
    kv_idx = torch.full((H, nqb, stride), -1, dtype=torch.int32, device=q.device)
    kv_count = torch.zeros((H, nqb), dtype=torch.int32, device=q.device)
    kinds = (ctypes.c_int8 * max(T, 1))()
    errors = []

    def exchange(local_ptr, h_local, all_ptr, h_total, _user):
        try:
            local = torch.tensor([local_ptr[i] for i in range(h_local)], dtype=torch.float64)
            if gather is not None:
                ent_all, _ = gather(local)
            elif group is not None:
                import torch.distributed as dist
                mine = local.to(q.device) if dist.get_backend(group) == "nccl" else local
                ent_all, _ = gather_head_entropies(mine, group)
            else:
                ent_all = local
            vals = [float(x) for x in ent_all]
            if len(vals) != h_total:
                raise ValueError(f"gathered {len(vals)} head entropies, the layer has {h_total}")
            for i, x in enumerate(vals):
                all_ptr[i] = x
            return 0
        except Exception as e:  # reported after the C call returns
            errors.append(e)
            return 1

    cb = _EXCHANGE_FN(exchange)
    rc = _lib.load().sparsed_run_steps_sharded(
        _ptr(q), _ptr(k), _ptr(v), H, L, d, scale, bq, bk, keep, mode, H * world, H * rank, T, warmup_frac,
        refresh_every, _ptr(kv_idx), _ptr(kv_count), kv_idx.shape[2], _ptr(out), _ptr(lse),
        ctypes.cast(kinds, ctypes.c_void_p), ctypes.cast(cb, ctypes.c_void_p), None, _ptr(workspace),
        workspace.numel(), _stream(stream))
    if errors:
        raise errors[0]
    check(rc, "sparsed_run_steps_sharded")
    return RunResult(out, lse, list(kinds[:T]), None, kv_idx, kv_count)

"""The allocation-free pattern selection entry point.

sparsed_select_pattern_noalloc serves callers that may not allocate device
memory (a host framework that owns the device-memory budget through its own
pool, or latency-critical loops where cudaMalloc/cudaFree would synchronise
the device): it takes no workspace and uses a fixed scratch array inside the
library. These tests call it through the C ABI and check it against
sparsed_select_pattern, which uses a caller workspace, on two calls in a row
with different inputs and budgets, so stale scratch from the first call would
show in the second. This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

from block_sparse_bidirectional_select_b200 import _lib
from block_sparse_bidirectional_select_b200.inputs import WORKLOADS, make_inputs
from gpu_common import LSE_MAX_ABS, O_MAX_ABS, O_MEAN_ABS

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 16 << 20


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _outputs(H, L, d, bq, bk, stride):
    nqb, nkb = -(-L // bq), -(-L // bk)
    return dict(
        o=torch.empty((H, L, d), dtype=torch.bfloat16, device="cuda"),
        lse=torch.empty((H, L), dtype=torch.float32, device="cuda"),
        kv_idx=torch.full((H, nqb, stride), -1, dtype=torch.int32, device="cuda"),
        kv_count=torch.zeros((H, nqb), dtype=torch.int32, device="cuda"),
        mass=torch.empty((H, nqb, nkb), dtype=torch.float32, device="cuda"),
        head_k=torch.zeros(H, dtype=torch.int32, device="cuda"),
    )


def _run(lib, noalloc, q, k, v, scale, bq, bk, keep, mode, out, stride):
    H, L, d = q.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    common = [_p(q), _p(k), _p(v), H, L, d, scale, bq, bk, keep, mode, _p(out["o"]), _p(out["lse"]),
              _p(out["kv_idx"]), _p(out["kv_count"]), stride, _p(out["mass"]), _p(out["head_k"])]
    if noalloc:
        rc = lib.sparsed_select_pattern_noalloc(*common, stream)
    else:
        nbytes = ctypes.c_size_t()
        assert lib.sparsed_workspace_bytes(H, L, bq, bk, ctypes.byref(nbytes)) == 0
        ws = torch.empty(nbytes.value, dtype=torch.uint8, device="cuda")
        rc = lib.sparsed_select_pattern(*common, _p(ws), nbytes.value, stream)
    assert rc == 0, lib.sparsed_strerror(rc)
    assert lib.sparsed_check(stream) == 0


def _compare(ref, got):
    err = (ref["o"].float() - got["o"].float()).abs()
    assert err.max().item() <= O_MAX_ABS and err.mean().item() <= O_MEAN_ABS
    assert (ref["lse"] - got["lse"]).abs().max().item() <= LSE_MAX_ABS
    assert torch.equal(ref["kv_count"], got["kv_count"])
    assert torch.equal(ref["kv_idx"], got["kv_idx"])
    assert torch.equal(ref["head_k"], got["head_k"])
    assert torch.allclose(ref["mass"], got["mass"], rtol=1e-6, atol=0)


CASES = [
    # (name, H, L, d, bq, bk, keep, budget, seed) -- two different calls in a row
    ("band, entropy budget", 4, 2048, 128, 128, 128, 0.2, _lib.BUDGET_ENTROPY, 71),
    ("iid, uniform budget, ragged L", 3, 1000, 64, 64, 64, 0.25, _lib.BUDGET_UNIFORM, 72),
]


def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row():
    lib = _lib.load()
    for name, H, L, d, bq, bk, keep, mode, seed in CASES:
        structure = "band" if "band" in name else "iid"
        wl = WORKLOADS["tiny"].scaled(H=H, L=L, d=d, seed=seed, structure=structure)
        q, k, v = (t.cuda() for t in make_inputs(wl))
        nkb = -(-L // bk)
        stride = nkb
        ref = _outputs(H, L, d, bq, bk, stride)
        got = _outputs(H, L, d, bq, bk, stride)
        _run(lib, False, q, k, v, wl.scale, bq, bk, keep, mode, ref, stride)
        _run(lib, True, q, k, v, wl.scale, bq, bk, keep, mode, got, stride)
        torch.cuda.synchronize()
        _compare(ref, got)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = _lib.load()
    H, L, d = 32, 65536, 128  # block-mass grid alone is 32 MiB > 16 MiB
    nbytes = ctypes.c_size_t()
    assert lib.sparsed_workspace_bytes(H, L, 128, 128, ctypes.byref(nbytes)) == 0
    assert nbytes.value > SCRATCH_BYTES
    P = ctypes.c_void_p(0x10000)
    rc = lib.sparsed_select_pattern_noalloc(P, P, P, H, L, d, 0.088, 128, 128, 0.1, 0, P, P, P, P, 52,
                                            None, None, None)
    assert rc == _lib.ERR_WORKSPACE

"""ctypes loader for libsparsed.so (the C ABI declared in include/sparsed.h).

The library is built in-tree by ``build.py``. If it is missing this module
raises: there is no fallback implementation of any entry point.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsparsed.so")

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_WORKSPACE = -3
ERR_BAD_PATTERN = -4
ERR_CUDA = -5
ERR_DEVICE_TIMEOUT = -6
ERR_NO_DEVICE = -7
ERR_EXCHANGE = -8

BUDGET_UNIFORM = 0
BUDGET_ENTROPY = 1
STEP_DENSE, STEP_SELECT, STEP_SPARSE = 0, 1, 2

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t

# name -> (restype, argtypes); mirrors include/sparsed.h
SIGNATURES = {
    "sparsed_version": (_I, []),
    "sparsed_strerror": (ctypes.c_char_p, [_I]),
    "sparsed_last_cuda_error": (_I, []),
    "sparsed_check": (_I, [_P]),
    "sparsed_selftest_wait_timeout": (_I, [ctypes.c_ulonglong, _P]),
    "sparsed_uniform_keep": (_I, [_I, _I, _F, ctypes.POINTER(_I)]),
    "sparsed_schedule": (_I, [_I, _F, _I, _P]),
    "sparsed_workspace_bytes": (_I, [_I, _I, _I, _I, ctypes.POINTER(_SZ)]),
    "sparsed_dense_attn": (_I, [_P, _P, _P, _I, _I, _I, _F, _I, _I, _P, _P, _P]),
    "sparsed_select_pattern": (_I, [_P, _P, _P, _I, _I, _I, _F, _I, _I, _F, _I, _P, _P, _P, _P, _I,
                                    _P, _P, _P, _SZ, _P]),
    "sparsed_block_sparse_attn": (_I, [_P, _P, _P, _I, _I, _I, _F, _I, _I, _P, _P, _I, _P, _P, _P]),
    "sparsed_select_pattern_noalloc": (_I, [_P, _P, _P, _I, _I, _I, _F, _I, _I, _F, _I, _P, _P, _P, _P,
                                            _I, _P, _P, _P]),
    "sparsed_run_steps": (_I, [_P, _P, _P, _I, _I, _I, _F, _I, _I, _F, _I, _I, _F, _I, _I, _I, _P, _P,
                               _I, _P, _P, _P, _P, _P, _SZ, _P]),
    "sparsed_run_steps_workspace_bytes": (_I, [_I, _I, _I, _I, ctypes.POINTER(_SZ)]),
    "sparsed_drift_queries": (_I, [_P, _I, _I, _I, ctypes.c_uint, _I, _F, _P, _P]),
    "sparsed_run_steps_sharded": (_I, [_P, _P, _P, _I, _I, _I, _F, _I, _I, _F, _I, _I, _I, _I, _F, _I, _P, _P,
                                       _I, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "sparsed_run_steps_drift": (_I, [_P, _P, _P, _I, _I, _I, _F, _I, _I, _F, _I, _I, _F, _I, _I, _I, _I,
                                     ctypes.c_uint, _F, _P, _P, _P, _I, _P, _P, _P, _P, _P, _SZ, _P]),
    "sparsed_run_steps_span": (_I, [_P, _P, _P, _I, _I, _I, _F, _I, _I, _F, _I, _I, _F, _I, _I, _I, _I, _P,
                                    _P, _I, _P, _P, _P, _P, _P, _SZ, _P]),
    "sparsed_select_head_entropy": (_I, [_P, _P, _P, _I, _I, _I, _F, _I, _I, _P, _P, _P, _P, _SZ, _P]),
    "sparsed_entropy_budget": (_I, [_P, _I, _I, _F, _P]),
    "sparsed_select_with_head_k": (_I, [_I, _I, _I, _I, _P, _P, _P, _I, _P, _SZ, _P]),
    "sparsed_column_keep": (_I, [_I, _F, ctypes.POINTER(_I)]),
    "sparsed_column_workspace_bytes": (_I, [_I, _I, _I, _I, ctypes.POINTER(_SZ)]),
    "sparsed_select_columns": (_I, [_P, _P, _P, _I, _I, _I, _F, _I, _I, _F, _P, _P, _P, _I, _P, _P, _SZ, _P]),
    "sparsed_column_sparse_attn": (_I, [_P, _P, _P, _I, _I, _I, _F, _I, _I, _P, _I, _I, _P, _P, _P, _SZ, _P]),
    "sparsed_run_steps_columns": (_I, [_P, _P, _P, _I, _I, _I, _F, _I, _I, _F, _I, _F, _I, _I, _I, _P, _I,
                                       _P, _P, _P, _P, _P, _SZ, _P]),
    "sparsed_losa_splits": (_I, [_I, _I, _I, _I, _I, _I, ctypes.POINTER(_I)]),
    "sparsed_losa_workspace_bytes": (_I, [_I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_SZ)]),
    "sparsed_losa_init": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _I, _I, _I, _P, _P, _P, _P, _P,
                               _P, _P, _SZ, _P]),
    "sparsed_losa_step": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _I, _I, _F, _I, _P, _P, _P,
                               _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "sparsed_losa_block": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _I, _I, _F, _I, _P, _P, _P,
                                _P, _P, _P, _P, _P, _SZ, _P]),
}

_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libsparsed.so once and attach the declared signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python -m block_sparse_bidirectional_select_b200.build`"
            " (nvcc, sm_100a). There is no CPU fallback.")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class SparsedError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = status
        msg = load().sparsed_strerror(status).decode()
        extra = ""
        if status == ERR_CUDA:
            extra = f" (cudaError {load().sparsed_last_cuda_error()})"
        super().__init__(f"{where}: status {status}: {msg}{extra}")


def check(status: int, where: str) -> None:
    if status != OK:
        raise SparsedError(status, where)

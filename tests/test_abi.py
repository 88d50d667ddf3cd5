"""The C ABI without a GPU: the library loads, exports every symbol the header
declares, and its host-side logic (argument validation, budgets, schedule,
workspace sizing) behaves as documented. No compute call reaches a device."""
import ctypes
import os
import re

import pytest
import torch

import oracle as O
import block_sparse_bidirectional_select_b200 as sp
from block_sparse_bidirectional_select_b200 import _lib

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "sparsed.h")
lib = _lib.load()
GPU = torch.cuda.is_available()
P = ctypes.c_void_p(0x10000)          # aligned, never dereferenced by these calls
MIS = ctypes.c_void_p(0x10008)        # 8-byte aligned only


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sparsed_\w+)\s*\(", text)))


def test_header_symbols_exported():
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), f"{n} declared in sparsed.h but not exported"
    assert set(names) == set(_lib.SIGNATURES)


def test_version_and_strerror():
    assert sp.version() == 100
    for code in range(-7, 1):
        msg = lib.sparsed_strerror(code)
        assert msg and len(msg) > 1
    assert lib.sparsed_strerror(-99) == b"unknown status"


@pytest.mark.parametrize("L,bk", [(8192, 128), (65536, 128), (1000, 64), (1, 128), (130, 64)])
def test_uniform_keep_matches_oracle(L, bk):
    nkb = -(-L // bk)
    for keep in (0.01, 0.1, 0.15, 0.25, 0.3333, 0.5, 0.999, 1.0):
        assert sp.uniform_keep(L, bk, keep) == O.uniform_keep(nkb, keep)


def test_uniform_keep_rejects():
    k = ctypes.c_int()
    assert lib.sparsed_uniform_keep(100, 64, 0.0, ctypes.byref(k)) == _lib.ERR_INVALID_ARG
    assert lib.sparsed_uniform_keep(100, 64, 1.5, ctypes.byref(k)) == _lib.ERR_INVALID_ARG
    assert lib.sparsed_uniform_keep(0, 64, 0.5, ctypes.byref(k)) == _lib.ERR_INVALID_ARG


def test_schedule_matches_oracle():
    for T in (1, 2, 3, 5, 17, 256, 512, 1024):
        for w in (0.0, 0.1, 0.2, 0.34, 0.5, 0.99, 1.0):
            for R in (0, 1, 3, 64):
                assert sp.schedule(T, w, R) == O.schedule(T, w, R), (T, w, R)


def test_schedule_rejects():
    buf = (ctypes.c_int8 * 4)()
    assert lib.sparsed_schedule(4, 1.5, 0, ctypes.cast(buf, ctypes.c_void_p)) == _lib.ERR_INVALID_ARG
    assert lib.sparsed_schedule(4, 0.5, -1, ctypes.cast(buf, ctypes.c_void_p)) == _lib.ERR_INVALID_ARG
    assert lib.sparsed_schedule(4, 0.5, 0, None) == _lib.ERR_INVALID_ARG
    assert lib.sparsed_schedule(0, 0.5, 0, None) == _lib.OK


def test_workspace_bytes():
    a = sp.workspace_bytes(32, 8192)
    b = sp.workspace_bytes(32, 65536)
    assert 0 < a < b
    assert a % 256 == 0
    # grid alone is H * nqb * nkb floats
    assert b >= 32 * 512 * 512 * 4
    n = ctypes.c_size_t()
    assert lib.sparsed_workspace_bytes(4, 100, 96, 64, ctypes.byref(n)) == _lib.ERR_UNSUPPORTED


def _dense(Q=P, K=P, V=P, H=2, L=256, d=128, scale=0.088, bq=128, bk=128, O_=P, LSE=P):
    return lib.sparsed_dense_attn(Q, K, V, H, L, d, scale, bq, bk, O_, LSE, None)


def test_dense_validation_before_any_launch():
    assert _dense(d=96) == _lib.ERR_UNSUPPORTED
    assert _dense(bq=32) == _lib.ERR_UNSUPPORTED
    assert _dense(bk=256) == _lib.ERR_UNSUPPORTED
    assert _dense(H=-1) == _lib.ERR_INVALID_ARG
    assert _dense(Q=None) == _lib.ERR_INVALID_ARG
    assert _dense(LSE=None) == _lib.ERR_INVALID_ARG
    assert _dense(K=MIS) == _lib.ERR_INVALID_ARG
    assert _dense(scale=float("nan")) == _lib.ERR_INVALID_ARG
    assert _dense(H=70000) == _lib.ERR_UNSUPPORTED
    assert _dense(H=64, L=1 << 20) == _lib.ERR_UNSUPPORTED   # H*L*d >= 2^31
    # empty problems are no-ops even with null pointers
    assert _dense(Q=None, K=None, V=None, O_=None, LSE=None, H=0) == _lib.OK
    assert _dense(Q=None, K=None, V=None, O_=None, LSE=None, L=0) == _lib.OK


@pytest.mark.skipif(GPU, reason="checks the no-device path")
def test_valid_call_without_device_reports_no_device():
    assert _dense() == _lib.ERR_NO_DEVICE
    assert lib.sparsed_check(None) == _lib.ERR_NO_DEVICE


def _select(keep=0.1, mode=0, stride=7, ws=P, ws_bytes=1 << 30, idx=P, cnt=P, L=8192):
    return lib.sparsed_select_pattern(P, P, P, 2, L, 128, 0.088, 128, 128, keep, mode, P, P, idx, cnt,
                                      stride, None, None, ws, ws_bytes, None)


def test_select_validation():
    assert _select(keep=0.0) == _lib.ERR_INVALID_ARG
    assert _select(keep=1.01) == _lib.ERR_INVALID_ARG
    assert _select(mode=2) == _lib.ERR_INVALID_ARG
    assert _select(stride=6) == _lib.ERR_INVALID_ARG          # k = 7 at keep 0.1, nkb 64
    assert _select(mode=1, stride=63) == _lib.ERR_INVALID_ARG  # entropy needs nkb
    assert _select(idx=None) == _lib.ERR_INVALID_ARG
    assert _select(ws=None) == _lib.ERR_WORKSPACE
    assert _select(ws_bytes=1024) == _lib.ERR_WORKSPACE
    assert _select(ws=ctypes.c_void_p(0x10010)) == _lib.ERR_WORKSPACE  # not 256-aligned
    if not GPU:
        assert _select() == _lib.ERR_NO_DEVICE


def test_block_sparse_validation():
    f = lib.sparsed_block_sparse_attn
    assert f(P, P, P, 2, 256, 128, 0.1, 128, 128, None, P, 4, P, P, None) == _lib.ERR_INVALID_ARG
    assert f(P, P, P, 2, 256, 128, 0.1, 128, 128, P, P, 0, P, P, None) == _lib.ERR_INVALID_ARG
    assert f(P, P, P, 2, 256, 80, 0.1, 128, 128, P, P, 4, P, P, None) == _lib.ERR_UNSUPPORTED


def test_run_steps_validation():
    f = lib.sparsed_run_steps
    args = [P, P, P, 2, 512, 128, 0.088, 128, 128, 0.5, 0, 10, 0.2, 0, 0, 0, P, P, 2, P, P, None, None,
            P, 1 << 20, None]
    a = list(args)
    a[14] = 11                      # start_step > T
    assert f(*a) == _lib.ERR_INVALID_ARG
    a = list(args)
    a[14] = 5                       # resume after the switch without a pattern
    assert f(*a) == _lib.ERR_INVALID_ARG
    a = list(args)
    a[23] = None                    # a SELECT step needs a workspace
    assert f(*a) == _lib.ERR_WORKSPACE
    kinds = (ctypes.c_int8 * 10)()
    a = list(args)
    a[5] = 96                       # unsupported d: the kinds are still reported
    a[21] = ctypes.cast(kinds, ctypes.c_void_p)
    assert f(*a) == _lib.ERR_UNSUPPORTED
    assert list(kinds) == O.schedule(10, 0.2, 0)


def test_python_binding_type_checks():
    q = torch.zeros((1, 64, 64), dtype=torch.float32)
    with pytest.raises(TypeError):
        sp.dense_attn(q, q, q)
    q = torch.zeros((1, 64, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        sp.dense_attn(q, q, q)


def _losa_splits(H=32, B=64, bq=64, P_=32768, bk=64, sms=148):
    s = ctypes.c_int(-1)
    rc = lib.sparsed_losa_splits(H, B, bq, P_, bk, sms, ctypes.byref(s))
    return rc, s.value


def test_losa_splits():
    assert _losa_splits() == (_lib.OK, 4)                      # 148 SMs / 32 work items per split
    assert _losa_splits(B=128) == (_lib.OK, 2)                 # two query tiles per split
    assert _losa_splits(H=200) == (_lib.OK, 1)                 # at least one split
    assert _losa_splits(H=1, P_=100) == (_lib.OK, 1)           # at most ceil(nkb / 4): nkb = 2
    assert _losa_splits(H=1, P_=64 * 40) == (_lib.OK, 10)      # nkb = 40 -> at most 10
    assert _losa_splits(H=1, P_=64 * 1000) == (_lib.OK, 32)    # never more than 32
    assert _losa_splits(sms=0)[0] == _lib.ERR_INVALID_ARG
    assert _losa_splits(bq=32)[0] == _lib.ERR_UNSUPPORTED


def _losa_ws(H=32, B=64, P_=32768, d=128, bq=64, bk=64, splits=4):
    n = ctypes.c_size_t(0)
    rc = lib.sparsed_losa_workspace_bytes(H, B, P_, d, bq, bk, splits, ctypes.byref(n))
    return rc, n.value


def test_losa_workspace_bytes():
    rc, n4 = _losa_ws()
    assert rc == _lib.OK
    # the per-token block mass [H, B, nkb] fp32 and the replicated queries and
    # partial outputs [H, splits*64, d] bf16 are the large parts
    assert n4 >= 32 * 64 * 512 * 4 + 2 * 32 * 4 * 64 * 128 * 2
    assert _losa_ws(splits=8)[1] > n4
    assert _losa_ws(splits=1000)[1] == _losa_ws(splits=128)[1]  # clamped to ceil(nkb / 4)
    assert _losa_ws(B=1025)[0] == _lib.ERR_UNSUPPORTED
    assert _losa_ws(d=96)[0] == _lib.ERR_UNSUPPORTED
    assert _losa_ws(P_=0)[0] == _lib.ERR_INVALID_ARG
    assert _losa_ws(splits=0)[0] == _lib.ERR_INVALID_ARG
    assert _losa_ws(P_=64 * 32768 + 1, H=1, d=64)[0] == _lib.ERR_UNSUPPORTED  # nkb > 32768


def _losa_step(tau=0.01, ws=P, ws_bytes=1 << 30, qprev=P, sel=P, n_sel=2, B=64, active=None, uidx=None,
               ucount=None):
    return lib.sparsed_losa_step(P, P, P, qprev, P, P, 2, B, 4096, 128, 0.088, 64, 64, n_sel, tau, 2,
                                 P, P, sel, P, P, active, uidx, ucount, ws, ws_bytes, None)


def test_losa_step_validation():
    assert _losa_step(tau=float("nan")) == _lib.ERR_INVALID_ARG
    assert _losa_step(tau=-1.0) == _lib.ERR_INVALID_ARG
    assert _losa_step(qprev=None) == _lib.ERR_INVALID_ARG
    assert _losa_step(qprev=MIS) == _lib.ERR_INVALID_ARG
    assert _losa_step(sel=None) == _lib.ERR_INVALID_ARG
    assert _losa_step(n_sel=0) == _lib.ERR_INVALID_ARG
    assert _losa_step(ws=None) == _lib.ERR_WORKSPACE
    assert _losa_step(ws_bytes=4096) == _lib.ERR_WORKSPACE
    assert _losa_step(B=2000) == _lib.ERR_UNSUPPORTED
    # the optional int32 outputs must be 4-byte aligned
    odd = ctypes.c_void_p(0x10002)
    assert _losa_step(active=odd) == _lib.ERR_INVALID_ARG
    assert _losa_step(uidx=odd) == _lib.ERR_INVALID_ARG
    assert _losa_step(ucount=odd) == _lib.ERR_INVALID_ARG
    if not GPU:
        assert _losa_step() == _lib.ERR_NO_DEVICE
        assert _losa_step(active=P, uidx=ctypes.c_void_p(0x10004), ucount=ctypes.c_void_p(0x10008)) == \
            _lib.ERR_NO_DEVICE


def test_losa_block_validation():
    f = lib.sparsed_losa_block
    args = [P, P, P, P, P, 3, 2, 64, 4096, 128, 0.088, 64, 64, 2, 0.01, 2, P, P, P, P, P, None, None,
            P, 1 << 30, None]
    a = list(args)
    a[5] = 0  # T
    assert f(*a) == _lib.ERR_INVALID_ARG
    a = list(args)
    a[21] = ctypes.c_void_p(0x10002)  # actives not 4-byte aligned
    assert f(*a) == _lib.ERR_INVALID_ARG
    if not GPU:
        assert f(*args) == _lib.ERR_NO_DEVICE


def test_run_steps_span_validation():
    f = lib.sparsed_run_steps_span
    # T=10, warm-up 0.2: steps 0 dense, 1 select, 2..9 sparse
    args = [P, P, P, 2, 512, 128, 0.088, 128, 128, 0.5, 0, 10, 0.2, 0, 0, 10, 0, P, P, 2, P, P, None, None,
            P, 1 << 20, None]
    a = list(args)
    a[14], a[15] = 4, 3             # start after end
    assert f(*a) == _lib.ERR_INVALID_ARG
    a = list(args)
    a[15] = 11                      # end past T
    assert f(*a) == _lib.ERR_INVALID_ARG
    a = list(args)
    a[14], a[15] = 2, 5             # sparse steps without a pattern
    assert f(*a) == _lib.ERR_INVALID_ARG
    a = list(args)
    a[14], a[15], a[16] = 2, 5, 1   # ... with one: no workspace needed (no select in the span)
    a[24] = None
    if not GPU:
        assert f(*a) == _lib.ERR_NO_DEVICE
    a = list(args)
    a[14], a[15] = 0, 2             # the span holds the select: it needs the workspace
    a[24] = None
    assert f(*a) == _lib.ERR_WORKSPACE
    a = list(args)
    a[14], a[15] = 3, 3             # an empty span validates and launches nothing
    a[16] = 1
    kinds = (ctypes.c_int8 * 10)()
    a[22] = ctypes.cast(kinds, ctypes.c_void_p)
    rc = f(*a)
    assert list(kinds) == O.schedule(10, 0.2, 0)
    if not GPU:
        assert rc == _lib.ERR_NO_DEVICE


def _losa_init(**kw):
    a = dict(Q=P, K=P, V=P, Kp=P, Vp=P, H=2, B=64, P_=4096, d=128, scale=0.088, bq=64, bk=64, n_sel=2, splits=2,
             oc=P, lc=P, sel=P, O_=P, LSE=P, mass=None, ws=P, ws_bytes=1 << 30)
    a.update(kw)
    return lib.sparsed_losa_init(a["Q"], a["K"], a["V"], a["Kp"], a["Vp"], a["H"], a["B"], a["P_"], a["d"],
                                 a["scale"], a["bq"], a["bk"], a["n_sel"], a["splits"], a["oc"], a["lc"],
                                 a["sel"], a["O_"], a["LSE"], a["mass"], a["ws"], a["ws_bytes"], None)


def test_losa_init_validation():
    assert _losa_init(Kp=None) == _lib.ERR_INVALID_ARG
    assert _losa_init(sel=None) == _lib.ERR_INVALID_ARG
    assert _losa_init(oc=MIS) == _lib.ERR_INVALID_ARG            # the cache must be 16-byte aligned
    assert _losa_init(lc=ctypes.c_void_p(0x10002)) == _lib.ERR_INVALID_ARG
    assert _losa_init(mass=ctypes.c_void_p(0x10001)) == _lib.ERR_INVALID_ARG
    assert _losa_init(scale=float("inf")) == _lib.ERR_INVALID_ARG
    assert _losa_init(d=96) == _lib.ERR_UNSUPPORTED
    assert _losa_init(bk=32) == _lib.ERR_UNSUPPORTED
    assert _losa_init(B=0) == _lib.ERR_INVALID_ARG
    assert _losa_init(P_=0) == _lib.ERR_INVALID_ARG
    assert _losa_init(n_sel=0) == _lib.ERR_INVALID_ARG
    assert _losa_init(splits=0) == _lib.ERR_INVALID_ARG
    assert _losa_init(ws=None) == _lib.ERR_WORKSPACE
    assert _losa_init(ws=ctypes.c_void_p(0x10010)) == _lib.ERR_WORKSPACE   # not 256-byte aligned
    assert _losa_init(ws_bytes=1 << 10) == _lib.ERR_WORKSPACE
    if not GPU:
        assert _losa_init() == _lib.ERR_NO_DEVICE


def test_drift_entry_points_validate_on_the_host():
    f = lib.sparsed_drift_queries
    assert f(None, 2, 64, 64, 1, 0, 0.0156, P, None) == _lib.ERR_INVALID_ARG
    assert f(P, 2, 64, 64, 1, 0, 0.0156, None, None) == _lib.ERR_INVALID_ARG
    assert f(MIS, 2, 64, 64, 1, 0, 0.0156, P, None) == _lib.ERR_INVALID_ARG
    assert f(P, 2, 64, 64, 1, -1, 0.0156, P, None) == _lib.ERR_INVALID_ARG
    assert f(P, 2, 64, 64, 1, 0, float("nan"), P, None) == _lib.ERR_INVALID_ARG
    assert f(P, 2, 64, 96, 1, 0, 0.0156, P, None) == _lib.ERR_UNSUPPORTED
    assert f(P, 0, 64, 64, 1, 0, 0.0156, P, None) == _lib.OK          # empty: nothing to do
    if not GPU:
        assert f(P, 2, 64, 64, 1, 0, 0.0156, P, None) == _lib.ERR_NO_DEVICE
    g = lib.sparsed_run_steps_drift

    def run(q_step=P, amp=0.0156):
        return g(P, P, P, 2, 1024, 64, 0.125, 64, 64, 0.25, 0, 4, 0.5, 0, 0, 4, 0, 7, amp, q_step,
                 P, P, 4, P, P, None, None, P, 1 << 30, None)
    assert run(q_step=None) == _lib.ERR_INVALID_ARG
    assert run(q_step=MIS) == _lib.ERR_INVALID_ARG
    assert run(amp=float("inf")) == _lib.ERR_INVALID_ARG
    if not GPU:
        assert run() == _lib.ERR_NO_DEVICE


def test_sharded_loop_validates_on_the_host():
    f = lib.sparsed_run_steps_sharded

    def run(budget=1, h_total=4, offset=2, exchange=P):
        return f(P, P, P, 2, 1024, 64, 0.125, 64, 64, 0.25, budget, h_total, offset, 8, 0.3, 2,
                 P, P, 16, P, P, None, exchange, None, P, 1 << 30, None)
    assert run(h_total=1) == _lib.ERR_INVALID_ARG          # fewer heads in the layer than here
    assert run(offset=3) == _lib.ERR_INVALID_ARG           # heads past the layer's end
    assert run(offset=-1) == _lib.ERR_INVALID_ARG
    assert run(exchange=None) == _lib.ERR_INVALID_ARG      # the entropy budget needs the exchange
    assert run(budget=5) == _lib.ERR_INVALID_ARG
    assert lib.sparsed_strerror(_lib.ERR_EXCHANGE).decode().startswith("the exchange callback")
    if not GPU:
        assert run() == _lib.ERR_NO_DEVICE
        assert run(budget=0, exchange=None) == _lib.ERR_NO_DEVICE


def _c_kind(decl):
    """Kind of a C parameter or return type: 'ptr' (any pointer, the exchange
    callback), 'int', 'float', 'u64' (size_t, uint64_t), 'u32' (uint32_t)."""
    t = decl.strip()
    if "*" in t or "sparsed_exchange_fn" in t:
        return "ptr"
    t = re.sub(r"\bconst\b", "", t).split()
    base = " ".join(t[:-1]) if len(t) > 1 else t[0]
    return {"int": "int", "float": "float", "size_t": "u64", "uint64_t": "u64", "unsigned long long": "u64",
            "uint32_t": "u32", "unsigned": "u32", "unsigned int": "u32"}[base]


def _ctypes_kind(tp):
    if tp in (ctypes.c_void_p, ctypes.c_char_p) or isinstance(tp, type) and issubclass(tp, ctypes._Pointer):
        return "ptr"
    return {ctypes.c_int: "int", ctypes.c_float: "float", ctypes.c_size_t: "u64", ctypes.c_ulonglong: "u64",
            ctypes.c_uint: "u32"}[tp]


def test_binding_prototypes_match_the_header():
    """Every declaration of sparsed.h against the binding's ctypes prototype:
    the same number of parameters, each of the same kind, and the same return
    kind, so a float passed where the ABI takes an int (or a dropped argument)
    fails here rather than on a device."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    decls = re.findall(r"([A-Za-z_][\w \t\*]*?)\s*\b(sparsed_\w+)\s*\(([^;]*?)\)\s*;", text, flags=re.S)
    seen = set()
    for ret, name, params in decls:
        params = " ".join(params.split())
        c_args = [] if params in ("", "void") else [_c_kind(p) for p in params.split(",")]
        restype, argtypes = _lib.SIGNATURES[name]
        assert [_ctypes_kind(a) for a in argtypes] == c_args, name
        ret_kind = "ptr" if "*" in ret else _c_kind(ret + " r")
        assert _ctypes_kind(restype) == ret_kind, name
        seen.add(name)
    assert seen == set(_lib.SIGNATURES)

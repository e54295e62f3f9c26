"""fp64 CPU oracle of the routed MoE decode layer (ctypes binding of
liboracle.so).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg may import this package; the product path never does.
Every function cites the passage it follows in oracle.h / oracle.c.
"""
import ctypes
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
_lib = None

_EXPERT_FIELDS = ("q_gate", "q_up", "s_gate", "s_up", "q_down", "s_down")


class _Cfg(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("inter", ctypes.c_int),
                ("n_experts", ctypes.c_int), ("top_k", ctypes.c_int),
                ("n_group", ctypes.c_int), ("topk_group", ctypes.c_int),
                ("group_size", ctypes.c_int), ("rsf", ctypes.c_double)]


class _Expert(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _EXPERT_FIELDS]


def lib():
    global _lib
    if _lib is None:
        so = os.path.join(HERE, "liboracle.so")
        if not os.path.exists(so):
            from . import build as _b
            _b.build()
        L = ctypes.CDLL(so)
        p, i, d = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        L.orc_bf16_value.restype = d
        L.orc_bf16_value.argtypes = [ctypes.c_uint16]
        L.orc_f16_value.restype = d
        L.orc_f16_value.argtypes = [ctypes.c_uint16]
        L.orc_round_bf16.restype = ctypes.c_uint16
        L.orc_round_bf16.argtypes = [d]
        L.orc_set_threads.restype = i
        L.orc_set_threads.argtypes = [i]
        L.orc_router_logits.argtypes = [p, p, p, i, p]
        L.orc_select_scores.restype = i
        L.orc_select_scores.argtypes = [p, p, p, i, i, p, p, p]
        L.orc_route.restype = i
        L.orc_route.argtypes = [p, p, p, i, p, p, p, p]
        L.orc_topp.restype = i
        L.orc_topp.argtypes = [p, p, i, d, p, p, p, p]
        L.orc_gemv_int4.argtypes = [p, p, i, i, i, p, p]
        L.orc_expert_ffn.argtypes = [p, p, p, p, p]
        L.orc_experts_combine.argtypes = [p, p, p, p, i, p, p, p]
        L.orc_layer_forward.restype = i
        L.orc_layer_forward.argtypes = [p, p, p, p, p, p, i, p, p, p, p]
        L.orc_rmsnorm.argtypes = [p, i, d, p]
        L.orc_lru_sim.restype = i
        L.orc_lru_sim.argtypes = [i, i, i, i, i, p, p, p]
        L.orc_lru_sim_pinned.restype = i
        L.orc_lru_sim_pinned.argtypes = [i, i, i, i, i, p, i, p, p, p]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def cfg(shape):
    """ctypes config from any object with the layer's shape attributes."""
    return _Cfg(shape.hidden, shape.inter, shape.n_experts, shape.top_k,
                shape.n_group, shape.topk_group, shape.group_size, float(shape.rsf))


def _expert_struct(e, keep):
    arrs = []
    for n in _EXPERT_FIELDS:
        a = np.ascontiguousarray(e[n])
        keep.append(a)
        arrs.append(a.ctypes.data)
    return _Expert(*arrs)


def set_threads(n):
    return lib().orc_set_threads(int(n))


def bf16_value(b):
    return lib().orc_bf16_value(int(b))


def f16_value(h):
    return lib().orc_f16_value(int(h))


def round_bf16(v):
    return lib().orc_round_bf16(float(v))


def router_logits(shape, w_router, x_bf16):
    x = _c(np.atleast_2d(x_bf16), np.uint16)
    w = _c(w_router, np.float32)
    T = x.shape[0]
    out = np.empty((T, shape.n_experts), dtype=np.float64)
    lib().orc_router_logits(ctypes.byref(cfg(shape)), _p(w), _p(x), T, _p(out))
    return out


def select_scores(shape, s, sp, round_group_f32=False):
    s = _c(np.atleast_2d(s), np.float64)
    sp = _c(np.atleast_2d(sp), np.float64)
    T = s.shape[0]
    idx = np.empty((T, shape.top_k), dtype=np.int32)
    w = np.empty((T, shape.top_k), dtype=np.float64)
    margin = np.empty((T,), dtype=np.float64)
    rc = lib().orc_select_scores(ctypes.byref(cfg(shape)), _p(s), _p(sp), T,
                                 int(bool(round_group_f32)), _p(idx), _p(w), _p(margin))
    if rc != 0:
        raise ValueError("oracle selection rejected the configuration")
    return idx, w, margin


def route(shape, logits, bias):
    """Returns (idx [T][k] int32, w [T][k] f64, margin [T], scores [T][E])."""
    lg = _c(np.atleast_2d(logits), np.float64)
    b = _c(bias, np.float32)
    T = lg.shape[0]
    idx = np.empty((T, shape.top_k), dtype=np.int32)
    w = np.empty((T, shape.top_k), dtype=np.float64)
    margin = np.empty((T,), dtype=np.float64)
    s = np.empty_like(lg)
    rc = lib().orc_route(ctypes.byref(cfg(shape)), _p(lg), _p(b), T, _p(idx), _p(w),
                         _p(margin), _p(s))
    if rc != 0:
        raise ValueError("oracle routing rejected the configuration")
    return idx, w, margin, s


def topp(shape, s, idx, w, p):
    """Adaptive expert top-p (reading R16) on routes from route() /
    select_scores(): returns (idx, w, n_keep, margin); dropped slots are -1
    with weight 0, after the kept ids (ascending)."""
    s = _c(np.atleast_2d(s), np.float64)
    idx = np.array(np.atleast_2d(idx), dtype=np.int32, copy=True, order="C")
    w = np.array(np.atleast_2d(w), dtype=np.float64, copy=True, order="C")
    T = idx.shape[0]
    n_keep = np.empty((T,), dtype=np.int32)
    margin = np.empty((T,), dtype=np.float64)
    rc = lib().orc_topp(ctypes.byref(cfg(shape)), _p(s), T, float(p), _p(idx), _p(w),
                        _p(n_keep), _p(margin))
    if rc != 0:
        raise ValueError("oracle top-p rejected the arguments")
    return idx, w, n_keep, margin


def gemv_int4(q, s, cols, group_size, x):
    q = _c(q, np.uint8)
    s = _c(s, np.uint16)
    x = _c(x, np.float64)
    rows = q.shape[0]
    y = np.empty((rows,), dtype=np.float64)
    lib().orc_gemv_int4(_p(q), _p(s), rows, cols, group_size, _p(x), _p(y))
    return y


def expert_ffn(shape, e, x, return_h=False):
    keep = []
    es = _expert_struct(e, keep)
    x = _c(x, np.float64)
    y = np.empty((shape.hidden,), dtype=np.float64)
    h = np.empty((shape.inter,), dtype=np.float64)
    lib().orc_expert_ffn(ctypes.byref(cfg(shape)), ctypes.byref(es), _p(x), _p(y), _p(h))
    return (y, h) if return_h else y


def experts_combine(shape, experts, shared, x, idx, w):
    """experts: dict id -> expert arrays (must hold every id in idx)."""
    x = _c(np.atleast_2d(x), np.float64)
    idx = _c(np.atleast_2d(idx), np.int32)
    w = _c(np.atleast_2d(w), np.float64)
    T = x.shape[0]
    keep = []
    blank = None
    table = (_Expert * shape.n_experts)()
    for eid in range(shape.n_experts):
        if eid in experts:
            table[eid] = _expert_struct(experts[eid], keep)
        else:
            if blank is None:
                blank = _Expert()
            table[eid] = blank
    sh = _expert_struct(shared, keep) if shared is not None else None
    y = np.empty((T, shape.hidden), dtype=np.float64)
    lib().orc_experts_combine(ctypes.byref(cfg(shape)), table,
                              ctypes.byref(sh) if sh is not None else None,
                              _p(x), T, _p(idx), _p(w), _p(y))
    return y


def layer_forward(shape, w_router, bias, experts, shared, x_bf16):
    """Full layer (route + experts + combine) for T tokens.
    experts: list/dict of all n_experts experts' arrays."""
    x = _c(np.atleast_2d(x_bf16), np.uint16)
    T = x.shape[0]
    keep = []
    table = (_Expert * shape.n_experts)()
    for eid in range(shape.n_experts):
        table[eid] = _expert_struct(experts[eid], keep)
    sh = _expert_struct(shared, keep) if shared is not None else None
    wr = _c(w_router, np.float32)
    b = _c(bias, np.float32)
    y = np.empty((T, shape.hidden), dtype=np.float64)
    idx = np.empty((T, shape.top_k), dtype=np.int32)
    w = np.empty((T, shape.top_k), dtype=np.float64)
    margin = np.empty((T,), dtype=np.float64)
    rc = lib().orc_layer_forward(ctypes.byref(cfg(shape)), _p(wr), _p(b), table,
                                 ctypes.byref(sh) if sh is not None else None,
                                 _p(x), T, _p(y), _p(idx), _p(w), _p(margin))
    if rc != 0:
        raise ValueError("oracle layer rejected the configuration")
    return y, idx, w, margin


def rmsnorm(x, eps=1e-6):
    x = _c(x, np.float64)
    out = np.empty_like(x)
    lib().orc_rmsnorm(_p(x), x.size, eps, _p(out))
    return out


def lru_sim(trace, n_experts, capacity):
    """trace [T][L][k] int32 -> (hits[L], misses[L]) uint64."""
    tr = _c(trace, np.int32)
    T, L, k = tr.shape
    hits = np.zeros((L,), dtype=np.uint64)
    misses = np.zeros((L,), dtype=np.uint64)
    rc = lib().orc_lru_sim(L, n_experts, capacity, k, T, _p(tr), _p(hits), _p(misses))
    if rc != 0:
        raise ValueError("bad LRU simulation arguments")
    return hits, misses


def lru_sim_pinned(trace, n_experts, capacity, pinned):
    """trace [T][L][k] int32, pinned [L][n_pin] -> (hits[L], misses[L]):
    the LRU with each layer's pinned experts held for the whole trace."""
    tr = _c(trace, np.int32)
    T, L, k = tr.shape
    pn = _c(np.asarray(pinned).reshape(L, -1), np.int32)
    hits = np.zeros((L,), dtype=np.uint64)
    misses = np.zeros((L,), dtype=np.uint64)
    rc = lib().orc_lru_sim_pinned(L, n_experts, capacity, k, T, _p(tr), pn.shape[1], _p(pn),
                                  _p(hits), _p(misses))
    if rc != 0:
        raise ValueError("bad LRU simulation arguments")
    return hits, misses

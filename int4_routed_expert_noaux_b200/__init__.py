"""Thin Python binding of libmoe.so, the C ABI of include/moe.h (int4
routed-expert MoE decode layer for B200 / sm_100a).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch provides device memory and streams.  There is no CPU
fallback: loading fails loudly when libmoe.so is missing.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe.so")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_CUDA", 3: "MOE_ERR_OOM",
                4: "MOE_ERR_TIMEOUT", 5: "MOE_ERR_UNSUPPORTED", 6: "MOE_ERR_DEVICE"}

EXPERT_FIELDS = ("q_gate", "q_up", "s_gate", "s_up", "q_down", "s_down")


class MoeError(RuntimeError):
    def __init__(self, status, where, detail):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {detail}")


class Config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("inter", ctypes.c_int32),
                ("n_experts", ctypes.c_int32), ("n_shared", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("n_group", ctypes.c_int32),
                ("topk_group", ctypes.c_int32), ("group_size", ctypes.c_int32),
                ("routed_scaling_factor", ctypes.c_float)]

    @classmethod
    def from_shape(cls, s):
        return cls(s.hidden, s.inter, s.n_experts, s.n_shared, s.top_k, s.n_group,
                   s.topk_group, s.group_size, float(s.rsf))


class Expert(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in EXPERT_FIELDS]

    @classmethod
    def from_ptrs(cls, d):
        return cls(*[int(d[n]) for n in EXPERT_FIELDS])


_lib = None


def lib():
    """Load libmoe.so (built in-tree by build.py); raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "python -m int4_routed_expert_noaux_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        p, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        st = ctypes.c_int
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_status_string.argtypes = [st]
        L.moe_last_error.restype = ctypes.c_char_p
        L.moe_last_error.argtypes = []
        L.moe_layer_create.restype = st
        L.moe_layer_create.argtypes = [p, p, p, p, p, ctypes.POINTER(p)]
        L.moe_layer_destroy.restype = None
        L.moe_layer_destroy.argtypes = [p]
        L.moe_layer_set_top_p.restype = st
        L.moe_layer_set_top_p.argtypes = [p, ctypes.c_float]
        L.moe_layer_set_expert.restype = st
        L.moe_layer_set_expert.argtypes = [p, i, p, p]
        L.moe_workspace_bytes.restype = sz
        L.moe_workspace_bytes.argtypes = [p, i]
        L.moe_ws_check.restype = st
        L.moe_ws_check.argtypes = [p, sz, p]
        L.moe_route.restype = st
        L.moe_route.argtypes = [p, p, i, p, p, p, p, sz, p]
        L.moe_expert_ffn.restype = st
        L.moe_expert_ffn.argtypes = [p, p, i, p, p, p, p, sz, p]
        L.moe_expert_ffn_part.restype = st
        L.moe_expert_ffn_part.argtypes = [p, p, i, p, p, p, ctypes.c_uint64, i, p, sz, p]
        L.moe_layer_forward.restype = st
        L.moe_layer_forward.argtypes = [p, p, i, p, p, p, p, sz, p]
        L.moe_layer_forward_noalloc.restype = st
        L.moe_layer_forward_noalloc.argtypes = [p, p, p, p, p, p, p]
        L.moe_layer_forward_residual.restype = st
        L.moe_layer_forward_residual.argtypes = [p, p, p, p, p, p, ctypes.c_float, p, sz, p]
        L.moe_stack_forward.restype = st
        L.moe_stack_forward.argtypes = [p, i, p, p, p, p, ctypes.c_float, p, sz, p]
        L.moe_cache_create.restype = st
        L.moe_cache_create.argtypes = [p, i, i, p, ctypes.POINTER(p)]
        L.moe_cache_destroy.restype = None
        L.moe_cache_destroy.argtypes = [p]
        L.moe_cache_layer.restype = st
        L.moe_cache_layer.argtypes = [p, i, p, p, p, ctypes.POINTER(p)]
        L.moe_cache_acquire.restype = st
        L.moe_cache_acquire.argtypes = [p, i, p, i, p]
        L.moe_cache_acquire_split.restype = st
        L.moe_cache_acquire_split.argtypes = [p, i, p, i, p, p]
        L.moe_cache_wait_expert.restype = st
        L.moe_cache_wait_expert.argtypes = [p, i, i, p]
        L.moe_cache_expert_ffn.restype = st
        L.moe_cache_expert_ffn.argtypes = [p, i, p, p, p, p, p, p, sz, p, p]
        L.moe_cache_release.restype = st
        L.moe_cache_release.argtypes = [p, i, p]
        L.moe_cache_stats.restype = st
        L.moe_cache_stats.argtypes = [p, i, p, p, p]
        L.moe_cache_sync.restype = st
        L.moe_cache_sync.argtypes = [p]
        L.moe_cache_wait.restype = st
        L.moe_cache_wait.argtypes = [p, i]
        L.moe_debug_inject_fault.restype = st
        L.moe_debug_inject_fault.argtypes = [i, i]
        L.moe_lru_replay.restype = st
        L.moe_lru_replay.argtypes = [i, i, i, i, i, p, p, p]
        L.moe_lru_replay_pinned.restype = st
        L.moe_lru_replay_pinned.argtypes = [i, i, i, i, i, p, i, p, p, p]
        L.moe_cache_pin.restype = st
        L.moe_cache_pin.argtypes = [p, i, p, i, p]
        L.moe_cache_usage.restype = st
        L.moe_cache_usage.argtypes = [p, i, p]
        L.moe_debug_gemv_int4.restype = st
        L.moe_debug_gemv_int4.argtypes = [p, p, i, i, p, p, p]
        _lib = L
    return _lib


def check(status, where):
    if status != MOE_OK:
        raise MoeError(status, where, lib().moe_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def workspace_bytes(cfg, T):
    return int(lib().moe_workspace_bytes(ctypes.byref(cfg), int(T)))


def alloc_workspace(cfg, T, device="cuda"):
    """Zero-filled workspace tensor (torch allocations are 512-byte aligned)."""
    import torch
    n = workspace_bytes(cfg, T)
    if n == 0:
        raise MoeError(1, "workspace_bytes", "unsupported config or T")
    return torch.zeros(n, dtype=torch.uint8, device=device)


class Layer:
    """A layer view over caller-owned device tensors (see moe_layer_create).

    experts: list of n_experts dicts name -> device address (int) or tensor;
    shared: one such dict or None.  The tensors must outlive the Layer."""

    def __init__(self, cfg, w_router, bias, experts, shared):
        self.cfg = cfg
        arr = (Expert * cfg.n_experts)()
        for e, d in enumerate(experts):
            arr[e] = Expert.from_ptrs({k: _addr(v) for k, v in d.items()})
        sh = Expert.from_ptrs({k: _addr(v) for k, v in shared.items()}) if shared else None
        out = ctypes.c_void_p()
        check(lib().moe_layer_create(ctypes.byref(cfg), _addr(w_router), _addr(bias), arr,
                                     ctypes.byref(sh) if sh is not None else None,
                                     ctypes.byref(out)), "moe_layer_create")
        self.handle = out
        self._keep = (w_router, bias, experts, shared)

    def close(self):
        if getattr(self, "handle", None):
            lib().moe_layer_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_expert(self, e, ptrs, stream=None):
        ex = Expert.from_ptrs({k: _addr(v) for k, v in ptrs.items()})
        check(lib().moe_layer_set_expert(self.handle, int(e), ctypes.byref(ex), _stream(stream)),
              "moe_layer_set_expert")

    def set_top_p(self, p):
        """Adaptive expert top-p (moe_layer_set_top_p); p >= 1 turns it off."""
        check(lib().moe_layer_set_top_p(self.handle, float(p)), "moe_layer_set_top_p")

    def route(self, x, idx, w, ws, scores=None, stream=None):
        T = x.shape[0]
        check(lib().moe_route(self.handle, _ptr(x), T, _ptr(idx), _ptr(w), _ptr(scores),
                              _ptr(ws), ws.numel(), _stream(stream)), "moe_route")

    def expert_ffn(self, x, idx, w, y, ws, stream=None):
        T = x.shape[0]
        check(lib().moe_expert_ffn(self.handle, _ptr(x), T, _ptr(idx), _ptr(w), _ptr(y),
                                   _ptr(ws), ws.numel(), _stream(stream)), "moe_expert_ffn")

    def expert_ffn_part(self, x, idx, w, y, ws, slot_mask, combine, stream=None):
        """moe_expert_ffn for the slots in slot_mask (bit top_k: the shared
        expert); combine: write y from every slot's partial output."""
        T = x.shape[0]
        check(lib().moe_expert_ffn_part(self.handle, _ptr(x), T, _ptr(idx), _ptr(w), _ptr(y),
                                        int(slot_mask), int(bool(combine)), _ptr(ws),
                                        ws.numel(), _stream(stream)), "moe_expert_ffn_part")

    def forward(self, x, y, ws, idx=None, w=None, stream=None):
        T = x.shape[0]
        check(lib().moe_layer_forward(self.handle, _ptr(x), T, _ptr(y), _ptr(idx), _ptr(w),
                                      _ptr(ws), ws.numel(), _stream(stream)),
              "moe_layer_forward")


def forward_noalloc(layer, x, y, idx=None, w=None, status=None, stream=None):
    """Layer.forward for one token with the library's fixed scratch array
    (no workspace argument, no device allocation).  status: optional int32
    device tensor of one element that receives the device error word."""
    check(lib().moe_layer_forward_noalloc(layer.handle, _ptr(x), _ptr(y), _ptr(idx), _ptr(w),
                                          _ptr(status), _stream(stream)),
          "moe_layer_forward_noalloc")


NORM_EPS = 1e-6


def forward_residual(layer, x, x_next, ws, xn=None, idx=None, w=None, eps=NORM_EPS, stream=None):
    """x_next = x + MoE(bf16(RMSNorm(x))) for one token (fp32 [hidden] tensors)."""
    check(lib().moe_layer_forward_residual(layer.handle, _ptr(x), _ptr(x_next), _ptr(xn),
                                           _ptr(idx), _ptr(w), float(eps), _ptr(ws), ws.numel(),
                                           _stream(stream)), "moe_layer_forward_residual")


def stack_forward(layers, x_in, x_out, x_tmp, ws, idx=None, eps=NORM_EPS, stream=None):
    """Residual steps through layers[0..L-1] for one token."""
    arr = (ctypes.c_void_p * len(layers))(*[l.handle.value for l in layers])
    check(lib().moe_stack_forward(arr, len(layers), _ptr(x_in), _ptr(x_out), _ptr(x_tmp), _ptr(idx),
                                  float(eps), _ptr(ws), ws.numel(), _stream(stream)),
          "moe_stack_forward")


def lru_replay(trace, n_experts, capacity, pinned=None):
    """The cache's LRU rule on a host trace [T][L][k] -> (hits[L], misses[L]).
    pinned: optional [L][n_pinned] ascending ids pinned before the first call."""
    import numpy as np
    tr = np.ascontiguousarray(trace, dtype=np.int32)
    T, Lyr, k = tr.shape
    hits = np.zeros(Lyr, dtype=np.uint64)
    misses = np.zeros(Lyr, dtype=np.uint64)
    if pinned is None:
        check(lib().moe_lru_replay(Lyr, n_experts, capacity, k, T, tr.ctypes.data,
                                   hits.ctypes.data, misses.ctypes.data), "moe_lru_replay")
    else:
        pn = np.ascontiguousarray(pinned, dtype=np.int32).reshape(Lyr, -1)
        check(lib().moe_lru_replay_pinned(Lyr, n_experts, capacity, k, T, tr.ctypes.data,
                                          pn.shape[1], pn.ctypes.data, hits.ctypes.data,
                                          misses.ctypes.data), "moe_lru_replay_pinned")
    return hits, misses


class _LayerView:
    """A moe_layer owned by something else (a cache view)."""

    def __init__(self, handle, cfg):
        self.handle = handle
        self.cfg = cfg

    route = Layer.route
    expert_ffn = Layer.expert_ffn
    expert_ffn_part = Layer.expert_ffn_part
    forward = Layer.forward
    set_top_p = Layer.set_top_p


class Cache:
    """Per-layer LRU cache of routed experts in HBM over a pinned host store.

    host_experts: list over layers of lists over experts of dicts name ->
    pinned host address (int) or pinned tensor."""

    def __init__(self, cfg, host_experts, slots_per_layer):
        self.cfg = cfg
        n_layers = len(host_experts)
        arr = (Expert * (n_layers * cfg.n_experts))()
        for l, layer in enumerate(host_experts):
            for e, d in enumerate(layer):
                arr[l * cfg.n_experts + e] = Expert.from_ptrs({k: _addr(v) for k, v in d.items()})
        out = ctypes.c_void_p()
        check(lib().moe_cache_create(ctypes.byref(cfg), n_layers, int(slots_per_layer), arr,
                                     ctypes.byref(out)), "moe_cache_create")
        self.handle = out
        self._keep = host_experts
        self._views = {}

    def layer(self, l, w_router, bias, shared):
        if l not in self._views:
            sh = Expert.from_ptrs({k: _addr(v) for k, v in shared.items()}) if shared else None
            out = ctypes.c_void_p()
            check(lib().moe_cache_layer(self.handle, int(l), _addr(w_router), _addr(bias),
                                        ctypes.byref(sh) if sh is not None else None,
                                        ctypes.byref(out)), "moe_cache_layer")
            self._views[l] = (_LayerView(out, self.cfg), (w_router, bias, shared))
        return self._views[l][0]

    def acquire(self, l, ids, stream=None):
        import numpy as np
        a = np.ascontiguousarray(ids, dtype=np.int32)
        check(lib().moe_cache_acquire(self.handle, int(l), a.ctypes.data, a.size, _stream(stream)),
              "moe_cache_acquire")

    def acquire_split(self, l, ids, stream=None):
        """acquire without waiting for the copies: returns a bool array, True
        where ids[j] was copied (wait_expert before computing it)."""
        import numpy as np
        a = np.ascontiguousarray(ids, dtype=np.int32)
        missed = np.zeros(a.size, dtype=np.int32)
        check(lib().moe_cache_acquire_split(self.handle, int(l), a.ctypes.data, a.size,
                                            _stream(stream), missed.ctypes.data),
              "moe_cache_acquire_split")
        return missed.astype(bool)

    def wait_expert(self, l, expert, stream=None):
        check(lib().moe_cache_wait_expert(self.handle, int(l), int(expert), _stream(stream)),
              "moe_cache_wait_expert")

    def expert_ffn(self, l, x, idx, w, ids_host, y, ws, stream=None):
        """moe_cache_expert_ffn: one token of layer l through the cache, the
        resident experts first, each copied one once its copy is done.
        Returns the number of copied experts."""
        import numpy as np
        a = np.ascontiguousarray(ids_host, dtype=np.int32)
        n = ctypes.c_int()
        check(lib().moe_cache_expert_ffn(self.handle, int(l), _ptr(x), a.ctypes.data, _ptr(idx),
                                         _ptr(w), _ptr(y), _ptr(ws), ws.numel(), _stream(stream),
                                         ctypes.byref(n)), "moe_cache_expert_ffn")
        return n.value

    def pin(self, l, ids, stream=None):
        """Make ids (ascending) the pinned hot-store of layer l."""
        import numpy as np
        a = np.ascontiguousarray(ids, dtype=np.int32)
        check(lib().moe_cache_pin(self.handle, int(l), a.ctypes.data if a.size else None, a.size,
                                  _stream(stream)), "moe_cache_pin")

    def usage(self, l):
        """Usage log of layer l: uint64 [n_experts] acquire counts."""
        import numpy as np
        out = np.zeros(self.cfg.n_experts, dtype=np.uint64)
        check(lib().moe_cache_usage(self.handle, int(l), out.ctypes.data), "moe_cache_usage")
        return out

    def release(self, l, stream=None):
        check(lib().moe_cache_release(self.handle, int(l), _stream(stream)), "moe_cache_release")

    def stats(self, l):
        h, m, b = ctypes.c_uint64(), ctypes.c_uint64(), ctypes.c_uint64()
        check(lib().moe_cache_stats(self.handle, int(l), ctypes.byref(h), ctypes.byref(m),
                                    ctypes.byref(b)), "moe_cache_stats")
        return h.value, m.value, b.value

    def sync(self):
        check(lib().moe_cache_sync(self.handle), "moe_cache_sync")

    def wait(self, timeout_ms):
        """Wait at most timeout_ms for the copies (MoeError MOE_ERR_TIMEOUT
        if they are still running then)."""
        check(lib().moe_cache_wait(self.handle, int(timeout_ms)), "moe_cache_wait")

    def close(self):
        if getattr(self, "handle", None):
            lib().moe_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


FAULT_NONE, FAULT_CACHE_ALLOC, FAULT_CACHE_COPY, FAULT_CACHE_STALL = 0, 1, 2, 3


def inject_fault(kind, n=0):
    """Arm a host-side fault of the library's error paths (moe.h,
    moe_debug_inject_fault); kind FAULT_NONE disarms."""
    check(lib().moe_debug_inject_fault(int(kind), int(n)), "moe_debug_inject_fault")


def gemv_int4(q, s, rows, cols, x, y, stream=None):
    """y = dequant(q, s) @ x through the library's int4 group dot product."""
    check(lib().moe_debug_gemv_int4(_ptr(q), _ptr(s), int(rows), int(cols), _ptr(x), _ptr(y),
                                    _stream(stream)), "moe_debug_gemv_int4")


def ws_check(ws, stream=None):
    check(lib().moe_ws_check(_ptr(ws), ws.numel(), _stream(stream)), "moe_ws_check")


def _addr(v):
    if v is None:
        return None
    if isinstance(v, int):
        return v
    return v.data_ptr()

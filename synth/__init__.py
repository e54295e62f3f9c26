"""Seeded synthetic inputs for the routed-MoE layer (shared by the tests, the
benchmark, the oracle side and the CUDA side).

Holds no arithmetic of the method: only stream keys, random bits and the
input distributions of the workloads.  The host library (libsynth.so)
generates every tensor; the device library (libsynth_dev.so) generates the
large packed-int4 weight and fp16 scale tensors in place on the GPU, with
bytes identical to the host ones.

Workload shapes (the layer spec's configurations):
  TINY  hidden 256, expert inter 128, 16 routed experts + 1 shared, top_k 2,
        n_group 4, topk_group 2, routed_scaling_factor 2.5
  GLM   hidden 6144, expert inter 2048, 256 routed experts + 1 shared,
        top_k 8, n_group 8, topk_group 4, routed_scaling_factor 2.5
Distributions: int4 codes uniform over -8..7; fp16 scales U(0.005, 0.02);
router weight fp32 N(0, 0.02); correction bias fp32 U(-0.1, 0.1);
hidden states bf16 N(0, 1).  The shared expert of a layer is expert id
n_experts in the key space.
"""
import ctypes
import os
from dataclasses import dataclass, asdict

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))

T_Q_GATE, T_Q_UP, T_Q_DOWN, T_S_GATE, T_S_UP, T_S_DOWN = range(6)
T_W_ROUTER, T_BIAS, T_X, T_EPS, T_PERM, T_TRACE = range(6, 12)

SCALE_LO, SCALE_HI = 0.005, 0.02
ROUTER_SIGMA = 0.02
BIAS_LO, BIAS_HI = -0.1, 0.1
X_SIGMA = 1.0


@dataclass(frozen=True)
class Shape:
    hidden: int
    inter: int
    n_experts: int
    n_shared: int
    top_k: int
    n_group: int
    topk_group: int
    group_size: int = 32
    rsf: float = 2.5

    def as_dict(self):
        return asdict(self)

    @property
    def expert_bytes(self):
        """Bytes of one int4 expert: 3*H*I/2 codes + 3*H*I/32 fp16 scales."""
        H, I, gs = self.hidden, self.inter, self.group_size
        return 3 * H * I // 2 + 3 * H * I // gs * 2


TINY = Shape(hidden=256, inter=128, n_experts=16, n_shared=1, top_k=2,
             n_group=4, topk_group=2)
GLM = Shape(hidden=6144, inter=2048, n_experts=256, n_shared=1, top_k=8,
            n_group=8, topk_group=4)

_host = None
_dev = None


def _load_host():
    global _host
    if _host is None:
        so = os.path.join(HERE, "libsynth.so")
        if not os.path.exists(so):
            from . import build as _b
            _b.build(device=False)
        lib = ctypes.CDLL(so)
        u64, sz, dbl, p = ctypes.c_uint64, ctypes.c_size_t, ctypes.c_double, ctypes.c_void_p
        lib.synth_key_c.restype = u64
        lib.synth_key_c.argtypes = [u64, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32]
        lib.synth_draw_c.restype = u64
        lib.synth_draw_c.argtypes = [u64, u64]
        lib.synth_fill_bytes.argtypes = [u64, p, sz]
        lib.synth_fill_scales_f16.argtypes = [u64, p, sz, dbl, dbl]
        lib.synth_fill_normal_f32.argtypes = [u64, p, sz, dbl]
        lib.synth_fill_normal_bf16.argtypes = [u64, p, sz, dbl]
        lib.synth_fill_uniform_f32.argtypes = [u64, p, sz, dbl, dbl]
        lib.synth_fill_perturbed_bf16.argtypes = [u64, p, p, sz, dbl]
        lib.synth_zipf_trace.restype = ctypes.c_int
        lib.synth_zipf_trace.argtypes = [u64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, dbl, p]
        _host = lib
    return _host


def _load_dev():
    global _dev
    if _dev is None:
        so = os.path.join(HERE, "libsynth_dev.so")
        if not os.path.exists(so):
            from . import build as _b
            _b.build(device=True)
        lib = ctypes.CDLL(so)
        u64, sz, dbl, p = ctypes.c_uint64, ctypes.c_size_t, ctypes.c_double, ctypes.c_void_p
        lib.synth_dev_fill_bytes.restype = ctypes.c_int
        lib.synth_dev_fill_bytes.argtypes = [u64, p, sz, p]
        lib.synth_dev_fill_scales_f16.restype = ctypes.c_int
        lib.synth_dev_fill_scales_f16.argtypes = [u64, p, sz, dbl, dbl, p]
        _dev = lib
    return _dev


def key(seed, layer, expert, tensor):
    return int(_load_host().synth_key_c(seed, layer, expert, tensor))


def draw(k, i):
    return int(_load_host().synth_draw_c(k, i))


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


# ---- host tensors ---------------------------------------------------------

def expert_layout(shape):
    """Names, numpy dtypes and shapes of an expert's six tensors, in the
    canonical layout: q_* packed int4 rows, s_* fp16 scale rows."""
    H, I, gs = shape.hidden, shape.inter, shape.group_size
    return [
        ("q_gate", np.uint8, (I, H // 2), T_Q_GATE),
        ("q_up", np.uint8, (I, H // 2), T_Q_UP),
        ("s_gate", np.uint16, (I, H // gs), T_S_GATE),
        ("s_up", np.uint16, (I, H // gs), T_S_UP),
        ("q_down", np.uint8, (H, I // 2), T_Q_DOWN),
        ("s_down", np.uint16, (H, I // gs), T_S_DOWN),
    ]


def expert(shape, seed, layer, expert_id):
    """Host arrays of one expert (routed id < n_experts; shared = n_experts)."""
    lib = _load_host()
    out = {}
    for name, dt, shp, tag in expert_layout(shape):
        a = np.empty(shp, dtype=dt)
        k = key(seed, layer, expert_id, tag)
        if dt == np.uint8:
            lib.synth_fill_bytes(k, _ptr(a), a.size)
        else:
            lib.synth_fill_scales_f16(k, _ptr(a), a.size, SCALE_LO, SCALE_HI)
        out[name] = a
    return out


def expert_into(shape, seed, layer, expert_id, base_ptr):
    """Generate one expert (same values as expert()) into caller memory at
    base_ptr, laid out as expert_layout(shape) in order, each tensor 256-byte
    aligned; returns {name: byte offset}."""
    lib = _load_host()
    offs, off = {}, 0
    for name, dt, shp, tag in expert_layout(shape):
        n = int(np.prod(shp))
        k = key(seed, layer, expert_id, tag)
        if dt == np.uint8:
            lib.synth_fill_bytes(k, ctypes.c_void_p(base_ptr + off), n)
        else:
            lib.synth_fill_scales_f16(k, ctypes.c_void_p(base_ptr + off), n, SCALE_LO, SCALE_HI)
        offs[name] = off
        off += (n * np.dtype(dt).itemsize + 255) // 256 * 256
    return offs


def expert_stride(shape):
    """Bytes one expert takes in expert_into's layout."""
    return sum((int(np.prod(shp)) * np.dtype(dt).itemsize + 255) // 256 * 256
               for _, dt, shp, _ in expert_layout(shape))


def router(shape, seed, layer):
    """Router weight fp32 [E][H] ~ N(0, 0.02) and bias fp32 [E] ~ U(-0.1, 0.1)."""
    lib = _load_host()
    w = np.empty((shape.n_experts, shape.hidden), dtype=np.float32)
    b = np.empty((shape.n_experts,), dtype=np.float32)
    lib.synth_fill_normal_f32(key(seed, layer, 0, T_W_ROUTER), _ptr(w), w.size, ROUTER_SIGMA)
    lib.synth_fill_uniform_f32(key(seed, layer, 0, T_BIAS), _ptr(b), b.size, BIAS_LO, BIAS_HI)
    return w, b


def tokens(shape, seed, first, T, layer=0):
    """bf16 bit patterns [T][H] ~ N(0, 1); token t uses stream first + t."""
    lib = _load_host()
    x = np.empty((T, shape.hidden), dtype=np.uint16)
    for t in range(T):
        lib.synth_fill_normal_bf16(key(seed, layer, first + t, T_X), _ptr(x[t]),
                                   shape.hidden, X_SIGMA)
    return x


def correlated_tokens(shape, seed, T, c=0.05, layer=0):
    """Correlated batch: x_t = bf16(x_0 + c * eps_t), eps_t ~ N(0, 1), with
    x_0 the token of stream 0.  Routes of such tokens overlap heavily."""
    lib = _load_host()
    x0 = tokens(shape, seed, 0, 1, layer)[0]
    x = np.empty((T, shape.hidden), dtype=np.uint16)
    for t in range(T):
        lib.synth_fill_perturbed_bf16(key(seed, layer, t, T_EPS), _ptr(x0), _ptr(x[t]),
                                      shape.hidden, c)
    return x


def zipf_trace(seed, n_layers, n_experts, k, n_tokens, s=1.1):
    """[n_tokens][n_layers][k] int32 expert ids, Zipf(s) popularity over a
    seeded permutation per layer, k distinct ids per row, ascending."""
    out = np.empty((n_tokens, n_layers, k), dtype=np.int32)
    rc = _load_host().synth_zipf_trace(seed, n_layers, n_experts, k, n_tokens, s, _ptr(out))
    if rc != 0:
        raise ValueError("bad zipf trace arguments")
    return out


def bf16_to_f32(bits):
    """Value of bf16 bit patterns as float32 (bit placement only)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ---- device tensors -----------------------------------------------------------

def fill_expert_device(shape, seed, layer, expert_id, ptrs, stream=0):
    """Fill an expert's six device tensors in place.  ptrs maps the names of
    expert_layout() to device addresses (ints).  stream: a cudaStream_t as int."""
    lib = _load_dev()
    for name, dt, shp, tag in expert_layout(shape):
        n = int(np.prod(shp))
        k = key(seed, layer, expert_id, tag)
        if dt == np.uint8:
            rc = lib.synth_dev_fill_bytes(k, ptrs[name], n, stream)
        else:
            rc = lib.synth_dev_fill_scales_f16(k, ptrs[name], n, SCALE_LO, SCALE_HI, stream)
        if rc != 0:
            raise RuntimeError(f"synth device fill failed (cuda error {rc})")


def fill_bytes_device(k, ptr, n, stream=0):
    rc = _load_dev().synth_dev_fill_bytes(k, ptr, n, stream)
    if rc != 0:
        raise RuntimeError(f"synth device fill failed (cuda error {rc})")


def fill_scales_device(k, ptr, n, stream=0):
    rc = _load_dev().synth_dev_fill_scales_f16(k, ptr, n, SCALE_LO, SCALE_HI, stream)
    if rc != 0:
        raise RuntimeError(f"synth device fill failed (cuda error {rc})")

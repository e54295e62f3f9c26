"""The C-ABI library loads and exports every entry point include/moe.h
declares; host-side argument checks run without a GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

import int4_routed_expert_noaux_b200 as moe
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*(moe_[a-z0-9_]+)\s*\(",
                             text, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    lib = moe.lib()
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings_and_config_checks():
    lib = moe.lib()
    assert lib.moe_status_string(0) == b"ok"
    assert lib.moe_status_string(5) == b"unsupported shape"
    cfg = moe.Config.from_shape(synth.GLM)
    glm = moe.workspace_bytes(cfg, 1)
    assert glm > 0 and glm % 256 == 0
    assert moe.workspace_bytes(cfg, 0) == 0
    assert moe.workspace_bytes(cfg, 65) == 0
    # a workspace sized for T tokens serves every smaller call
    sizes = [moe.workspace_bytes(cfg, T) for T in range(1, 65)]
    assert all(a < b for a, b in zip(sizes, sizes[1:]))
    assert all(v % 256 == 0 for v in sizes)
    assert moe.workspace_bytes(moe.Config.from_shape(synth.TINY), 4) > 0
    bad = moe.Config.from_shape(synth.GLM)
    bad.hidden = 6000
    assert moe.workspace_bytes(bad, 1) == 0
    bad = moe.Config.from_shape(synth.GLM)
    bad.top_k = 200
    assert moe.workspace_bytes(bad, 1) == 0


def test_create_rejects_null_pointers():
    cfg = moe.Config.from_shape(synth.TINY)
    out = ctypes.c_void_p()
    rc = moe.lib().moe_layer_create(ctypes.byref(cfg), None, None, None, None, ctypes.byref(out))
    assert rc == 1
    assert b"NULL" in moe.lib().moe_last_error()
    assert not out.value



def test_stack_rejects_bad_layer_lists():
    """moe_stack_forward checks its layer list before it touches any pointer."""
    L = moe.lib()
    arr = (ctypes.c_void_p * 2)(None, None)
    assert L.moe_stack_forward(arr, 0, None, None, None, None, 1e-6, None, 0, None) == 1
    assert L.moe_stack_forward(arr, 2, None, None, None, None, 1e-6, None, 0, None) == 1
    assert b"x_tmp" in L.moe_last_error()
    assert L.moe_stack_forward(arr, 1, None, None, None, None, 1e-6, None, 0, None) == 1
    assert b"layers[0] is NULL" in L.moe_last_error()

def test_library_lru_matches_oracle_lru():
    # the cache's replacement rule (C++ in the library) against the oracle's
    # independent simulation, on Zipf traces at several capacities
    import oracle
    for seed, (L, E, k, T) in enumerate([(3, 256, 8, 300), (2, 16, 2, 200), (1, 64, 6, 500)]):
        tr = synth.zipf_trace(seed, L, E, k, T)
        for cap in sorted({k, k + 1, 2 * k, 4 * k, E // 2, E}):
            if cap < k or cap > E:
                continue
            h1, m1 = moe.lru_replay(tr, E, cap)
            h2, m2 = oracle.lru_sim(tr, E, cap)
            assert np.array_equal(h1, h2) and np.array_equal(m1, m2), (seed, cap)


def hot_set(counts, n):
    """The n most used experts (ties to the lower id), ascending."""
    order = np.lexsort((np.arange(len(counts)), -np.asarray(counts, dtype=np.int64)))
    return np.sort(order[:n])


def test_library_pinned_lru_matches_oracle():
    # the hot-store: pin the experts most used in the first half of a Zipf
    # trace, replay the whole trace in the library and in the oracle
    import oracle
    for seed, (L, E, k, T) in enumerate([(3, 256, 8, 300), (2, 16, 2, 200), (1, 64, 6, 500)]):
        tr = synth.zipf_trace(seed, L, E, k, T)
        for cap in sorted({k + 1, 2 * k, 4 * k, E // 2, E}):
            for n_pin in sorted({1, (cap - k) // 2, cap - k}):
                if n_pin < 1 or cap - n_pin < k or cap > E:
                    continue
                pinned = np.stack([hot_set(np.bincount(tr[:T // 2, l, :].ravel(), minlength=E),
                                           n_pin) for l in range(L)])
                h1, m1 = moe.lru_replay(tr, E, cap, pinned=pinned)
                h2, m2 = oracle.lru_sim_pinned(tr, E, cap, pinned)
                assert np.array_equal(h1, h2) and np.array_equal(m1, m2), (seed, cap, n_pin)


def test_pinned_lru_replay_rejects_bad_arguments():
    tr = np.array([[[0, 1]], [[1, 2]]], dtype=np.int32)
    with pytest.raises(moe.MoeError):
        moe.lru_replay(tr, 8, 3, pinned=np.array([[0, 1]]))    # 3 - 2 < k
    with pytest.raises(moe.MoeError):
        moe.lru_replay(tr, 8, 4, pinned=np.array([[1, 0]]))    # not ascending
    with pytest.raises(moe.MoeError):
        moe.lru_replay(tr, 8, 4, pinned=np.array([[0, 9]]))    # out of range


def test_lru_replay_rejects_bad_traces():
    tr = np.array([[[3, 1]]], dtype=np.int32)  # not ascending
    with pytest.raises(moe.MoeError):
        moe.lru_replay(tr, 8, 2)
    with pytest.raises(moe.MoeError):
        moe.lru_replay(np.array([[[0, 1]]], dtype=np.int32), 8, 1)  # capacity < k


def test_fault_injection_arguments():
    # the injection switch is host-only: arming, disarming and bad kinds
    # need no GPU
    with pytest.raises(moe.MoeError) as ei:
        moe.inject_fault(9, 0)
    assert ei.value.status == 1
    with pytest.raises(moe.MoeError):
        moe.inject_fault(moe.FAULT_CACHE_COPY, -1)
    moe.inject_fault(moe.FAULT_CACHE_COPY, 2)
    moe.inject_fault(moe.FAULT_NONE, 0)


def test_hot_store_hit_rate_gain_on_zipf_trace():
    # the hot-store's measured effect, on the host (the cache's own rule): a
    # learning session fills the usage log, the next session of the same
    # popularity pins the most used experts; at every size with room to pin,
    # more accesses hit than under plain LRU with the same slots
    L, E, k, T = 4, 256, 8, 512
    full = synth.zipf_trace(5, L, E, k, 2 * T)
    learn, trace = full[:T], np.ascontiguousarray(full[T:])
    usage = [np.bincount(learn[:, l].ravel(), minlength=E) for l in range(L)]
    for cap in (16, 32, 64, 128):
        h0, m0 = moe.lru_replay(trace, E, cap)
        pinned = np.stack([hot_set(usage[l], cap - k) for l in range(L)])
        h1, m1 = moe.lru_replay(trace, E, cap, pinned=pinned)
        assert int(h1.sum()) > int(h0.sum()), cap
        assert int(h1.sum() + m1.sum()) == int(h0.sum() + m0.sum()) == L * T * k

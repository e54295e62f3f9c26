"""The C-ABI library loads and exports every entry point include/moe.h
declares; host-side argument checks run without a GPU."""
import ctypes
import os
import re

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

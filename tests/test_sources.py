"""Source checks of the CUDA library (CPU only).

A kernel started as a programmatic dependent launch may be scheduled while the
kernel before it on the stream is still running; it sees that kernel's writes
only after `griddepcontrol.wait`.  So every kernel passed to `launch_pdl` must
wait before it touches memory: here, its first statement is `pdl_wait();`.
"""
import os
import re

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "int4_routed_expert_noaux_b200", "csrc")


def _sources():
    out = {}
    for fn in sorted(os.listdir(CSRC)):
        if fn.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(CSRC, fn)) as f:
                out[fn] = f.read()
    return out


def _first_statement(src, name):
    """The first statement of the body of `__global__ ... name(...)`, or None."""
    m = re.search(r"__global__[^;{]*?\b" + re.escape(name) + r"\(", src)
    if not m:
        return None
    i, depth = m.end(), 1
    while depth:
        depth += {"(": 1, ")": -1}.get(src[i], 0)
        i += 1
    body = src[src.index("{", i) + 1:]
    return body.lstrip().split(";", 1)[0].strip() + ";"


def test_dependent_launches_wait_first():
    srcs = _sources()
    launched = set()
    for text in srcs.values():
        for m in re.finditer(r"launch_pdl\(\s*([A-Za-z_]\w*)\s*[,<]", text):
            launched.add(m.group(1))
    # the batched path: router slices, selection, union kernels, tensor-core
    # scaling, packing and GEMM, and the combine
    assert len(launched) >= 9, sorted(launched)
    for name in sorted(launched):
        found = [fn for fn, text in srcs.items() if _first_statement(text, name) is not None]
        assert found, f"kernel {name} is launched with launch_pdl but not defined"
        for fn in found:
            assert _first_statement(srcs[fn], name) == "pdl_wait();", (
                f"{fn}: {name} is a dependent launch and must wait first")


def test_first_statement_parser_catches_a_missing_wait():
    src = ("__global__ void __launch_bounds__(256) k1(const int* a,\n int n) {\n"
           "  pdl_wait();\n  a[0];\n}\n"
           "__global__ void k2(int* a) {\n  a[0] = 1;\n  pdl_wait();\n}\n")
    assert _first_statement(src, "k1") == "pdl_wait();"
    assert _first_statement(src, "k2") == "a[0] = 1;"
    assert _first_statement(src, "k3") is None

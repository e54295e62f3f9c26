"""A device-side wait that runs out: the fused kernel reports MOE_ERR_TIMEOUT,
winds down, and leaves the context and the workspace usable (no fault, no
hang: every wait in the kernel has a one-second limit)."""
import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")
import int4_routed_expert_noaux_b200 as moe  # noqa: E402
from test_gpu_parity import get_layer, to_dev_bf16  # noqa: E402

pytestmark = pytest.mark.gpu

# Tiny layer (hidden 256, inter 128, top-2 + shared): a gate/up item covers
# 96 rows of inter, so each slot has 2 gate/up items: 2 shared + 2 * 2 routed
# gate/up items in all.
TINY_GATE_UP_ITEMS = 6


def test_wait_runs_out_and_reports_timeout():
    shape = synth.TINY
    dl, L = get_layer(shape)
    cfg = moe.Config.from_shape(shape)
    x = to_dev_bf16(synth.tokens(shape, 0, 11, 1))
    y_ref = torch.empty((1, shape.hidden), dtype=torch.float32, device="cuda")
    ws_ref = moe.alloc_workspace(cfg, 1)
    L.forward(x, y_ref, ws_ref)
    moe.ws_check(ws_ref)

    ws = moe.alloc_workspace(cfg, 1)
    # control word 1 offsets the first gate/up item of every CTA: past the
    # last one, the producers go on to down items whose h is never
    # published, and wait for it (a count nothing raises) until the limit
    ws[:4096].view(torch.int32)[1] = TINY_GATE_UP_ITEMS
    y = torch.zeros((1, shape.hidden), dtype=torch.float32, device="cuda")
    L.forward(x, y, ws)
    with pytest.raises(moe.MoeError) as e:
        moe.ws_check(ws)
    assert moe.STATUS_NAMES[e.value.status] == "MOE_ERR_TIMEOUT"
    words = ws[:4096].view(torch.int32).cpu().numpy()
    assert words[0] == 0  # cleared by ws_check
    assert words[1] == 0  # the offset word was reset on the way out
    # the same workspace serves the next call normally
    y2 = torch.empty_like(y_ref)
    L.forward(x, y2, ws)
    moe.ws_check(ws)
    assert torch.equal(y2, y_ref)

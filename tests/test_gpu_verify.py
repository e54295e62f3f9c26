"""Batched verify (T tokens per call, each distinct expert read once for all
its tokens) against the fp64 oracle, on a GPU."""
import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")
import int4_routed_expert_noaux_b200 as moe  # noqa: E402
from test_gpu_parity import (MEDIUM, Y_TOL, assert_y_close, check_forward, get_layer,  # noqa: E402
                             run_forward, to_dev_bf16)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T", [2, 3, 4, 8, 32])
def test_verify_parity_glm(T):
    # independent tokens: routes overlap only by chance (many distinct experts)
    dl, L = get_layer(synth.GLM)
    x_bits = synth.tokens(synth.GLM, 0, 200 + T, T)
    y, gidx, gw = run_forward(synth.GLM, L, x_bits)
    check_forward(synth.GLM, dl, x_bits, y, gidx, gw)


@pytest.mark.parametrize("T", [8, 32])
def test_verify_correlated_glm(T):
    # draft tokens close to one another: most experts serve many tokens
    dl, L = get_layer(synth.GLM)
    x_bits = synth.correlated_tokens(synth.GLM, 3, T)
    y, gidx, gw = run_forward(synth.GLM, L, x_bits)
    _, counts = np.unique(gidx, return_counts=True)
    assert counts.max() >= T // 2
    check_forward(synth.GLM, dl, x_bits, y, gidx, gw)


@pytest.mark.parametrize("shape,T", [(synth.TINY, 64), (synth.TINY, 17), (MEDIUM, 16)],
                         ids=["tiny-max", "tiny-17", "medium-16"])
def test_verify_parity_small(shape, T):
    # T = 64 is the largest batch; 17 tokens need two passes of 16 for the
    # shared expert (and usually for some routed ones)
    dl, L = get_layer(shape)
    x_bits = synth.tokens(shape, 0, 900, T)
    y, gidx, gw = run_forward(shape, L, x_bits)
    check_forward(shape, dl, x_bits, y, gidx, gw)


def test_verify_agrees_with_single_token_calls():
    shape = synth.GLM
    dl, L = get_layer(shape)
    x_bits = synth.tokens(shape, 0, 40, 4)
    yb, ib, wb = run_forward(shape, L, x_bits)
    for t in range(4):
        y1, i1, w1 = run_forward(shape, L, x_bits[t:t + 1])
        assert np.array_equal(i1[0], ib[t])
        rms = np.sqrt(np.mean(y1[0].astype(np.float64) ** 2))
        assert np.max(np.abs(y1[0] - yb[t])) <= 2 * Y_TOL * rms


@pytest.mark.parametrize("T", [0, 65])
def test_verify_rejects_batch_sizes(T):
    shape = synth.TINY
    dl, L = get_layer(shape)
    cfg = moe.Config.from_shape(shape)
    ws = moe.alloc_workspace(cfg, 64)
    x = torch.zeros((max(T, 1), shape.hidden), dtype=torch.int16, device="cuda")[:T]
    y = torch.zeros((max(T, 1), shape.hidden), dtype=torch.float32, device="cuda")
    with pytest.raises(moe.MoeError) as e:
        L.forward(x, y, ws)
    assert moe.STATUS_NAMES[e.value.status] == "MOE_ERR_INVALID_ARG"

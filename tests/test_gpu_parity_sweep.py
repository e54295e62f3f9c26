"""The one-token fused decode kernel against the fp64 oracle over the whole
benchmark workload, and on inputs that reach the method's edge cases.

- Every token the benchmark times (1000 seeded tokens) is routed through
  every one of the 8 layer copies the benchmark rotates over: 8000 routings,
  ids bit-exact against the oracle outside flagged near-ties; outputs of 32
  tokens spread over the copies against the oracle's layer.
- Exact ties (a zero router weight): every score is 1/2, every group score
  1, so the lower-index rule alone decides groups and experts.
- Crafted tied group sums and a 4-way tie at the top-k boundary.
- Tokens whose 32-input groups each span at least a 2^12 range of
  magnitudes: the int16 group format of the activations rounds the small
  inputs there.
"""
import numpy as np
import pytest

import oracle
import synth
from synth.layers import DeviceLayer

torch = pytest.importorskip("torch")
import int4_routed_expert_noaux_b200 as moe  # noqa: E402
from test_gpu_parity import (FLAG_MARGIN, assert_y_close, check_forward, get_layer,  # noqa: E402
                             kernel_precision_ids, needs_gpu, oracle_y, report_flagged,
                             to_dev_bf16)

pytestmark = pytest.mark.gpu

GLM = synth.GLM
COPIES = 8          # the benchmark's rotating layer copies
BENCH_TOKENS = 1000


def forward_one_token_each(L, x, n, shape):
    """n one-token calls (the fused kernel) on one workspace."""
    cfg = moe.Config.from_shape(shape)
    ws = moe.alloc_workspace(cfg, 1)
    y = torch.empty((n, shape.hidden), dtype=torch.float32, device="cuda")
    idx = torch.empty((n, shape.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((n, shape.top_k), dtype=torch.float32, device="cuda")
    for t in range(n):
        L.forward(x[t:t + 1], y[t:t + 1], ws, idx=idx[t:t + 1], w=w[t:t + 1])
    moe.ws_check(ws)
    return y.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()


def test_bench_workload_routing_sweep():
    needs_gpu()
    shape = GLM
    cfg = moe.Config.from_shape(shape)
    x_bits = synth.tokens(shape, 0, 0, BENCH_TOKENS)   # the benchmark's tokens
    x = to_dev_bf16(x_bits)
    flagged_total, checked_y = 0, 0
    for c in range(COPIES):
        if c == 0:
            dl, L = get_layer(shape, 0, 0)
            owned = None
        else:
            dl = DeviceLayer(shape, 0, c)
            L = moe.Layer(cfg, dl.w_router, dl.bias, dl.routed, dl.shared)
            owned = (dl, L)
        y, gidx, gw = forward_one_token_each(L, x, BENCH_TOKENS, shape)
        W, b = dl.host_router()
        lg = oracle.router_logits(shape, W, x_bits)
        oidx, ow, margin, osc = oracle.route(shape, lg, b)
        flagged = margin <= FLAG_MARGIN
        ok = ~flagged
        assert np.array_equal(gidx[ok], oidx[ok]), c
        assert np.allclose(gw[ok], ow[ok], rtol=2e-6, atol=1e-7), c
        if flagged.any():
            didx = kernel_precision_ids(shape, b, osc)
            assert np.array_equal(gidx[flagged], didx[flagged]), c
        flagged_total += int(flagged.sum())
        # outputs: 4 tokens of this copy, spread over the workload
        pick = [(c * 125 + 37 * j) % BENCH_TOKENS for j in range(4)]
        pick = [t for t in pick if ok[t]]
        assert_y_close(y[pick], oracle_y(shape, dl, x_bits[pick], oidx[pick], ow[pick]))
        checked_y += len(pick)
        if owned is not None:
            del owned, L, dl
            torch.cuda.empty_cache()
    report_flagged("bench workload, 1000 tokens x 8 layer copies", flagged_total,
                   BENCH_TOKENS * COPIES)
    assert checked_y >= 30


def custom_router_layer(dl, shape, w_router, bias):
    """The layer's experts behind another router (device copies of the given
    fp32 weight and bias)."""
    cfg = moe.Config.from_shape(shape)
    wd = torch.from_numpy(np.ascontiguousarray(w_router, dtype=np.float32)).cuda()
    bd = torch.from_numpy(np.ascontiguousarray(bias, dtype=np.float32)).cuda()
    L = moe.Layer(cfg, wd, bd, dl.routed, dl.shared)
    return L, (wd, bd)


def run_both_paths(L, shape, x_bits):
    """One-token fused calls and one batched call over the same tokens."""
    cfg = moe.Config.from_shape(shape)
    T = x_bits.shape[0]
    x = to_dev_bf16(x_bits)
    y1, i1, w1 = forward_one_token_each(L, x, T, shape)
    ws = moe.alloc_workspace(cfg, T)
    yb = torch.empty((T, shape.hidden), dtype=torch.float32, device="cuda")
    ib = torch.empty((T, shape.top_k), dtype=torch.int32, device="cuda")
    wb = torch.empty((T, shape.top_k), dtype=torch.float32, device="cuda")
    L.forward(x, yb, ws, idx=ib, w=wb)
    moe.ws_check(ws)
    return (y1, i1, w1), (yb.cpu().numpy(), ib.cpu().numpy(), wb.cpu().numpy())


def test_exact_ties_zero_router():
    # W_g = 0 and b = 0: every logit is 0, every score exactly 1/2, every
    # group score exactly 1.  Groups 0..3 are kept and experts 0..7 selected
    # by the lower-index rule alone; each weight is rsf / 8.
    dl, _ = get_layer(GLM)
    shape = GLM
    W = np.zeros((shape.n_experts, shape.hidden), dtype=np.float32)
    b = np.zeros(shape.n_experts, dtype=np.float32)
    L, keep = custom_router_layer(dl, shape, W, b)
    x_bits = synth.tokens(shape, 0, 900, 3)
    oidx, ow, margin, osc = oracle.route(shape, oracle.router_logits(shape, W, x_bits), b)
    assert np.all(osc == 0.5) and np.all(margin == 0.0)
    assert np.all(oidx == np.arange(8)[None, :])
    for y, gidx, gw in run_both_paths(L, shape, x_bits):
        assert np.all(gidx == np.arange(8)[None, :])
        assert np.all(gw == np.float32(shape.rsf / 8))
        assert_y_close(y, oracle_y(shape, dl, x_bits, oidx, ow))
    del keep


def crafted_bias(shape):
    """Bias (multiples of 2^-10, so 1/2 + b and every group sum are exact in
    fp32) with tied group scores at the topk_group boundary and a 4-way tie
    at the top-k boundary; returns the bias and the ids the rules give."""
    per = shape.n_experts // shape.n_group
    b = np.full(shape.n_experts, -100.0, dtype=np.float64)
    top = {  # group: {position in group: bias * 1024}
        0: {5: 40, 17: 30, 2: 30},   # group score 70; two 30s tie
        1: {31: 50, 0: 30},          # 80
        2: {3: 45, 4: 35, 20: 30},   # 80 (tie with group 1)
        3: {7: 60, 8: 10},           # 70: ties group 0 and 4, loses to group 0
        4: {1: 35, 2: 35},           # 70
        5: {10: 80, 9: 0, 11: 0},    # 80
        6: {0: 20, 1: 20},           # 40
        7: {0: 30, 31: 30},          # 60
    }
    for g, d in top.items():
        for pos, v in d.items():
            b[g * per + pos] = v
    # groups kept: the three at 80 (1, 2, 5) and, of the three at 70, group 0.
    # Candidates: 80, 50, 45, 40, 35, then four 30s (ids 2, 17, 32, 84) for
    # the last three places: the lower ids 2, 17, 32 win.
    expect = sorted([5 * per + 10, 1 * per + 31, 2 * per + 3, 0 * per + 5, 2 * per + 4,
                     2, 17, 32])
    return (b / 1024.0).astype(np.float32), expect


def test_crafted_tied_group_sums():
    dl, _ = get_layer(GLM)
    shape = GLM
    W = np.zeros((shape.n_experts, shape.hidden), dtype=np.float32)
    b, expect = crafted_bias(shape)
    L, keep = custom_router_layer(dl, shape, W, b)
    x_bits = synth.tokens(shape, 0, 910, 2)
    oidx, ow, margin, _ = oracle.route(shape, oracle.router_logits(shape, W, x_bits), b)
    assert np.all(oidx == np.array(expect)[None, :])
    assert np.all(margin == 0.0)
    for y, gidx, gw in run_both_paths(L, shape, x_bits):
        assert np.all(gidx == np.array(expect)[None, :])
        assert np.all(gw == np.float32(shape.rsf / 8))
        assert_y_close(y, oracle_y(shape, dl, x_bits, oidx, ow))
    del keep


def wide_range_tokens(shape, n, span_log2=13, seed=77):
    """bf16 tokens whose every 32-input group spans 2^span_log2 in magnitude:
    input j of a group has magnitude about 2^(-span_log2 * j / 31)."""
    rng = np.random.default_rng(seed)
    H = shape.hidden
    j = np.arange(H) % 32
    mag = 2.0 ** (-span_log2 * j / 31.0)
    rows = []
    for _ in range(n):
        v = rng.choice([-1.0, 1.0], size=H) * mag * rng.uniform(1.0, 2.0, size=H) * 2.0
        rows.append(np.array([oracle.round_bf16(float(a)) for a in v], dtype=np.uint16))
    return np.stack(rows)


def test_wide_dynamic_range_groups():
    dl, L = get_layer(GLM)
    shape = GLM
    x_bits = wide_range_tokens(shape, 3)
    xv = synth.bf16_to_f32(x_bits).reshape(3, -1, 32)
    ratio = np.abs(xv).max(axis=2) / np.abs(xv).min(axis=2)
    assert ratio.min() >= 2.0 ** 12
    (y1, i1, w1), (yb, ib, wb) = run_both_paths(L, shape, x_bits)
    check_forward(shape, dl, x_bits, y1, i1, w1, what="wide-range tokens, one-token kernel")
    check_forward(shape, dl, x_bits, yb, ib, wb, what="wide-range tokens, batched path")

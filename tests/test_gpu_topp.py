"""Adaptive expert top-p on the GPU against the fp64 oracle.  The page names
the option but gives no formula; the reading used: keep the fewest selected
experts, in descending weight, whose weights reach p * rsf; renormalise over
the kept ones.

A token is flagged when its noaux_tc decision margin or its top-p margin
(distance of a cumulative weight share to p at the boundary, or the share
gap between the last kept and the first dropped expert) is at most 1e-6:
the kernels decide in fp32, the oracle in fp64.  Flagged tokens are checked
for validity only (kept ids among the selected ones, weights summing to
rsf, -1 / 0 padding); every other token must match the oracle exactly in
ids and within fp32 rounding in weights, and outputs within the usual bar."""
import numpy as np
import pytest

import oracle
import synth

torch = pytest.importorskip("torch")
import int4_routed_expert_noaux_b200 as moe  # noqa: E402
from test_gpu_parity import (FLAG_MARGIN, MEDIUM, assert_y_close, get_layer, oracle_y,  # noqa: E402
                             report_flagged, to_dev_bf16)

pytestmark = pytest.mark.gpu


def oracle_topp(shape, dl, x_bits, p):
    W, b = dl.host_router()
    lg = oracle.router_logits(shape, W, x_bits)
    oidx, ow, m_sel, osc = oracle.route(shape, lg, b)
    tidx, tw, n_keep, m_p = oracle.topp(shape, osc, oidx, ow, p)
    flagged = (m_sel <= FLAG_MARGIN) | (m_p <= FLAG_MARGIN)
    return tidx, tw, n_keep, flagged, oidx


def check_topp_routes(shape, gidx, gw, tidx, tw, flagged, oidx, what):
    ok = ~flagged
    assert np.array_equal(gidx[ok], tidx[ok]), what
    assert np.allclose(gw[ok], tw[ok], rtol=2e-6, atol=1e-7), what
    for t in np.nonzero(flagged)[0]:
        kept = gidx[t][gidx[t] >= 0]
        n = len(kept)
        assert n >= 1 and np.all(gidx[t][n:] == -1) and np.all(gw[t][n:] == 0)
        assert np.all(np.diff(kept) > 0) and set(kept.tolist()) <= set(oidx[t].tolist())
        assert abs(float(gw[t][:n].sum()) - shape.rsf) <= 1e-5 * shape.rsf
    report_flagged(what, int(flagged.sum()), len(flagged))


def set_p(L, p):
    L.set_top_p(p)
    return L


@pytest.mark.parametrize("p", [0.7, 0.4])
def test_topp_route_parity_glm(p):
    shape = synth.GLM
    dl, L = get_layer(shape)
    try:
        L.set_top_p(p)
        T = 64
        x_bits = synth.tokens(shape, 0, 1200, T)
        cfg = moe.Config.from_shape(shape)
        idx = torch.empty((T, shape.top_k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, shape.top_k), dtype=torch.float32, device="cuda")
        ws = moe.alloc_workspace(cfg, T)
        L.route(to_dev_bf16(x_bits), idx, w, ws)
        moe.ws_check(ws)
        tidx, tw, n_keep, flagged, oidx = oracle_topp(shape, dl, x_bits, p)
        check_topp_routes(shape, idx.cpu().numpy(), w.cpu().numpy(), tidx, tw, flagged, oidx,
                          f"top-p {p} route, GLM x{T}")
        assert n_keep.mean() < shape.top_k
        print(f"[top-p] p={p}: mean experts kept {n_keep.mean():.2f} of {shape.top_k}")
    finally:
        L.set_top_p(1.0)


@pytest.mark.parametrize("shape,p,n", [(synth.GLM, 0.7, 24), (MEDIUM, 0.6, 12),
                                       (synth.TINY, 0.5, 24)], ids=["glm", "medium", "tiny"])
def test_topp_fused_one_token(shape, p, n):
    # one-token calls run the fused kernel: dropped slots read no bytes and
    # add nothing to y
    dl, L = get_layer(shape)
    try:
        L.set_top_p(p)
        cfg = moe.Config.from_shape(shape)
        x_bits = synth.tokens(shape, 0, 1300, n)
        x = to_dev_bf16(x_bits)
        y = torch.empty((n, shape.hidden), dtype=torch.float32, device="cuda")
        idx = torch.empty((n, shape.top_k), dtype=torch.int32, device="cuda")
        w = torch.empty((n, shape.top_k), dtype=torch.float32, device="cuda")
        ws = moe.alloc_workspace(cfg, 1)
        for t in range(n):
            L.forward(x[t:t + 1], y[t:t + 1], ws, idx=idx[t:t + 1], w=w[t:t + 1])
        moe.ws_check(ws)
        gidx, gw = idx.cpu().numpy(), w.cpu().numpy()
        tidx, tw, n_keep, flagged, oidx = oracle_topp(shape, dl, x_bits, p)
        check_topp_routes(shape, gidx, gw, tidx, tw, flagged, oidx,
                          f"top-p {p} fused, {shape.n_experts}x{n}")
        assert_y_close(y.cpu().numpy(), oracle_y(shape, dl, x_bits, gidx, gw))
        ok = ~flagged
        if ok.any():
            assert_y_close(y.cpu().numpy()[ok], oracle_y(shape, dl, x_bits[ok], tidx[ok], tw[ok]))
        # the control words are back to zero after every call
        words = ws[:4096].view(torch.int32).cpu().numpy()
        assert np.count_nonzero(np.delete(words[1:], 1)) == 0
    finally:
        L.set_top_p(1.0)


def test_topp_batched_forward_glm():
    shape = synth.GLM
    dl, L = get_layer(shape)
    try:
        L.set_top_p(0.6)
        T = 8
        cfg = moe.Config.from_shape(shape)
        x_bits = synth.tokens(shape, 0, 1400, T)
        y = torch.empty((T, shape.hidden), dtype=torch.float32, device="cuda")
        idx = torch.empty((T, shape.top_k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, shape.top_k), dtype=torch.float32, device="cuda")
        ws = moe.alloc_workspace(cfg, T)
        L.forward(to_dev_bf16(x_bits), y, ws, idx=idx, w=w)
        moe.ws_check(ws)
        gidx, gw = idx.cpu().numpy(), w.cpu().numpy()
        tidx, tw, _, flagged, oidx = oracle_topp(shape, dl, x_bits, 0.6)
        check_topp_routes(shape, gidx, gw, tidx, tw, flagged, oidx, "top-p 0.6 batched, GLM x8")
        assert_y_close(y.cpu().numpy(), oracle_y(shape, dl, x_bits, gidx, gw))
    finally:
        L.set_top_p(1.0)


def test_topp_off_is_bitwise_default():
    # p >= 1 is the default path, bit for bit
    shape = synth.GLM
    dl, L = get_layer(shape)
    cfg = moe.Config.from_shape(shape)
    x = to_dev_bf16(synth.tokens(shape, 0, 1500, 1))
    outs = []
    for p in (None, 1.0, 3.0):
        if p is not None:
            L.set_top_p(p)
        y = torch.empty((1, shape.hidden), dtype=torch.float32, device="cuda")
        ws = moe.alloc_workspace(cfg, 1)
        L.forward(x, y, ws)
        moe.ws_check(ws)
        outs.append(y)
    L.set_top_p(1.0)
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])
    with pytest.raises(moe.MoeError):
        L.set_top_p(0.0)

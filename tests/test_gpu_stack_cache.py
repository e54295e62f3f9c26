"""Stacked layers (pre-norm residual stream) and host-streamed experts, on a
GPU, against the fp64 oracle and against the resident path."""
import numpy as np
import pytest

import oracle
import synth
from synth.layers import DeviceLayer

torch = pytest.importorskip("torch")
import int4_routed_expert_noaux_b200 as moe  # noqa: E402

pytestmark = pytest.mark.gpu

Y_TOL = 2e-3
FLAG_MARGIN = 1e-5


def needs_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def bf16_round_oracle(v):
    return np.array([oracle.round_bf16(float(a)) for a in v], dtype=np.uint16)


@pytest.mark.parametrize("shape,L", [(synth.TINY, 4), (synth.GLM, 2)], ids=["tiny", "glm"])
def test_stack_teacher_forced(shape, L):
    # Each layer is checked on the GPU's own input to it (teacher forcing):
    # x_next - x must match the oracle layer applied to the bf16 normalised
    # input the kernel used, and that input must match the oracle's fp64
    # RMSNorm rounded to bf16.
    needs_gpu()
    cfg = moe.Config.from_shape(shape)
    dls = [DeviceLayer(shape, 0, l) for l in range(L)]
    views = [moe.Layer(cfg, d.w_router, d.bias, d.routed, d.shared) for d in dls]
    ws = moe.alloc_workspace(cfg, 1)
    x0 = synth.bf16_to_f32(synth.tokens(shape, 3, 0, 1)[0]).astype(np.float32)
    cur = torch.from_numpy(x0).cuda()
    xs = [x0]
    for l in range(L):
        nxt = torch.empty_like(cur)
        xn = torch.empty(shape.hidden, dtype=torch.int16, device="cuda")
        idx = torch.empty((1, shape.top_k), dtype=torch.int32, device="cuda")
        w = torch.empty((1, shape.top_k), dtype=torch.float32, device="cuda")
        moe.forward_residual(views[l], cur, nxt, ws, xn=xn, idx=idx, w=w)
        moe.ws_check(ws)
        x_l = cur.cpu().numpy().astype(np.float64)
        x_n = nxt.cpu().numpy().astype(np.float64)
        xn_g = xn.cpu().numpy().view(np.uint16)
        # the normalisation: fp64 RMSNorm rounded to bf16, within one bf16 step
        ref = bf16_round_oracle(oracle.rmsnorm(x_l, eps=moe.NORM_EPS))
        diff = np.abs(synth.bf16_to_f32(xn_g).astype(np.float64) - synth.bf16_to_f32(ref))
        ulp = np.abs(synth.bf16_to_f32(ref).astype(np.float64)) * 2.0 ** -7 + 1e-30
        assert np.all(diff <= ulp)
        assert np.mean(xn_g == ref) > 0.99
        # the layer on the kernel's own normalised input
        W, b = dls[l].host_router()
        lg = oracle.router_logits(shape, W, xn_g[None])
        oidx, ow, margin, _ = oracle.route(shape, lg, b)
        gidx = idx.cpu().numpy()
        if margin[0] > FLAG_MARGIN:
            assert np.array_equal(gidx, oidx)
        ex = {e: dls[l].host_expert(e) for e in gidx[0]}
        sh = dls[l].host_expert(shape.n_experts)
        y_ref = oracle.experts_combine(shape, ex, sh, synth.bf16_to_f32(xn_g)[None].astype(np.float64),
                                       gidx, w.cpu().numpy().astype(np.float64))[0]
        rms = np.sqrt(np.mean(y_ref ** 2))
        err = np.max(np.abs((x_n - x_l) - y_ref))
        assert err <= Y_TOL * rms + 1e-6 * np.max(np.abs(x_n)), (l, err, rms)
        xs.append(x_n.astype(np.float32))
        cur = nxt
    # the stack call gives the same bits as the sequence of steps
    x_in = torch.from_numpy(x0).cuda()
    x_out = torch.empty_like(x_in)
    x_tmp = torch.empty_like(x_in)
    idx_all = torch.empty((L, shape.top_k), dtype=torch.int32, device="cuda")
    moe.stack_forward(views, x_in, x_out, x_tmp, ws, idx=idx_all)
    moe.ws_check(ws)
    assert np.array_equal(x_out.cpu().numpy(), xs[-1])


def pinned_expert(shape, seed, layer, e):
    arrs = synth.expert(shape, seed, layer, e)
    out = {}
    for name, a in arrs.items():
        t = torch.from_numpy(a.reshape(-1).view(np.uint8).copy()).pin_memory()
        out[name] = t
    return out


@pytest.mark.parametrize("cap", [2, 5, 16], ids=["cap-k", "cap5", "cap-all"])
def test_cache_streamed_matches_resident(cap):
    needs_gpu()
    shape = synth.TINY
    L, T = 3, 30
    cfg = moe.Config.from_shape(shape)
    host = [[pinned_expert(shape, 0, l, e) for e in range(shape.n_experts)] for l in range(L)]
    dls = [DeviceLayer(shape, 0, l) for l in range(L)]
    resident = [moe.Layer(cfg, d.w_router, d.bias, d.routed, d.shared) for d in dls]
    cache = moe.Cache(cfg, host, cap)
    views = [cache.layer(l, dls[l].w_router, dls[l].bias, dls[l].shared) for l in range(L)]
    trace = synth.zipf_trace(5, L, shape.n_experts, shape.top_k, T)
    x_bits = synth.tokens(shape, 0, 50, T)
    x = torch.from_numpy(x_bits.view(np.int16)).cuda()
    wts = torch.tensor([[1.25, 1.25]], dtype=torch.float32, device="cuda")
    ws = moe.alloc_workspace(cfg, 1)
    ws2 = moe.alloc_workspace(cfg, 1)
    y_s = torch.empty((T, L, shape.hidden), dtype=torch.float32, device="cuda")
    y_r = torch.empty_like(y_s)
    for t in range(T):
        for l in range(L):
            ids = trace[t, l]
            idx = torch.from_numpy(ids.reshape(1, -1).copy()).cuda()
            cache.acquire(l, ids)
            views[l].expert_ffn(x[t:t + 1], idx, wts, y_s[t, l:l + 1], ws)
            cache.release(l)
            resident[l].expert_ffn(x[t:t + 1], idx, wts, y_r[t, l:l + 1], ws2)
    moe.ws_check(ws)
    moe.ws_check(ws2)
    cache.sync()
    assert torch.equal(y_s, y_r)
    h_ref, m_ref = oracle.lru_sim(trace, shape.n_experts, cap)
    for l in range(L):
        h, m, b = cache.stats(l)
        assert (h, m) == (int(h_ref[l]), int(m_ref[l]))
        assert b == m * shape.expert_bytes
    cache.close()

"""Stacked layers (pre-norm residual stream) and host-streamed experts, on a
GPU, against the fp64 oracle and against the resident path."""
import numpy as np
import pytest

import oracle
import synth
from synth.layers import DeviceLayer

torch = pytest.importorskip("torch")
import int4_routed_expert_noaux_b200 as moe  # noqa: E402
from test_gpu_parity import FLAG_MARGIN, Y_TOL, kernel_precision_ids, report_flagged  # noqa: E402

pytestmark = pytest.mark.gpu


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
    flagged = 0
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
        oidx, ow, margin, osc = oracle.route(shape, lg, b)
        gidx = idx.cpu().numpy()
        if margin[0] > FLAG_MARGIN:
            assert np.array_equal(gidx, oidx)
        else:
            flagged += 1
            assert np.array_equal(gidx, kernel_precision_ids(shape, b, osc))
        ex = {e: dls[l].host_expert(e) for e in gidx[0]}
        sh = dls[l].host_expert(shape.n_experts)
        y_ref = oracle.experts_combine(shape, ex, sh, synth.bf16_to_f32(xn_g)[None].astype(np.float64),
                                       gidx, w.cpu().numpy().astype(np.float64))[0]
        rms = np.sqrt(np.mean(y_ref ** 2))
        err = np.max(np.abs((x_n - x_l) - y_ref))
        assert err <= Y_TOL * rms + 1e-6 * np.max(np.abs(x_n)), (l, err, rms)
        xs.append(x_n.astype(np.float32))
        cur = nxt
    report_flagged(f"stack {shape.n_experts}x{L} layers", flagged, L)
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


# ---------------------------------------------------------------------------
# failure paths of the cache, injected on the host (no GPU work is faulted)

def tiny_cache_setup(cap, L=1):
    needs_gpu()
    shape = synth.TINY
    cfg = moe.Config.from_shape(shape)
    host = [[pinned_expert(shape, 0, l, e) for e in range(shape.n_experts)] for l in range(L)]
    dls = [DeviceLayer(shape, 0, l) for l in range(L)]
    resident = [moe.Layer(cfg, d.w_router, d.bias, d.routed, d.shared) for d in dls]
    return shape, cfg, host, dls, resident


def ffn_pair(shape, cfg, view, resident, ids, x, stream=None):
    """The routed FFN of ids through the cache view and through the
    resident layer, on the same token and weights."""
    wts = torch.tensor([[1.25, 1.25]], dtype=torch.float32, device="cuda")
    idx = torch.from_numpy(np.asarray(ids, dtype=np.int32).reshape(1, -1).copy()).cuda()
    ws, ws2 = moe.alloc_workspace(cfg, 1), moe.alloc_workspace(cfg, 1)
    y_c = torch.empty((1, shape.hidden), dtype=torch.float32, device="cuda")
    y_r = torch.empty_like(y_c)
    view.expert_ffn(x, idx, wts, y_c, ws, stream=stream)
    resident.expert_ffn(x, idx, wts, y_r, ws2, stream=stream)
    return y_c, y_r, (ws, ws2, idx, wts)


def test_cache_failed_copy_enqueue_rolls_back():
    # Two slots (= top_k).  After [1, 5] is resident, the acquire of [2, 9]
    # evicts both; its fourth copy enqueue fails (after three tensors of
    # expert 2 were enqueued into expert 1's old slot).  The call reports
    # MOE_ERR_CUDA and changes no counter; expert 1's slot no longer counts
    # as holding expert 1, so acquiring [1, 5] again reloads expert 1 (a miss)
    # and keeps expert 5 (a hit), and the output is bitwise the resident one.
    shape, cfg, host, dls, resident = tiny_cache_setup(cap=2)
    cache = moe.Cache(cfg, host, 2)
    view = cache.layer(0, dls[0].w_router, dls[0].bias, dls[0].shared)
    x = torch.from_numpy(synth.tokens(shape, 0, 60, 1).view(np.int16)).cuda()
    cache.acquire(0, [1, 5])
    y_c, y_r, keep = ffn_pair(shape, cfg, view, resident[0], [1, 5], x)
    cache.release(0)
    torch.cuda.synchronize()
    assert torch.equal(y_c, y_r)
    before = cache.stats(0)
    assert before[:2] == (0, 2)
    moe.inject_fault(moe.FAULT_CACHE_COPY, 3)
    with pytest.raises(moe.MoeError) as ei:
        cache.acquire(0, [2, 9])
    assert ei.value.status == 2
    assert cache.stats(0) == before
    cache.sync()
    cache.acquire(0, [1, 5])
    h, m, b = cache.stats(0)
    assert (h - before[0], m - before[1]) == (1, 1)
    y_c, y_r, keep = ffn_pair(shape, cfg, view, resident[0], [1, 5], x)
    cache.release(0)
    torch.cuda.synchronize()
    assert torch.equal(y_c, y_r)
    # the evicted-by-failure path leaves the cache fully usable
    cache.acquire(0, [2, 9])
    y_c, y_r, keep = ffn_pair(shape, cfg, view, resident[0], [2, 9], x)
    cache.release(0)
    torch.cuda.synchronize()
    assert torch.equal(y_c, y_r)
    cache.close()


def test_cache_failed_allocation_reports_oom():
    shape, cfg, host, dls, resident = tiny_cache_setup(cap=4)
    moe.inject_fault(moe.FAULT_CACHE_ALLOC, 0)
    with pytest.raises(moe.MoeError) as ei:
        moe.Cache(cfg, host, 4)
    assert ei.value.status == 3
    cache = moe.Cache(cfg, host, 4)   # disarmed after one failure
    cache.close()


def test_cache_wait_deadline():
    # The copy stream is held for 1.5 s (a host function): a 100 ms wait
    # returns MOE_ERR_TIMEOUT, a longer one succeeds, and the result is the
    # resident one.
    shape, cfg, host, dls, resident = tiny_cache_setup(cap=4)
    cache = moe.Cache(cfg, host, 4)
    view = cache.layer(0, dls[0].w_router, dls[0].bias, dls[0].shared)
    x = torch.from_numpy(synth.tokens(shape, 0, 61, 1).view(np.int16)).cuda()
    moe.inject_fault(moe.FAULT_CACHE_STALL, 1500)
    cache.acquire(0, [3, 4])
    with pytest.raises(moe.MoeError) as ei:
        cache.wait(100)
    assert ei.value.status == 4
    cache.wait(20000)
    y_c, y_r, keep = ffn_pair(shape, cfg, view, resident[0], [3, 4], x)
    cache.release(0)
    torch.cuda.synchronize()
    assert torch.equal(y_c, y_r)
    cache.close()


def test_cache_reacquire_without_release():
    # acquire, compute, acquire again (evicting the slots that compute reads)
    # with no release in between: the second acquire's copies wait for the
    # compute already enqueued, so both results are the resident ones.
    shape, cfg, host, dls, resident = tiny_cache_setup(cap=2)
    cache = moe.Cache(cfg, host, 2)
    view = cache.layer(0, dls[0].w_router, dls[0].bias, dls[0].shared)
    x = torch.from_numpy(synth.tokens(shape, 0, 62, 1).view(np.int16)).cuda()
    outs = []
    for ids in ([1, 5], [2, 9], [0, 15], [1, 5]):
        cache.acquire(0, ids)
        outs.append(ffn_pair(shape, cfg, view, resident[0], ids, x))
    cache.release(0)
    torch.cuda.synchronize()
    for y_c, y_r, _ in outs:
        assert torch.equal(y_c, y_r)
    cache.close()


# ---------------------------------------------------------------------------
# hot-store: pinned experts over the LRU (reading R19)

def hot_set(counts, n):
    """The n most used experts (ties to the lower id), ascending."""
    order = np.lexsort((np.arange(len(counts)), -np.asarray(counts, dtype=np.int64)))
    return np.sort(order[:n])


WIDE = synth.Shape(hidden=256, inter=128, n_experts=64, n_shared=1, top_k=2, n_group=4,
                   topk_group=2)


@pytest.mark.parametrize("shape,L,T,cap,n_pin", [(synth.TINY, 3, 40, 6, 3), (WIDE, 2, 30, 48, 40)],
                         ids=["tiny", "64-experts-40-pinned"])
def test_cache_hot_store_matches_resident_and_oracle(shape, L, T, cap, n_pin):
    # A learning pass over the first half of a Zipf trace fills the usage
    # log; a fresh cache pins each layer's most used experts, then runs the
    # whole trace.  Outputs are bitwise the resident ones, the counters are
    # the oracle's pinned LRU, and the usage log counts the trace's ids.
    # (40 pinned experts take two pointer-table updates.)
    needs_gpu()
    cfg = moe.Config.from_shape(shape)
    host = [[pinned_expert(shape, 0, l, e) for e in range(shape.n_experts)] for l in range(L)]
    dls = [DeviceLayer(shape, 0, l) for l in range(L)]
    resident = [moe.Layer(cfg, d.w_router, d.bias, d.routed, d.shared) for d in dls]
    trace = synth.zipf_trace(7, L, shape.n_experts, shape.top_k, T)
    learn = moe.Cache(cfg, host, cap)
    for l in range(L):
        learn.layer(l, dls[l].w_router, dls[l].bias, dls[l].shared)
    for t in range(T // 2):
        for l in range(L):
            learn.acquire(l, trace[t, l])
            learn.release(l)
    learn.sync()
    usage = [learn.usage(l) for l in range(L)]
    for l in range(L):
        assert np.array_equal(usage[l], np.bincount(trace[:T // 2, l].ravel(),
                                                    minlength=shape.n_experts))
    learn.close()
    pinned = np.stack([hot_set(usage[l], n_pin) for l in range(L)])

    cache = moe.Cache(cfg, host, cap)
    views = [cache.layer(l, dls[l].w_router, dls[l].bias, dls[l].shared) for l in range(L)]
    for l in range(L):
        cache.pin(l, pinned[l])
    x = torch.from_numpy(synth.tokens(shape, 0, 70, T).view(np.int16)).cuda()
    wts = torch.tensor([[1.25, 1.25]], dtype=torch.float32, device="cuda")
    ws, ws2 = moe.alloc_workspace(cfg, 1), moe.alloc_workspace(cfg, 1)
    y_s = torch.empty((T, L, shape.hidden), dtype=torch.float32, device="cuda")
    y_r = torch.empty_like(y_s)
    for t in range(T):
        for l in range(L):
            idx = torch.from_numpy(trace[t, l].reshape(1, -1).copy()).cuda()
            cache.acquire(l, trace[t, l])
            views[l].expert_ffn(x[t:t + 1], idx, wts, y_s[t, l:l + 1], ws)
            cache.release(l)
            resident[l].expert_ffn(x[t:t + 1], idx, wts, y_r[t, l:l + 1], ws2)
    moe.ws_check(ws)
    moe.ws_check(ws2)
    cache.sync()
    assert torch.equal(y_s, y_r)
    h_ref, m_ref = oracle.lru_sim_pinned(trace, shape.n_experts, cap, pinned)
    for l in range(L):
        h, m, b = cache.stats(l)
        assert (h, m) == (int(h_ref[l]), int(m_ref[l]))
        assert b == (m + n_pin) * shape.expert_bytes
        assert np.array_equal(cache.usage(l), np.bincount(trace[:, l].ravel(),
                                                          minlength=shape.n_experts))
    cache.close()


def test_cache_pin_changes_and_limits():
    # Re-pinning mid-run, unpinning, the slot limits, and a failed copy
    # during a pin (rolled back; the next acquire is bitwise correct).
    shape, cfg, host, dls, resident = tiny_cache_setup(cap=4)
    cache = moe.Cache(cfg, host, 4)
    view = cache.layer(0, dls[0].w_router, dls[0].bias, dls[0].shared)
    x = torch.from_numpy(synth.tokens(shape, 0, 63, 1).view(np.int16)).cuda()
    with pytest.raises(moe.MoeError):
        cache.pin(0, [1, 2, 3])           # 4 slots - top_k 2 = at most 2 pinned
    with pytest.raises(moe.MoeError):
        cache.pin(0, [3, 1])              # not ascending
    cache.pin(0, [3, 7])
    with pytest.raises(moe.MoeError):
        cache.acquire(0, [0, 1, 2])       # 3 ids, 2 unpinned slots
    outs = []
    for ids, pin in (([3, 9], None), ([0, 7], [0, 9]), ([4, 9], []), ([3, 5], [5, 11])):
        if pin is not None:
            cache.pin(0, pin)
        cache.acquire(0, ids)
        outs.append(ffn_pair(shape, cfg, view, resident[0], ids, x))
        cache.release(0)
    torch.cuda.synchronize()
    for y_c, y_r, _ in outs:
        assert torch.equal(y_c, y_r)
    before = cache.stats(0)
    moe.inject_fault(moe.FAULT_CACHE_COPY, 2)
    with pytest.raises(moe.MoeError) as ei:
        cache.pin(0, [12, 13])            # both missing: the third copy fails
    assert ei.value.status == 2
    assert cache.stats(0) == before
    cache.sync()
    cache.acquire(0, [12, 13])
    y_c, y_r, keep = ffn_pair(shape, cfg, view, resident[0], [12, 13], x)
    cache.release(0)
    torch.cuda.synchronize()
    assert torch.equal(y_c, y_r)
    cache.close()


# ---------------------------------------------------------------------------
# the experts of a token in several calls, and compute that waits per expert

@pytest.mark.parametrize("shape,T", [(synth.TINY, 1), (synth.TINY, 6), (synth.GLM, 1)],
                         ids=["tiny-1", "tiny-6", "glm-1"])
def test_expert_ffn_parts_match_one_call(shape, T):
    # slots computed in three calls, in a scrambled order, then combined:
    # y is bitwise that of one moe_expert_ffn call, and a call with
    # combine = 0 leaves y alone
    from test_gpu_parity import get_layer, to_dev_bf16
    dl, L = get_layer(shape)
    cfg = moe.Config.from_shape(shape)
    k = shape.top_k
    x = to_dev_bf16(synth.tokens(shape, 0, 90, T))
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    ws = moe.alloc_workspace(cfg, T)
    L.route(x, idx, w, ws)
    y_ref = torch.empty((T, shape.hidden), dtype=torch.float32, device="cuda")
    L.expert_ffn(x, idx, w, y_ref, ws)
    ws2 = moe.alloc_workspace(cfg, T)
    y = torch.full((T, shape.hidden), 7.0, dtype=torch.float32, device="cuda")
    rng = np.random.default_rng(3)
    order = rng.permutation(k + 1)          # slot k: the shared expert
    parts = np.array_split(order, 3)
    for n, part in enumerate(parts):
        mask = sum(1 << int(j) for j in part)
        L.expert_ffn_part(x, idx, w, y, ws2, mask, n == len(parts) - 1)
        if n < len(parts) - 1:
            torch.cuda.synchronize()
            assert torch.all(y == 7.0)
    moe.ws_check(ws2)
    assert torch.equal(y, y_ref)


@pytest.mark.parametrize("cap", [2, 5], ids=["cap-k", "cap5"])
def test_cache_expert_ffn_waits_per_expert(cap):
    # moe_cache_expert_ffn (hits and the shared expert first, each copied
    # expert after its own copy): bitwise the resident output, and the
    # oracle's LRU counts
    needs_gpu()
    shape = synth.TINY
    L, T = 3, 30
    cfg = moe.Config.from_shape(shape)
    host = [[pinned_expert(shape, 0, l, e) for e in range(shape.n_experts)] for l in range(L)]
    dls = [DeviceLayer(shape, 0, l) for l in range(L)]
    resident = [moe.Layer(cfg, d.w_router, d.bias, d.routed, d.shared) for d in dls]
    cache = moe.Cache(cfg, host, cap)
    for l in range(L):
        cache.layer(l, dls[l].w_router, dls[l].bias, dls[l].shared)
    trace = synth.zipf_trace(9, L, shape.n_experts, shape.top_k, T)
    x = torch.from_numpy(synth.tokens(shape, 0, 80, T).view(np.int16)).cuda()
    wts = torch.tensor([[1.25, 0.75]], dtype=torch.float32, device="cuda")
    ws, ws2 = moe.alloc_workspace(cfg, 1), moe.alloc_workspace(cfg, 1)
    y_s = torch.empty((T, L, shape.hidden), dtype=torch.float32, device="cuda")
    y_r = torch.empty_like(y_s)
    copied = 0
    for t in range(T):
        for l in range(L):
            idx = torch.from_numpy(trace[t, l].reshape(1, -1).copy()).cuda()
            copied += cache.expert_ffn(l, x[t:t + 1], idx, wts, trace[t, l], y_s[t, l:l + 1], ws)
            cache.release(l)
            resident[l].expert_ffn(x[t:t + 1], idx, wts, y_r[t, l:l + 1], ws2)
    moe.ws_check(ws)
    moe.ws_check(ws2)
    cache.sync()
    assert torch.equal(y_s, y_r)
    h_ref, m_ref = oracle.lru_sim(trace, shape.n_experts, cap)
    assert copied == int(m_ref.sum())
    for l in range(L):
        h, m, b = cache.stats(l)
        assert (h, m) == (int(h_ref[l]), int(m_ref[l]))
    absent = [e for e in range(shape.n_experts) if e not in trace[:, 0]]
    if absent:  # an expert layer 0 never loaded is not in its cache
        with pytest.raises(moe.MoeError):
            cache.wait_expert(0, absent[0])
    cache.close()


def test_cache_argument_checks():
    # every refused argument returns MOE_ERR_INVALID_ARG (status 1) before
    # anything is allocated or copied, and leaves the cache usable
    shape, cfg, host, dls, resident = tiny_cache_setup(cap=4, L=2)
    for bad_cap in (shape.top_k - 1, shape.n_experts + 1):
        with pytest.raises(moe.MoeError) as ei:
            moe.Cache(cfg, host, bad_cap)
        assert ei.value.status == 1
    pageable = [[{k: torch.from_numpy(v.numpy().copy()) for k, v in e.items()}
                 for e in layer] for layer in host]
    with pytest.raises(moe.MoeError) as ei:
        moe.Cache(cfg, pageable, 4)  # not page-locked host memory
    assert ei.value.status == 1
    cache = moe.Cache(cfg, host, 4)
    with pytest.raises(moe.MoeError):
        cache.acquire(0, [1, 5])     # no layer view yet
    view = cache.layer(0, dls[0].w_router, dls[0].bias, dls[0].shared)
    for ids in ([5, 1], [1, 1], [1, shape.n_experts], [-1, 3], [0, 1, 2, 3, 4]):
        with pytest.raises(moe.MoeError) as ei:
            cache.acquire(0, ids)
        assert ei.value.status == 1
    with pytest.raises(moe.MoeError):
        cache.acquire(2, [1, 5])     # layer out of range
    with pytest.raises(moe.MoeError):
        cache.usage(5)
    with pytest.raises(moe.MoeError):
        cache.wait(-1)
    assert cache.stats(0) == (0, 0, 0)
    # still usable
    x = torch.from_numpy(synth.tokens(shape, 0, 64, 1).view(np.int16)).cuda()
    cache.acquire(0, [1, 5])
    y_c, y_r, keep = ffn_pair(shape, cfg, view, resident[0], [1, 5], x)
    cache.release(0)
    torch.cuda.synchronize()
    assert torch.equal(y_c, y_r)
    cache.close()

"""GPU parity of the hot path against the fp64 oracle, through the C ABI.

Bars: expert ids bit-exact (ties to the lower index); weights within fp32
rounding; outputs max |dy| <= 2e-3 * rms(y_oracle) per token.

The kernels sum the router logits in fp64 (every fp32 x bf16 product is
exact in fp64) and round the sigmoid score to fp32 once, so a score differs
from the oracle's by at most 2^-25 of itself, and a decision gap (k-th vs
(k+1)-th bias-corrected score, or topk_group-th vs next group score) moves
by less than 5e-7 between the two.  A token whose fp64 decision margin is
at most FLAG_MARGIN = 1e-6 is flagged: its ids are checked against the
oracle's selection run on the GPU's own fp32 scores (the kernel's precision)
instead of the fp64 one.  Every other token must match the fp64 oracle bit
for bit.  Each test prints its flagged count and bounds it."""
import numpy as np
import pytest

import oracle
import synth
from synth.layers import DeviceLayer

torch = pytest.importorskip("torch")
import int4_routed_expert_noaux_b200 as moe  # noqa: E402

pytestmark = pytest.mark.gpu

MEDIUM = synth.Shape(hidden=3072, inter=1024, n_experts=36, n_shared=1, top_k=5, n_group=4,
                     topk_group=2)
FLAG_MARGIN = 1e-6
Y_TOL = 2e-3
SCORE_TOL = 1e-7     # fp32 rounding of an exact sigmoid: at most 2^-25 * s


def flag_bound(n):
    """Most flagged tokens allowed among n: a decision gap below 1e-6 comes
    up in well under 0.5 % of tokens at these distributions, so more means
    the margins themselves are wrong."""
    return 2 + n // 200


def report_flagged(what, flagged, n):
    print(f"[parity] {what}: {flagged} of {n} tokens flagged (fp64 margin <= {FLAG_MARGIN:g})")
    assert flagged <= flag_bound(n), (what, flagged, n)


def needs_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


_LAYERS = {}


def get_layer(shape, seed=0, layer=0):
    needs_gpu()
    key = (shape, seed, layer)
    if key not in _LAYERS:
        dl = DeviceLayer(shape, seed, layer)
        L = moe.Layer(moe.Config.from_shape(shape), dl.w_router, dl.bias, dl.routed, dl.shared)
        _LAYERS[key] = (dl, L)
    return _LAYERS[key]


def to_dev_bf16(x_bits):
    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).cuda()


def oracle_y(shape, dl, x_bits, idx, w):
    needed = sorted(set(int(e) for e in np.ravel(idx)))
    ex = {e: dl.host_expert(e) for e in needed}
    sh = dl.host_expert(shape.n_experts) if shape.n_shared else None
    xd = synth.bf16_to_f32(x_bits).astype(np.float64)
    return oracle.experts_combine(shape, ex, sh, xd, idx, np.asarray(w, dtype=np.float64))


def assert_y_close(y_gpu, y_ref):
    for t in range(y_ref.shape[0]):
        rms = np.sqrt(np.mean(y_ref[t] ** 2))
        err = np.max(np.abs(y_gpu[t].astype(np.float64) - y_ref[t]))
        assert err <= Y_TOL * rms, (t, err, rms, err / rms)


def run_route(shape, L, x_bits):
    T = x_bits.shape[0]
    cfg = moe.Config.from_shape(shape)
    x = to_dev_bf16(x_bits)
    idx = torch.empty((T, shape.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, shape.top_k), dtype=torch.float32, device="cuda")
    sc = torch.empty((T, shape.n_experts), dtype=torch.float32, device="cuda")
    ws = moe.alloc_workspace(cfg, T)
    L.route(x, idx, w, ws, scores=sc)
    moe.ws_check(ws)
    return idx.cpu().numpy(), w.cpu().numpy(), sc.cpu().numpy()


def check_route(shape, dl, x_bits, gidx, gw, gsc):
    W, b = dl.host_router()
    lg = oracle.router_logits(shape, W, x_bits)
    oidx, ow, margin, osc = oracle.route(shape, lg, b)
    # (a) sigmoid scores: the exact score rounded to fp32
    assert np.max(np.abs(gsc.astype(np.float64) - osc)) <= SCORE_TOL
    # (b) the decision in the kernel's precision: oracle selection on the
    # GPU's fp32 scores and fp32 bias-corrected scores
    sp32 = (gsc + b[None, :]).astype(np.float32)
    didx, dw, _ = oracle.select_scores(shape, gsc.astype(np.float64), sp32.astype(np.float64),
                                       round_group_f32=True)
    assert np.array_equal(gidx, didx)
    assert np.allclose(gw, dw, rtol=2e-6, atol=1e-7)
    # (c) bit-exact against the fp64 oracle where the decision is not a near tie
    ok = margin > FLAG_MARGIN
    assert np.array_equal(gidx[ok], oidx[ok])
    assert np.allclose(gw[ok], ow[ok], rtol=2e-6, atol=1e-7)
    # invariants
    per = shape.n_experts // shape.n_group
    for t in range(gidx.shape[0]):
        assert np.all(np.diff(gidx[t]) > 0)
        assert len(set((gidx[t] // per).tolist())) <= shape.topk_group
        assert abs(float(gw[t].sum()) - shape.rsf) <= 1e-5 * shape.rsf
    return int((~ok).sum())


@pytest.mark.parametrize("shape,T", [(synth.TINY, 1), (synth.TINY, 13), (MEDIUM, 7),
                                     (synth.GLM, 64)], ids=["tiny1", "tiny13", "medium7", "glm64"])
def test_route_parity(shape, T):
    dl, L = get_layer(shape)
    x_bits = synth.tokens(shape, 0, 100, T)
    gidx, gw, gsc = run_route(shape, L, x_bits)
    report_flagged(f"route {shape.n_experts}x{T}", check_route(shape, dl, x_bits, gidx, gw, gsc), T)


@pytest.mark.parametrize("shape,T", [(synth.TINY, 4), (MEDIUM, 3), (synth.GLM, 2)],
                         ids=["tiny", "medium", "glm"])
def test_expert_ffn_parity(shape, T):
    dl, L = get_layer(shape)
    cfg = moe.Config.from_shape(shape)
    x_bits = synth.tokens(shape, 0, 200, T)
    rng = np.random.default_rng(T)
    idx = np.stack([np.sort(rng.choice(shape.n_experts, shape.top_k, replace=False))
                    for _ in range(T)]).astype(np.int32)
    w = rng.uniform(0.1, 1.0, size=(T, shape.top_k)).astype(np.float32)
    y = torch.empty((T, shape.hidden), dtype=torch.float32, device="cuda")
    ws = moe.alloc_workspace(cfg, T)
    L.expert_ffn(to_dev_bf16(x_bits), torch.from_numpy(idx).cuda(), torch.from_numpy(w).cuda(),
                 y, ws)
    moe.ws_check(ws)
    assert_y_close(y.cpu().numpy(), oracle_y(shape, dl, x_bits, idx, w))


def run_forward(shape, L, x_bits):
    T = x_bits.shape[0]
    cfg = moe.Config.from_shape(shape)
    y = torch.empty((T, shape.hidden), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, shape.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, shape.top_k), dtype=torch.float32, device="cuda")
    ws = moe.alloc_workspace(cfg, T)
    L.forward(to_dev_bf16(x_bits), y, ws, idx=idx, w=w)
    moe.ws_check(ws)
    return y.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()


def kernel_precision_ids(shape, b, osc):
    """The selection as the kernels make it: the exact sigmoid scores
    rounded to fp32, the bias added in fp32, group sums in fp32."""
    s32 = osc.astype(np.float32)
    sp32 = (s32 + b[None, :].astype(np.float32)).astype(np.float32)
    didx, _, _ = oracle.select_scores(shape, s32.astype(np.float64), sp32.astype(np.float64),
                                      round_group_f32=True)
    return didx


def check_forward(shape, dl, x_bits, y, gidx, gw, what=None):
    """ids bit-exact against the fp64 oracle except flagged near-ties, whose
    ids must equal the kernel-precision selection; weights; outputs against
    the oracle's routes where they agree and against the oracle FFN on the
    GPU's routes everywhere.  Returns the flagged count."""
    W, b = dl.host_router()
    lg = oracle.router_logits(shape, W, x_bits)
    oidx, ow, margin, osc = oracle.route(shape, lg, b)
    flagged = margin <= FLAG_MARGIN
    same = np.all(gidx == oidx, axis=1)
    assert np.all(same | flagged)
    if flagged.any():
        didx = kernel_precision_ids(shape, b, osc)
        assert np.array_equal(gidx[flagged], didx[flagged])
    assert np.allclose(gw[same], ow[same], rtol=2e-6, atol=1e-7)
    if same.any():
        assert_y_close(y[same], oracle_y(shape, dl, x_bits[same], oidx[same], ow[same]))
    assert_y_close(y, oracle_y(shape, dl, x_bits, gidx, gw))
    n_flag = int(flagged.sum())
    report_flagged(what or f"forward {shape.n_experts}x{x_bits.shape[0]}", n_flag, x_bits.shape[0])
    return n_flag


@pytest.mark.parametrize("shape,T,first", [(synth.TINY, 1, 0), (synth.TINY, 1, 1),
                                           (synth.TINY, 5, 7), (MEDIUM, 1, 0), (MEDIUM, 6, 3),
                                           (synth.GLM, 1, 0), (synth.GLM, 1, 1),
                                           (synth.GLM, 3, 10)],
                         ids=["tiny-a", "tiny-b", "tiny-T5", "medium-1", "medium-T6",
                              "glm-a", "glm-b", "glm-T3"])
def test_layer_forward_parity(shape, T, first):
    dl, L = get_layer(shape)
    x_bits = synth.tokens(shape, 0, first, T)
    y, gidx, gw = run_forward(shape, L, x_bits)
    check_forward(shape, dl, x_bits, y, gidx, gw)


def test_forward_deterministic():
    dl, L = get_layer(synth.GLM)
    x_bits = synth.tokens(synth.GLM, 0, 5, 1)
    y1, i1, w1 = run_forward(synth.GLM, L, x_bits)
    y2, i2, w2 = run_forward(synth.GLM, L, x_bits)
    assert np.array_equal(y1, y2) and np.array_equal(i1, i2) and np.array_equal(w1, w2)


def test_gemv_one_hot_columns():
    needs_gpu()
    rows, cols = 64, 256
    rng = np.random.default_rng(9)
    codes = rng.integers(-8, 8, size=(rows, cols))
    u = (codes & 0xF).astype(np.uint8)
    q = (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)
    sc = rng.uniform(0.005, 0.02, size=(rows, cols // 32)).astype(np.float16)
    qd = torch.from_numpy(q).cuda()
    sd = torch.from_numpy(sc.view(np.int16)).cuda()
    y = torch.empty(rows, dtype=torch.float32, device="cuda")
    for c in range(cols):
        x = torch.zeros(cols, dtype=torch.float32, device="cuda")
        x[c] = 1.0
        moe.gemv_int4(qd, sd, rows, cols, x, y)
        expect = (codes[:, c] * sc[:, c // 32].astype(np.float64)).astype(np.float32)
        assert np.array_equal(y.cpu().numpy(), expect), c


def test_bad_expert_id_reported():
    shape = synth.TINY
    dl, L = get_layer(shape)
    cfg = moe.Config.from_shape(shape)
    x_bits = synth.tokens(shape, 0, 0, 1)
    idx = torch.tensor([[3, 99]], dtype=torch.int32, device="cuda")
    w = torch.tensor([[1.0, 1.0]], dtype=torch.float32, device="cuda")
    y = torch.empty((1, shape.hidden), dtype=torch.float32, device="cuda")
    ws = moe.alloc_workspace(cfg, 1)
    L.expert_ffn(to_dev_bf16(x_bits), idx, w, y, ws)
    with pytest.raises(moe.MoeError) as ei:
        moe.ws_check(ws)
    assert ei.value.status == 6
    moe.ws_check(ws)  # cleared


@pytest.mark.parametrize("shape,n", [(synth.TINY, 24), (MEDIUM, 8), (synth.GLM, 6)],
                         ids=["tiny", "medium", "glm"])
def test_many_decode_calls_one_workspace(shape, n):
    # back-to-back single-token calls with no host sync in between: the fused
    # kernel's control counters must come back to zero after every call
    dl, L = get_layer(shape)
    cfg = moe.Config.from_shape(shape)
    x_bits = synth.tokens(shape, 0, 300, n)
    x = to_dev_bf16(x_bits)
    ys = torch.empty((n, shape.hidden), dtype=torch.float32, device="cuda")
    idx = torch.empty((n, shape.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((n, shape.top_k), dtype=torch.float32, device="cuda")
    ws = moe.alloc_workspace(cfg, 1)
    for t in range(n):
        L.forward(x[t:t + 1], ys[t:t + 1], ws, idx=idx[t:t + 1], w=w[t:t + 1])
    moe.ws_check(ws)
    # the counters are back to zero; the epoch word counts the calls and every
    # router score record (after the 4 KB of control words) carries the last
    # call's epoch
    words = ws[:4096].view(torch.int32).cpu().numpy()
    assert words[2] == n
    assert np.count_nonzero(np.delete(words[1:], 1)) == 0
    recs = ws[4096:4096 + 8 * shape.n_experts].view(torch.int64).cpu().numpy()
    assert np.all((recs >> 32) == n)
    check_forward(shape, dl, x_bits, ys.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy())



@pytest.mark.parametrize("shape", [synth.TINY, synth.GLM], ids=["tiny", "glm"])
def test_one_token_and_batched_calls_share_a_workspace(shape):
    # A workspace sized for 4 tokens serves one-token and batched calls in
    # any order.  The batched call leaves the one-token kernel's epoch-tagged
    # score records untouched (they would otherwise hold logit bits that a
    # later epoch could match), and the one-token result stays bitwise that
    # of a fresh workspace.
    dl, L = get_layer(shape)
    cfg = moe.Config.from_shape(shape)
    x_bits = synth.tokens(shape, 0, 500, 5)
    x = to_dev_bf16(x_bits)
    dev = dict(dtype=torch.float32, device="cuda")
    y_ref = torch.empty((1, shape.hidden), **dev)
    ws_fresh = moe.alloc_workspace(cfg, 1)
    L.forward(x[0:1], y_ref, ws_fresh)
    moe.ws_check(ws_fresh)
    ws = moe.alloc_workspace(cfg, 4)
    y1, y2 = torch.empty_like(y_ref), torch.empty_like(y_ref)
    y4 = torch.empty((4, shape.hidden), **dev)
    idx4 = torch.empty((4, shape.top_k), dtype=torch.int32, device="cuda")
    w4 = torch.empty((4, shape.top_k), **dev)
    records = lambda: ws[4096:4096 + 8 * shape.n_experts].view(torch.int64).cpu().numpy()
    L.forward(x[0:1], y1, ws)
    L.forward(x[1:5], y4, ws, idx=idx4, w=w4)
    moe.ws_check(ws)
    assert np.all((records() >> 32) == 1)
    L.forward(x[0:1], y2, ws)
    moe.ws_check(ws)
    assert np.all((records() >> 32) == 2)
    assert torch.equal(y1, y_ref) and torch.equal(y2, y_ref)
    check_forward(shape, dl, x_bits[1:5], y4.cpu().numpy(), idx4.cpu().numpy(), w4.cpu().numpy())

def test_fused_decode_matches_step_kernels():
    shape = synth.GLM
    dl, L = get_layer(shape)
    cfg = moe.Config.from_shape(shape)
    x_bits = synth.tokens(shape, 0, 42, 1)
    y_f, idx, w = run_forward(shape, L, x_bits)
    y_s = torch.empty((1, shape.hidden), dtype=torch.float32, device="cuda")
    ws = moe.alloc_workspace(cfg, 1)
    L.expert_ffn(to_dev_bf16(x_bits), torch.from_numpy(idx).cuda(), torch.from_numpy(w).cuda(),
                 y_s, ws)
    moe.ws_check(ws)
    y_s = y_s.cpu().numpy()
    rms = np.sqrt(np.mean(y_s.astype(np.float64) ** 2))
    assert np.max(np.abs(y_f - y_s)) <= 1e-4 * rms

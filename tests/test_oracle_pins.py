"""Pins of the fp64 oracle against facts outside the oracle itself: closed
forms, hand-worked cases, brute force on tiny inputs, exact rational
arithmetic, library primitives, and the byte figures the pages print.

Each test names the plausible oracle mistake it would catch."""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth

HERE = os.path.dirname(os.path.abspath(__file__))


# ---------------------------------------------------------------------------
# helpers written for the tests (independent of oracle.c)

def pack_int4(codes):
    """Pack an integer matrix of codes in [-8, 7] per the format reading:
    byte j of a row holds column 2j in the low nibble, 2j+1 in the high one."""
    codes = np.asarray(codes, dtype=np.int64)
    assert codes.min() >= -8 and codes.max() <= 7
    u = (codes & 0xF).astype(np.uint8)
    return (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)


def f16_bits(values):
    return np.asarray(values, dtype=np.float16).view(np.uint16)


class Shape:
    def __init__(self, **kw):
        self.__dict__.update(kw)


# ---------------------------------------------------------------------------
# number formats

def test_f16_decode_matches_ieee_table():
    # catches: wrong exponent bias, missing subnormal branch, sign dropped
    cases = {0x3C00: 1.0, 0x0001: 2.0 ** -24, 0x03FF: 1023 * 2.0 ** -24,
             0x0400: 2.0 ** -14, 0x7BFF: 65504.0, 0xC000: -2.0,
             0x3555: 0.333251953125, 0x2E66: 0.0999755859375}
    for bits, val in cases.items():
        assert oracle.f16_value(bits) == val
    # every finite fp16 against numpy's conversion (a library primitive)
    allbits = np.arange(0, 0x10000, dtype=np.uint32).astype(np.uint16)
    vals = allbits.view(np.float16).astype(np.float64)
    finite = np.isfinite(vals)
    rng = np.random.default_rng(1)
    for b in rng.choice(allbits[finite], 4000, replace=False):
        assert oracle.f16_value(int(b)) == float(np.uint16(b).view(np.float16))


def test_bf16_decode_and_round():
    # catches: bf16 read as the low half, rounding by truncation
    assert oracle.bf16_value(0x3F80) == 1.0
    assert oracle.bf16_value(0xC040) == -3.0
    assert oracle.bf16_value(0x3E80) == 0.25
    # ties go to even: 1 + 2^-8 is halfway between 1 and 1 + 2^-7
    assert oracle.round_bf16(1.0 + 2.0 ** -8) == 0x3F80
    assert oracle.round_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82
    assert oracle.round_bf16(1.0 + 2.0 ** -8 + 2.0 ** -20) == 0x3F81
    assert oracle.round_bf16(-2.5) == 0xC020


# ---------------------------------------------------------------------------
# int4 GEMV: one-hot columns and exact rational brute force

def test_gemv_one_hot_recovers_dequantised_columns():
    # P8: x = e_c returns column c of q * scale.  Catches swapped nibbles,
    # unsigned codes, scale indexed by col % 32 or by row.
    rows, cols, gs = 5, 96, 32
    codes = ((np.arange(rows)[:, None] * 7 + np.arange(cols)[None, :] * 3) % 16) - 8
    scales = np.array([[0.5, 0.25, 2.0], [1.0, 0.125, 4.0], [3.0, 0.75, 1.5],
                       [0.0625, 8.0, 0.5], [1.25, 0.375, 6.0]], dtype=np.float64)
    q = pack_int4(codes)
    s = f16_bits(scales)
    for c in range(cols):
        x = np.zeros(cols)
        x[c] = 1.0
        y = oracle.gemv_int4(q, s, cols, gs, x)
        expect = codes[:, c] * scales[:, c // gs]
        assert np.array_equal(y, expect), c


def test_gemv_exact_rational():
    # The exact sum (fractions) is within the fp64 rounding bound.
    rng = np.random.default_rng(2)
    rows, cols, gs = 3, 128, 32
    codes = rng.integers(-8, 8, size=(rows, cols))
    scales = rng.uniform(0.005, 0.02, size=(rows, cols // gs)).astype(np.float16)
    x = rng.standard_normal(cols)
    y = oracle.gemv_int4(pack_int4(codes), scales.view(np.uint16), cols, gs, x)
    for r in range(rows):
        exact = sum(Fraction(int(codes[r, c])) * Fraction(float(scales[r, c // gs]))
                    * Fraction(float(x[c])) for c in range(cols))
        bound = 2 * cols * 2.0 ** -53 * sum(abs(codes[r, c] * float(scales[r, c // gs]) * x[c])
                                            for c in range(cols))
        assert abs(y[r] - float(exact)) <= bound


# ---------------------------------------------------------------------------
# expert FFN: closed form with integer inputs

def silu(v):
    return v / (1.0 + math.exp(-v))


def test_expert_ffn_closed_form():
    # P7: scale 1, one-hot gate/up rows, small integer x: g and u are exact
    # integers and y follows in closed form.  Catches gate/up swapped,
    # SiLU applied to up, missing down projection, transposed down.
    H, I, gs = 64, 32, 32
    sh = Shape(hidden=H, inter=I, n_experts=1, top_k=1, n_group=1, topk_group=1,
               group_size=gs, rsf=1.0)
    x = np.array([(i % 5) - 2 for i in range(H)], dtype=np.float64)
    gate_codes = np.zeros((I, H), dtype=np.int64)
    up_codes = np.zeros((I, H), dtype=np.int64)
    for i in range(I):
        gate_codes[i, (3 * i) % H] = (i % 7) - 3
        up_codes[i, (5 * i + 1) % H] = 2 - (i % 4)
    down_codes = np.zeros((H, I), dtype=np.int64)
    for r in range(H):
        down_codes[r, r % I] = 1 if r < I else -1
    ones = lambda n, m: f16_bits(np.ones((n, m // gs)))
    e = dict(q_gate=pack_int4(gate_codes), s_gate=ones(I, H),
             q_up=pack_int4(up_codes), s_up=ones(I, H),
             q_down=pack_int4(down_codes), s_down=ones(H, I))
    y, h = oracle.expert_ffn(sh, e, x, return_h=True)
    g = np.array([((i % 7) - 3) * x[(3 * i) % H] for i in range(I)])
    u = np.array([(2 - (i % 4)) * x[(5 * i + 1) % H] for i in range(I)])
    h_exp = np.array([silu(g[i]) * u[i] for i in range(I)])
    assert np.allclose(h, h_exp, rtol=1e-15, atol=0)
    y_exp = np.array([h_exp[r % I] * (1 if r < I else -1) for r in range(H)])
    assert np.allclose(y, y_exp, rtol=1e-15, atol=1e-300)



def test_expert_ffn_silu_special_values():
    # SiLU values that follow from the definition without evaluating it:
    # silu(0) = 0; sigmoid(ln 3) = 3/4, so silu(ln 3) = 0.75 ln 3; silu(42) is
    # 42 and silu(-42) is 0 to well below fp64 resolution (e^-42 < 1e-18).
    # Catches a sign flip inside the sigmoid, SiLU applied to up, or a
    # different activation (ReLU, GELU) in its place.
    H, I, gs = 32, 4, 32
    sh = Shape(hidden=H, inter=I, n_experts=1, top_k=1, n_group=1, topk_group=1,
               group_size=gs, rsf=1.0)
    x = np.zeros(H)
    x[0:4] = [0.0, math.log(3.0), 42.0, -42.0]   # gate inputs
    x[8:12] = [5.0, 2.0, 1.0, 3.0]               # up inputs
    gate_codes = np.zeros((I, H), dtype=np.int64)
    up_codes = np.zeros((I, H), dtype=np.int64)
    for i in range(I):
        gate_codes[i, i] = 1
        up_codes[i, 8 + i] = 1
    ones = lambda n, m: f16_bits(np.ones((n, m // gs)))
    e = dict(q_gate=pack_int4(gate_codes), s_gate=ones(I, H),
             q_up=pack_int4(up_codes), s_up=ones(I, H),
             q_down=pack_int4(np.zeros((H, I), dtype=np.int64)), s_down=ones(H, I))
    _, h = oracle.expert_ffn(sh, e, x, return_h=True)
    assert h[0] == 0.0
    assert abs(h[1] - 0.75 * math.log(3.0) * 2.0) <= 4e-16 * abs(h[1])
    assert h[2] == 42.0
    assert abs(h[3]) < 1e-15

# ---------------------------------------------------------------------------
# router logits

def test_router_logits_one_hot_and_exact():
    # x = e_h picks column h of W (bf16 1.0 is exact); a random case is
    # within the fp64 bound of the exact rational sum.  Catches W read
    # transposed or x read as fp16.
    sh = Shape(hidden=64, inter=32, n_experts=8, top_k=2, n_group=2, topk_group=1,
               group_size=32, rsf=2.5)
    rng = np.random.default_rng(3)
    W = rng.normal(0, 0.02, size=(8, 64)).astype(np.float32)
    for hcol in (0, 17, 63):
        x = np.zeros((1, 64), dtype=np.uint16)
        x[0, hcol] = 0x3F80
        lg = oracle.router_logits(sh, W, x)
        assert np.array_equal(lg[0], W[:, hcol].astype(np.float64))
    xb = (rng.standard_normal((1, 64)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    lg = oracle.router_logits(sh, W, xb)
    xv = synth.bf16_to_f32(xb[0]).astype(np.float64)
    for e in range(8):
        exact = sum(Fraction(float(W[e, h])) * Fraction(float(xv[h])) for h in range(64))
        assert abs(lg[0, e] - float(exact)) <= 64 * 2.0 ** -52 * float(np.abs(W[e] * xv).sum())


# ---------------------------------------------------------------------------
# selection: hand-worked cases, brute force, reductions, invariants

def test_select_hand_worked_group_rule():
    # 8 experts in 4 groups of 2, keep 2 groups, top-2 (dyadic values, so
    # every sum is exact).  Group 0 holds the single best expert but a weak
    # pair: the top-2-sum rule (R1) drops it, a top-1 rule or no group limit
    # would select expert 0.  Weights use the unbiased scores (R4).
    sh = Shape(hidden=32, inter=32, n_experts=8, top_k=2, n_group=4, topk_group=2,
               group_size=32, rsf=2.5)
    sp = np.array([[0.875, 0.0, 0.5, 0.46875, 0.4375, 0.453125, 0.125, 0.25]])
    s = np.array([[0.90, 0.05, 0.60, 0.30, 0.20, 0.40, 0.15, 0.10]])
    idx, w, margin = oracle.select_scores(sh, s, sp)
    # group sums .875 .96875 .890625 .375 -> keep g1, g2
    assert idx.tolist() == [[2, 3]]
    assert np.allclose(w, [[2.5 * 0.6 / 0.9, 2.5 * 0.3 / 0.9]], rtol=1e-15)
    # group gap .890625 - .875, expert gap .46875 - .453125
    assert margin[0] == 0.015625

    # a tie at the group boundary goes to the lower group index (R3):
    # sums .875 .9375 .875 .375 -> keep g1 and g0 (not g2)
    sp2 = np.array([[0.875, 0.0, 0.5, 0.4375, 0.5, 0.375, 0.125, 0.25]])
    idx2, _, m2 = oracle.select_scores(sh, s, sp2)
    assert idx2.tolist() == [[0, 2]]
    assert m2[0] == 0.0


def test_select_group_sum_in_fp32():
    # The kernel-precision variant (round_group_f32) forms each group score
    # as the fp32 sum of the two addends, each rounded to fp32 first: the
    # float32 arithmetic a one-warp selection does.  Two hand cases, four
    # experts in two groups of two, keep one group, top-1:
    sh = Shape(hidden=32, inter=32, n_experts=4, top_k=1, n_group=2, topk_group=1,
               group_size=32, rsf=1.0)
    f32 = lambda v: float(np.float32(v))
    # (a) the SUM is rounded: 1 + 1.5*2^-24 and 1 + 1.75*2^-24 (exact fp32
    # addends) both round to 1 + 2^-23, a tie kept by the lower group.
    # Without rounding the sum (or in fp64) group 1 wins.
    sp_a = np.array([[1.0, 1.5 * 2.0**-24, 1.0, 1.75 * 2.0**-24]])
    assert f32(1.0 + 1.5 * 2.0**-24) == f32(1.0 + 1.75 * 2.0**-24) == 1.0 + 2.0**-23
    assert oracle.select_scores(sh, sp_a, sp_a, round_group_f32=True)[0].tolist() == [[0]]
    assert oracle.select_scores(sh, sp_a, sp_a)[0].tolist() == [[2]]
    # (b) each ADDEND is rounded first: 2^-24 + 2^-50 rounds to 2^-24, and
    # 1 + 2^-24 is a tie between fp32 neighbours that goes to even (1.0),
    # below group 1's exact 1 + 2^-23.  Rounding only the exact sum would
    # give 1 + 2^-23 for group 0 too, a tie won by group 0.
    sp_b = np.array([[1.0, 2.0**-24 + 2.0**-50, 1.0, 2.0**-23]])
    assert f32(2.0**-24 + 2.0**-50) == 2.0**-24
    assert f32(1.0 + 2.0**-24) == 1.0
    assert f32(1.0 + 2.0**-24 + 2.0**-50) == 1.0 + 2.0**-23
    assert oracle.select_scores(sh, sp_b, sp_b, round_group_f32=True)[0].tolist() == [[2]]
    assert oracle.select_scores(sh, sp_b, sp_b)[0].tolist() == [[2]]
    # So a variant that skips the sum's rounding (or rounds nothing) fails
    # (a), and one that rounds only the exact sum fails (b).


def test_topp_hand_cases():
    # R16: keep the fewest selected experts, taken in descending weight
    # (ties: the lower id first), whose weights reach p * rsf; the kept
    # weights are normalised again over the kept experts.
    sh = Shape(hidden=32, inter=32, n_experts=16, top_k=4, n_group=1, topk_group=1,
               group_size=32, rsf=2.0)
    s = np.zeros(16)
    s[[3, 7, 9, 12]] = [0.8, 0.4, 0.2, 0.2]          # shares .5 .25 .125 .125
    idx, w, _ = oracle.select_scores(sh, s[None], s[None])
    # p = 0.7: .5 < .7 <= .75, so the two heaviest, weights 2 * (.8, .4) / 1.2
    i2, w2, n2, m2 = oracle.topp(sh, s[None], idx, w, 0.7)
    assert i2.tolist() == [[3, 7, -1, -1]] and n2.tolist() == [2]
    assert np.allclose(w2, [[4 / 3, 2 / 3, 0.0, 0.0]], rtol=1e-15, atol=0)
    assert m2[0] == pytest.approx(0.05, abs=1e-15)
    # p reached exactly (.75): two kept, boundary margin 0 (flagged)
    _, _, n3, m3 = oracle.topp(sh, s[None], idx, w, 0.75)
    assert n3.tolist() == [2] and m3[0] == 0.0
    # p = 1 keeps every selected expert with its weight
    i4, w4, n4, m4 = oracle.topp(sh, s[None], idx, w, 1.0)
    assert i4.tolist() == idx.tolist() and np.array_equal(w4, w) and n4[0] == 4
    assert m4[0] == np.inf
    # a tiny p keeps only the heaviest, at weight rsf
    i5, w5, n5, _ = oracle.topp(sh, s[None], idx, w, 1e-9)
    assert i5.tolist() == [[3, -1, -1, -1]] and w5[0, 0] == pytest.approx(2.0, rel=1e-15)
    # equal weights across the boundary: the lower ids are kept, margin 0
    s2 = np.zeros(16)
    s2[[2, 5, 8, 11]] = 0.5
    idx2, wq, _ = oracle.select_scores(sh, s2[None], s2[None])
    i6, w6, n6, m6 = oracle.topp(sh, s2[None], idx2, wq, 0.6)
    assert i6.tolist() == [[2, 5, 8, -1]] and n6[0] == 3 and m6[0] == 0.0
    assert np.allclose(w6[0, :3], 2 / 3, rtol=1e-15, atol=0)


def test_topp_brute_force():
    # Independently of the prefix scan: the kept set is the smallest subset
    # of the selected experts whose weights reach p * rsf, and of the subsets
    # of that size the heaviest.  Trials whose decision is within 1e-9 of a
    # tie are skipped (the two formulations may then differ in rounding).
    sh = Shape(hidden=32, inter=32, n_experts=16, top_k=4, n_group=4, topk_group=2,
               group_size=32, rsf=2.5)
    rng = np.random.default_rng(21)
    checked = 0
    for _ in range(400):
        s = 1 / (1 + np.exp(-rng.normal(0, 1.5, size=16)))
        sp = s + rng.uniform(-0.1, 0.1, size=16)
        p = float(rng.uniform(0.05, 0.999))
        idx, w, _ = oracle.select_scores(sh, s[None], sp[None])
        i2, w2, n, m = oracle.topp(sh, s[None], idx, w, p)
        if m[0] < 1e-9:
            continue
        sel = idx[0].tolist()
        share = {e: s[e] / sum(s[x] for x in sel) for e in sel}
        best = None
        for r in range(1, 5):
            cands = [c for c in itertools.combinations(sel, r) if sum(share[e] for e in c) >= p]
            if cands:
                best = max(cands, key=lambda c: sum(share[e] for e in c))
                break
        assert sorted(best) == [e for e in i2[0].tolist() if e >= 0]
        assert n[0] == len(best)
        kept = sorted(best)
        assert np.allclose(w2[0, :len(kept)], [2.5 * s[e] / sum(s[x] for x in kept) for e in kept],
                           rtol=1e-14)
        assert np.all(i2[0, len(kept):] == -1) and np.all(w2[0, len(kept):] == 0)
        checked += 1
    assert checked > 300


def test_combine_skips_dropped_slots():
    # an id of -1 (a slot dropped by top-p) contributes nothing
    sh = synth.TINY
    rng = np.random.default_rng(8)
    ex = {e: synth.expert(sh, 0, 0, e) for e in (3, 9)}
    x = rng.normal(size=(1, sh.hidden))
    y_one = oracle.experts_combine(sh, ex, None, x, np.array([[3, -1]], dtype=np.int32),
                                   np.array([[1.5, 0.0]]))
    y_ref = oracle.experts_combine(sh, ex, None, x, np.array([[3, 9]], dtype=np.int32),
                                   np.array([[1.5, 0.0]]))
    assert np.array_equal(y_one, y_ref)


def test_select_ties_lower_index():
    sh = Shape(hidden=32, inter=32, n_experts=8, top_k=3, n_group=1, topk_group=1,
               group_size=32, rsf=1.0)
    sp = np.array([[0.3, 0.5, 0.5, 0.2, 0.5, 0.5, 0.1, 0.0]])
    idx, w, margin = oracle.select_scores(sh, sp, sp)
    assert idx.tolist() == [[1, 2, 4]]
    assert margin[0] == 0.0


def brute_force_route(sh, s, sp):
    """Independent enumeration for one token (reading R1-R4): rank groups by
    the top-2 sum (ties: lower group), then among all k-subsets of the kept
    groups' experts pick the one whose sorted score vector is largest, ties
    to the lexicographically smallest id tuple."""
    E, G, TG, k = sh.n_experts, sh.n_group, sh.topk_group, sh.top_k
    per = E // G
    gsum = [sum(sorted(sp[g * per:(g + 1) * per], reverse=True)[:2]) for g in range(G)]
    order = sorted(range(G), key=lambda g: (-gsum[g], g))
    kept = set(order[:TG])
    cand = [e for e in range(E) if e // per in kept]
    best = None
    for sub in itertools.combinations(cand, k):
        keyv = tuple(sorted(((-sp[e], e) for e in sub)))
        if best is None or keyv < best[0]:
            best = (keyv, sub)
    sel = sorted(best[1])
    tot = sum(s[e] for e in sel) + 1e-20
    return sel, [sh.rsf * s[e] / tot for e in sel]


def test_select_brute_force_tiny():
    # P6: every token of random tiny inputs, plus coarse-valued inputs that
    # force many ties.
    sh = synth.TINY
    rng = np.random.default_rng(4)
    for trial in range(300):
        if trial % 2:
            logits = rng.normal(0, 1.5, size=16)
            bias = rng.uniform(-0.1, 0.1, size=16)
            s = 1 / (1 + np.exp(-logits))
            sp = s + bias
        else:
            s = rng.integers(1, 5, size=16) / 4.0
            sp = s + rng.integers(-1, 2, size=16) / 8.0
        idx, w, _ = oracle.select_scores(sh, s[None], sp[None])
        sel, wexp = brute_force_route(sh, s, sp)
        assert idx[0].tolist() == sel
        assert np.allclose(w[0], wexp, rtol=1e-14)


def test_select_reduces_to_plain_topk():
    # P7: one group, keep it, bias 0: the selection is the top-k of the
    # logits (sigmoid is monotone), ties to the lower index = numpy stable
    # argsort of the negated logits.
    sh = Shape(hidden=32, inter=32, n_experts=64, top_k=6, n_group=1, topk_group=1,
               group_size=32, rsf=2.5)
    rng = np.random.default_rng(5)
    logits = np.round(rng.normal(0, 1, size=(50, 64)), 1)   # many ties
    idx, w, _, s = oracle.route(sh, logits, np.zeros(64, dtype=np.float32))
    for t in range(50):
        ref = np.sort(np.argsort(-logits[t], kind="stable")[:6])
        assert idx[t].tolist() == ref.tolist()
        st = 1 / (1 + np.exp(-logits[t][ref]))
        assert np.allclose(w[t], 2.5 * st / st.sum(), rtol=1e-14)


@pytest.mark.parametrize("shape", [synth.TINY, synth.GLM], ids=["tiny", "glm"])
def test_route_invariants(shape):
    # P5: k distinct ascending ids, from at most topk_group groups,
    # weights positive and summing to rsf.
    w_r, b = synth.router(shape, 0, 0)
    x = synth.tokens(shape, 0, 0, 64)
    lg = oracle.router_logits(shape, w_r, x)
    idx, w, margin, s = oracle.route(shape, lg, b)
    per = shape.n_experts // shape.n_group
    for t in range(64):
        ids = idx[t]
        assert len(set(ids.tolist())) == shape.top_k
        assert np.all(np.diff(ids) > 0)
        assert ids.min() >= 0 and ids.max() < shape.n_experts
        assert len(set((ids // per).tolist())) <= shape.topk_group
        assert np.all(w[t] > 0)
        assert abs(w[t].sum() - shape.rsf) <= 1e-12
        assert margin[t] >= 0


def test_route_bias_only_steers_selection():
    # R4: a bias that changes nothing about the order leaves weights equal
    # to the unbiased normalised scores; a large bias on one expert forces
    # it in but its weight still uses its own unbiased score.
    sh = Shape(hidden=32, inter=32, n_experts=8, top_k=2, n_group=1, topk_group=1,
               group_size=32, rsf=2.0)
    logits = np.array([[2.0, 1.0, 0.0, -1.0, -2.0, -3.0, -4.0, -5.0]])
    bias = np.zeros(8, dtype=np.float32)
    bias[7] = 10.0
    idx, w, _, s = oracle.route(sh, logits, bias)
    assert idx.tolist() == [[0, 7]]
    s0, s7 = 1 / (1 + math.exp(-2.0)), 1 / (1 + math.exp(5.0))
    assert np.allclose(w[0], [2.0 * s0 / (s0 + s7), 2.0 * s7 / (s0 + s7)], rtol=1e-14)



def test_route_sigmoid_scores_closed_form():
    # The score is the logistic sigmoid of the logit: at 0, +-ln 3, ln 7,
    # ln 15 and -ln 7 it takes the values 1/2, 3/4, 1/4, 7/8, 15/16, 1/8; at
    # +-40 it is 1 and e^-40 to fp64 resolution.  Weights of the two winners
    # (scores 1 and 15/16, rsf 2) are 32/31 and 30/31.  Catches softmax in
    # place of the sigmoid, a sign flip, or weights from the biased scores.
    sh = Shape(hidden=32, inter=32, n_experts=8, top_k=2, n_group=1, topk_group=1,
               group_size=32, rsf=2.0)
    ln = math.log
    logits = np.array([[0.0, ln(3.0), -ln(3.0), ln(7.0), 40.0, -40.0, -ln(7.0), ln(15.0)]])
    idx, w, _, s = oracle.route(sh, logits, np.zeros(8, dtype=np.float32))
    want = [0.5, 0.75, 0.25, 0.875, 1.0, math.exp(-40.0), 0.125, 0.9375]
    assert np.allclose(s[0], want, rtol=1e-15, atol=0)
    assert idx.tolist() == [[4, 7]]
    assert np.allclose(w[0], [32 / 31, 30 / 31], rtol=1e-15, atol=0)

# ---------------------------------------------------------------------------
# combine: linearity and the single-expert case (P9)

def test_combine_linearity_and_single_expert():
    sh = synth.TINY
    ex = {e: synth.expert(sh, 7, 0, e) for e in range(sh.n_experts)}
    shared = synth.expert(sh, 7, 0, sh.n_experts)
    x = synth.bf16_to_f32(synth.tokens(sh, 7, 0, 3)).astype(np.float64)
    idx = np.array([[1, 5], [0, 15], [3, 4]], dtype=np.int32)
    w = np.array([[0.7, 1.8], [1.0, 1.5], [2.0, 0.5]])
    y = oracle.experts_combine(sh, ex, shared, x, idx, w)
    y0 = oracle.experts_combine(sh, ex, None, x, idx, w)
    y2 = oracle.experts_combine(sh, ex, None, x, idx, 2 * w)
    assert np.allclose(y2, 2 * y0, rtol=1e-13, atol=1e-12)
    ysh = np.stack([oracle.expert_ffn(sh, shared, x[t]) for t in range(3)])
    assert np.allclose(y, y0 + ysh, rtol=1e-13, atol=1e-12)
    # single expert with weight 1 (other weight 0) is that expert's FFN
    w1 = np.array([[1.0, 0.0]] * 3)
    y1 = oracle.experts_combine(sh, ex, None, x, idx, w1)
    for t in range(3):
        assert np.allclose(y1[t], oracle.expert_ffn(sh, ex[int(idx[t, 0])], x[t]),
                           rtol=1e-14, atol=1e-13)
    # permuting tokens permutes outputs
    perm = [2, 0, 1]
    yp = oracle.experts_combine(sh, ex, shared, x[perm], idx[perm], w[perm])
    assert np.array_equal(yp, y[perm])


def test_layer_forward_is_route_then_combine():
    sh = synth.TINY
    w_r, b = synth.router(sh, 0, 0)
    ex = [synth.expert(sh, 0, 0, e) for e in range(sh.n_experts)]
    shared = synth.expert(sh, 0, 0, sh.n_experts)
    x = synth.tokens(sh, 0, 0, 4)
    y, idx, w, margin = oracle.layer_forward(sh, w_r, b, ex, shared, x)
    lg = oracle.router_logits(sh, w_r, x)
    idx2, w2, _, _ = oracle.route(sh, lg, b)
    assert np.array_equal(idx, idx2) and np.array_equal(w, w2)
    yc = oracle.experts_combine(sh, dict(enumerate(ex)), shared,
                                synth.bf16_to_f32(x).astype(np.float64), idx, w)
    assert np.array_equal(y, yc)


# ---------------------------------------------------------------------------
# RMSNorm (reading R9)

def test_rmsnorm_closed_form():
    x = np.full(16, -3.0)
    out = oracle.rmsnorm(x, eps=0.0)
    assert np.allclose(out, -1.0, rtol=1e-15)
    x = np.array([3.0, 4.0])            # mean square 12.5
    out = oracle.rmsnorm(x, eps=1e-6)
    assert np.allclose(out, x / math.sqrt(12.5 + 1e-6), rtol=1e-15)


# ---------------------------------------------------------------------------
# LRU simulation (reading R11)

def test_lru_hand_worked():
    # capacity 3, k 2, one layer.  Tokens: {0,1} {1,2} {0,3} {2,3} {1,3}
    # t0: miss 0 (slot a), miss 1 (slot b)            h0 m2
    # t1: hit 1; miss 2 -> empty slot c               h1 m1  [0:t0 1:t1 2:t1]
    # t2: miss 0? 0 still cached -> hit; miss 3 evicts LRU among {1,2}=1
    #     stamps: 0@t0(1) 1@t1(3) 2@t1(4) -> 0 touched (5); LRU of {1,2} is 1
    #                                                  h1 m1  cache {0,3,2}
    # t3: hit 2, hit 3                                 h2 m0
    # t4: hit 3; miss 1 evicts LRU not in {1,3}: 0@5 vs 2@(t3) -> 0
    trace = np.array([[[0, 1]], [[1, 2]], [[0, 3]], [[2, 3]], [[1, 3]]], dtype=np.int32)
    hits, misses = oracle.lru_sim(trace, n_experts=4, capacity=3)
    assert hits.tolist() == [5] and misses.tolist() == [5]
    # capacity >= distinct ids: only compulsory misses
    h, m = oracle.lru_sim(trace, n_experts=4, capacity=4)
    assert m.tolist() == [4] and h.tolist() == [6]
    # capacity == k and disjoint consecutive tokens: every access misses
    tr = np.array([[[0, 1]], [[2, 3]], [[0, 1]], [[2, 3]]], dtype=np.int32)
    h, m = oracle.lru_sim(tr, n_experts=4, capacity=2)
    assert h.tolist() == [0] and m.tolist() == [8]
    with pytest.raises(ValueError):
        oracle.lru_sim(tr, n_experts=4, capacity=1)


def test_lru_invariants_on_zipf_trace():
    tr = synth.zipf_trace(0, 3, 256, 8, 200)
    for cap in (8, 32, 128, 256):
        h, m = oracle.lru_sim(tr, 256, cap)
        assert np.all(h + m == 200 * 8)
        if cap == 256:
            for l in range(3):
                assert int(m[l]) == len(np.unique(tr[:, l, :]))
    h8, m8 = oracle.lru_sim(tr, 256, 8)
    h128, m128 = oracle.lru_sim(tr, 256, 128)
    assert np.all(m128 <= m8)


def test_lru_pinned_hand_worked():
    # capacity 3, k 2, expert 0 pinned: the LRU part has 2 slots.
    # t0 {0,1}: 0 pinned hit; 1 -> empty slot            h1 m1
    # t1 {0,2}: 0 hit; 2 -> empty slot                   h1 m1   [1@1 2@2]
    # t2 {1,2}: both hit, touched 1 then 2               h2 m0   [1@3 2@4]
    # t3 {0,3}: 0 hit; 3 evicts the LRU of {1,2}: 1      h1 m1   [3@5 2@4]
    # t4 {1,3}: 3 hit; 1 evicts the LRU not in {1,3}: 2  h1 m1
    trace = np.array([[[0, 1]], [[0, 2]], [[1, 2]], [[0, 3]], [[1, 3]]], dtype=np.int32)
    h, m = oracle.lru_sim_pinned(trace, 4, 3, np.array([[0]]))
    assert h.tolist() == [6] and m.tolist() == [4]
    # the same trace unpinned: 0 is evicted at t2 (the LRU then) and misses at t3
    h, m = oracle.lru_sim(trace, 4, 3)
    assert h.tolist() == [5] and m.tolist() == [5]
    # fewer than k free slots left is refused
    with pytest.raises(ValueError):
        oracle.lru_sim_pinned(trace, 4, 3, np.array([[0, 1]]))


def test_lru_pinned_special_cases():
    tr = synth.zipf_trace(3, 2, 64, 4, 300)
    # nothing pinned: the plain LRU
    for cap in (4, 9, 32):
        h0, m0 = oracle.lru_sim_pinned(tr, 64, cap, np.zeros((2, 0), dtype=np.int32))
        h1, m1 = oracle.lru_sim(tr, 64, cap)
        assert np.array_equal(h0, h1) and np.array_equal(m0, m1)
    # pinned experts never miss; with room for every other id seen, only
    # the first access of each unpinned id misses
    pinned = np.array([[0, 5, 17], [2, 3, 40]], dtype=np.int32)
    for l in range(2):
        other = np.setdiff1d(np.unique(tr[:, l, :]), pinned[l])
        cap = 3 + len(other)
        h, m = oracle.lru_sim_pinned(tr[:, l:l + 1, :], 64, cap, pinned[l:l + 1])
        assert int(m[0]) == len(other)
        assert int(h[0]) + int(m[0]) == 300 * 4
    # a trace made only of pinned ids never misses
    only = np.tile(np.array([[[0, 5]]], dtype=np.int32), (10, 1, 1))
    h, m = oracle.lru_sim_pinned(only, 64, 4, np.array([[0, 5]]))
    assert m.tolist() == [0] and h.tolist() == [20]


# ---------------------------------------------------------------------------
# byte figures printed on the pages (P1-P4)

def _golden_figures():
    rows = []
    with open(os.path.join(HERE, "golden", "page_byte_figures.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, val, unit, tol, formula, src = [c.strip() for c in line.split("|")]
            rows.append((name, float(val), unit, float(tol), formula))
    return rows


def test_page_byte_figures_pin_the_shapes():
    H, I = synth.GLM.hidden, synth.GLM.inter
    units = {"GiB": 2 ** 30, "GB": 1e9, "TB": 1e12, "MB": 1e6, "x": 1}
    rows = _golden_figures()
    assert len(rows) == 7
    for name, val, unit, tol, formula in rows:
        got = eval(formula, {"H": H, "I": I}) / units[unit]
        assert abs(got - val) <= tol * val, (name, got, val)


def test_expert_bytes_closed_form():
    # P4: 3*H*I/2 code bytes + 3*H*I/32 fp16 scales = 21,233,664 bytes
    assert synth.GLM.expert_bytes == 21_233_664
    assert synth.TINY.expert_bytes == 55_296
    for sh in (synth.TINY,):
        e = synth.expert(sh, 0, 0, 0)
        assert sum(a.nbytes for a in e.values()) == sh.expert_bytes
    # per token-layer algorithmic bytes at batch 1 (8 routed + shared experts,
    # fp32 router, bias, bf16 x, fp32 y)
    G = synth.GLM
    per_token = 9 * G.expert_bytes + G.n_experts * G.hidden * 4 + G.n_experts * 4 \
        + G.hidden * 2 + G.hidden * 4
    assert per_token == 197_432_320

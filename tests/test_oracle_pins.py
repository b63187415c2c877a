"""Pins for the float64 CPU oracle (runs without a GPU).

Each test ties the oracle to something other than itself: a hand-worked
example, a closed form, a special case that reduces to a numpy routine, or an
invariant of the method ("MINIMAX SIGNAL LAB · M1", §03 Lightning Attention).
A wrong sign, a dropped term, a transposed state or an off-by-one exponent in
any of the three forms fails at least one of these.
"""
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal(shape) * scale).astype(np.float32)


def _to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest even) and return the bit patterns."""
    u = x.astype(np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def _close(a, b, rtol):
    scale = max(np.max(np.abs(b)), 1e-300)
    assert np.max(np.abs(a - b)) <= rtol * scale, np.max(np.abs(a - b)) / scale


SLOPES_MIX = np.array([0.0, 0.05, 0.9, 3.0], dtype=np.float32)


@pytest.mark.parametrize("with_state", [False, True])
def test_three_forms_agree_for_every_block(with_state):
    b, h, L, d = 2, 4, 13, 5
    q, k, v = (_rand((b, h, L, d), s, 0.5) for s in (1, 2, 3))
    s0 = _rand((b, h, d, d), 4, 0.3) if with_state else None
    o1, s1 = oracle.prefill(q, k, v, SLOPES_MIX, s0, form="definition")
    o2, s2 = oracle.prefill(q, k, v, SLOPES_MIX, s0, form="recurrence")
    _close(o2, o1, 1e-12)
    _close(s2, s1, 1e-12)
    for B in range(1, L + 3):
        o3, s3 = oracle.prefill(q, k, v, SLOPES_MIX, s0, form="blockwise", block=B)
        _close(o3, o1, 1e-12)
        _close(s3, s1, 1e-12)


def test_bf16_inputs_are_widened_exactly():
    b, h, L, d = 1, 4, 9, 6
    qf, kf, vf = (_rand((b, h, L, d), s) for s in (5, 6, 7))
    qb, kb, vb = (_to_bf16_bits(x) for x in (qf, kf, vf))
    # the same values handed over as float32 must give the identical result
    widen = lambda bits: oracle.bf16_bits_to_f64(bits).astype(np.float32)
    o_b, s_b = oracle.prefill(qb, kb, vb, SLOPES_MIX)
    o_f, s_f = oracle.prefill(widen(qb), widen(kb), widen(vb), SLOPES_MIX)
    assert np.array_equal(o_b, o_f) and np.array_equal(s_b, s_f)
    # and the widening itself is exact: bf16 bits -> float64 -> bits round trip
    back = _to_bf16_bits(oracle.bf16_bits_to_f64(qb).astype(np.float32))
    assert np.array_equal(back, qb)


def test_hand_worked_example():
    rows = {}
    with open(os.path.join(GOLDEN, "hand_example_d1.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, *vals = line.split()
            rows[name] = np.array([float(x) for x in vals])
    shape = (1, 1, 3, 1)
    q, k, v = (rows[n].astype(np.float32).reshape(shape) for n in ("q", "k", "v"))
    slope = np.array([math.log(2.0)], dtype=np.float32)
    for form, blk in (("definition", None), ("recurrence", None), ("blockwise", 2)):
        o, s = oracle.prefill(q, k, v, slope, form=form, block=blk)
        np.testing.assert_allclose(o.ravel(), rows["o"], rtol=1e-7)
        np.testing.assert_allclose(s.ravel(), rows["state_out"], rtol=1e-7)


@pytest.mark.parametrize("s", [0.01, 0.3, 1.7])
def test_closed_form_constant_inputs(s):
    # q_i = q, k_j = k, v_j = v:  o_i = (q.k) v (1 - e^{-s(i+1)}) / (1 - e^{-s}),
    # S_L = (1 - e^{-sL}) / (1 - e^{-s}) k^T v  (geometric series).
    L, d = 40, 3
    qv = np.array([0.5, -1.0, 0.25], np.float32)
    kv = np.array([1.0, 0.5, -0.75], np.float32)
    vv = np.array([2.0, -0.5, 1.5], np.float32)
    q = np.broadcast_to(qv, (1, 1, L, d)).copy()
    k = np.broadcast_to(kv, (1, 1, L, d)).copy()
    v = np.broadcast_to(vv, (1, 1, L, d)).copy()
    sl = np.array([s], np.float32)
    sd = float(sl[0])
    r = math.exp(-sd)
    i = np.arange(L)
    expect_o = (float(qv.astype(np.float64) @ kv.astype(np.float64))
                * ((1 - r ** (i + 1)) / (1 - r))[:, None] * vv.astype(np.float64)[None, :])
    expect_s = (1 - r ** L) / (1 - r) * np.outer(kv.astype(np.float64), vv.astype(np.float64))
    for form, blk in (("definition", None), ("recurrence", None), ("blockwise", 16)):
        o, st = oracle.prefill(q, k, v, sl, form=form, block=blk)
        _close(o[0, 0], expect_o, 1e-12)
        _close(st[0, 0], expect_s, 1e-12)


def test_zero_slope_is_plain_causal_linear_attention():
    # s = 0: o_i = q_i (S_in + sum_{j<=i} k_j^T v_j), a prefix sum (numpy cumsum).
    b, h, L, d = 1, 2, 11, 4
    q, k, v = (_rand((b, h, L, d), s) for s in (8, 9, 10))
    s0 = _rand((b, h, d, d), 11)
    sl = np.zeros(h, np.float32)
    K, V, Q = (x.astype(np.float64) for x in (k, v, q))
    outer = np.einsum("bhjr,bhjc->bhjrc", K, V)
    pref = np.cumsum(outer, axis=2) + s0.astype(np.float64)[:, :, None]
    expect = np.einsum("bhir,bhirc->bhic", Q, pref)
    for form, blk in (("definition", None), ("recurrence", None), ("blockwise", 4)):
        o, st = oracle.prefill(q, k, v, sl, s0, form=form, block=blk)
        _close(o, expect, 1e-12)
        _close(st, pref[:, :, -1], 1e-12)


def test_large_slope_keeps_only_the_diagonal():
    # e^{-s} underflows to 0: o_i = (q_i . k_i) v_i and S_out = k_{L-1}^T v_{L-1}.
    b, h, L, d = 1, 1, 7, 4
    q, k, v = (_rand((b, h, L, d), s) for s in (12, 13, 14))
    s0 = _rand((b, h, d, d), 15)
    sl = np.array([1.0e4], np.float32)
    Q, K, V = (x.astype(np.float64)[0, 0] for x in (q, k, v))
    expect = np.sum(Q * K, axis=1)[:, None] * V
    for form, blk in (("definition", None), ("recurrence", None), ("blockwise", 3)):
        o, st = oracle.prefill(q, k, v, sl, s0, form=form, block=blk)
        _close(o[0, 0], expect, 1e-14)
        _close(st[0, 0], np.outer(K[-1], V[-1]), 1e-14)


def test_single_block_is_one_masked_matmul():
    # L <= B: O = ((Q K^T) ⊙ D) V + diag(d_q) Q S_in, written with numpy matmuls.
    L, d = 9, 6
    q, k, v = (_rand((1, 1, L, d), s) for s in (16, 17, 18))
    s0 = _rand((1, 1, d, d), 19)
    s = np.float32(0.37)
    Q, K, V = (x.astype(np.float64)[0, 0] for x in (q, k, v))
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    D = np.where(i >= j, np.exp(-float(s) * (i - j)), 0.0)
    dq = np.exp(-float(s) * (np.arange(L) + 1.0))
    expect = ((Q @ K.T) * D) @ V + dq[:, None] * (Q @ s0.astype(np.float64)[0, 0])
    for form, blk in (("definition", None), ("recurrence", None), ("blockwise", 16)):
        o, _ = oracle.prefill(q, k, v, np.array([s]), s0, form=form, block=blk)
        _close(o[0, 0], expect, 1e-12)


def test_linearity_in_v_and_state():
    b, h, L, d = 1, 3, 10, 4
    q, k, v1, v2 = (_rand((b, h, L, d), s) for s in (20, 21, 22, 23))
    sa, sb = _rand((b, h, d, d), 24), _rand((b, h, d, d), 25)
    sl = SLOPES_MIX[:3]
    a, c = 0.75, -1.5
    o1, t1 = oracle.prefill(q, k, v1, sl, sa)
    o2, t2 = oracle.prefill(q, k, v2, sl, sb)
    o12, t12 = oracle.prefill(q, k, (a * v1 + c * v2).astype(np.float32), sl,
                              (a * sa + c * sb).astype(np.float32))
    # inputs were rounded to float32 once, so compare against the rounded combination
    va = (a * v1 + c * v2).astype(np.float32)
    assert np.all(np.isfinite(va))
    _close(o12, a * o1 + c * o2, 1e-6)
    _close(t12, a * t1 + c * t2, 1e-6)


def test_chunked_prefill_and_decode_continue_the_sequence():
    b, h, L, d = 2, 4, 17, 5
    q, k, v = (_rand((b, h, L + 1, d), s) for s in (26, 27, 28))
    s0 = _rand((b, h, d, d), 29)
    o_full, s_full = oracle.prefill(q, k, v, SLOPES_MIX, s0)
    for cut in (1, 6, 16):
        oa, sa = oracle.prefill(q[:, :, :cut], k[:, :, :cut], v[:, :, :cut], SLOPES_MIX, s0)
        ob, sb = oracle.prefill(q[:, :, cut:], k[:, :, cut:], v[:, :, cut:], SLOPES_MIX,
                                sa.astype(np.float32))
        # the carried state is rounded to float32 between the two calls, as on the GPU
        _close(np.concatenate([oa, ob], axis=2), o_full, 1e-6)
        _close(sb, s_full, 1e-6)
    # decode of token L after a prefill of L tokens == prefill of L+1 tokens
    op, sp = oracle.prefill(q[:, :, :L], k[:, :, :L], v[:, :, :L], SLOPES_MIX, s0)
    od, sd = oracle.decode(q[:, :, L], k[:, :, L], v[:, :, L], SLOPES_MIX, sp)
    _close(od, o_full[:, :, L], 1e-12)
    _close(sd, s_full, 1e-12)


def test_carried_state_is_forgotten_at_the_slope_rate():
    # the state's share of o_i is e^{-s(i+1)} q_i S_in, so |share| <= e^{-s(i+1)} |q_i| |S_in|
    b, h, L, d = 1, 4, 30, 4
    q, k, v = (_rand((b, h, L, d), s) for s in (30, 31, 32))
    s0 = _rand((b, h, d, d), 33, 5.0)
    with_s, _ = oracle.prefill(q, k, v, SLOPES_MIX, s0)
    without, _ = oracle.prefill(q, k, v, SLOPES_MIX, None)
    share = with_s - without
    for hh, s in enumerate(SLOPES_MIX.astype(np.float64)):
        qn = np.linalg.norm(q[0, hh].astype(np.float64), axis=1)
        sn = np.linalg.norm(s0[0, hh].astype(np.float64), 2)
        bound = np.exp(-s * (np.arange(L) + 1)) * qn * sn
        # subtracting two float64 results leaves rounding noise of ~1e-16 |o|
        noise = 1e-13 * np.max(np.abs(without[0, hh]))
        assert np.all(np.linalg.norm(share[0, hh], axis=1) <= bound * (1 + 1e-12) + noise)


def test_empty_sequence_decays_nothing_and_returns_the_state():
    b, h, d = 1, 2, 3
    z = np.zeros((b, h, 0, d), np.float32)
    s0 = _rand((b, h, d, d), 34)
    for form, blk in (("definition", None), ("recurrence", None), ("blockwise", 4)):
        o, st = oracle.prefill(z, z, z, SLOPES_MIX[:2], s0, form=form, block=blk)
        assert o.shape == (b, h, 0, d)
        np.testing.assert_array_equal(st, s0.astype(np.float64))


def test_state_size_matches_the_printed_m1_figure():
    vals = {}
    with open(os.path.join(GOLDEN, "state_size_m1.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            key, val = line.split()
            vals[key] = float(val)
    H, d = int(vals["heads"]), int(vals["dim"])
    z = np.zeros((1, H, 1, d), np.float32)
    _, st = oracle.prefill(z, z, z, np.ones(H, np.float32))
    per_layer = st.astype(np.float32).nbytes
    total_mb = vals["layers"] * per_layer / 1e6
    assert abs(total_mb - vals["printed_megabytes"]) < 0.01


@pytest.mark.parametrize("with_state", [False, True])
def test_snapshots_are_the_states_of_the_prefixes(with_state):
    # snapshot n is the state a prefill of the first (n+1)*interval tokens leaves behind,
    # taken here from the quadratic definition (F1), an independent form
    b, h, L, d, interval = 2, 4, 23, 5, 4
    q, k, v = (_rand((b, h, L, d), s) for s in (40, 41, 42))
    s0 = _rand((b, h, d, d), 43) if with_state else None
    snaps = oracle.snapshots(k, v, SLOPES_MIX, interval, s0)
    assert snaps.shape == (b, h, L // interval, d, d)
    for n in range(L // interval):
        n_tok = (n + 1) * interval
        _, s_prefix = oracle.prefill(q[:, :, :n_tok], k[:, :, :n_tok], v[:, :, :n_tok], SLOPES_MIX, s0,
                                     form="definition")
        _close(snaps[:, :, n], s_prefix, 1e-12)
    # an interval longer than the sequence takes no snapshot; interval == L takes state_out
    assert oracle.snapshots(k, v, SLOPES_MIX, L + 1, s0).shape == (b, h, 0, d, d)
    _, s_out = oracle.prefill(q, k, v, SLOPES_MIX, s0, form="definition")
    _close(oracle.snapshots(k, v, SLOPES_MIX, L, s0)[:, :, 0], s_out, 1e-12)


def _exact_grid(shape, seed, lo=-2.0, hi=2.0):
    # values on a 1/64 grid: x +- 2^-12 stays exact in float32
    rng = np.random.default_rng(seed)
    return (np.round(rng.uniform(lo, hi, shape) * 64) / 64).astype(np.float32)


@pytest.mark.parametrize("with_state", [False, True])
def test_backward_matches_finite_differences_of_the_definition(with_state):
    # The loss sum(dO * o) + sum(dS_out * S_out) is linear in every single input
    # element, so a central difference of the definition (F1) is its exact derivative.
    b, h, L, d = 1, 2, 6, 3
    sl = np.array([0.25, 1.5], np.float32)
    q, k, v = (_exact_grid((b, h, L, d), s) for s in (50, 51, 52))
    s0 = _exact_grid((b, h, d, d), 53) if with_state else None
    d_o = _rand((b, h, L, d), 54)
    ds_out = _rand((b, h, d, d), 55)
    dq, dk, dv, ds_in = oracle.backward(q, k, v, d_o, sl, s0, ds_out)

    def loss(qq, kk, vv, ss):
        o, st = oracle.prefill(qq, kk, vv, sl, ss, form="definition")
        return float(np.sum(d_o.astype(np.float64) * o) + np.sum(ds_out.astype(np.float64) * st))

    eps = 2.0 ** -12
    for name, grad in (("q", dq), ("k", dk), ("v", dv), ("s", ds_in)):
        for idx in np.ndindex(*grad.shape):
            args = {"q": q, "k": k, "v": v, "s": s0 if s0 is not None else np.zeros((b, h, d, d), np.float32)}
            plus = {n: a.copy() for n, a in args.items()}
            minus = {n: a.copy() for n, a in args.items()}
            plus[name][idx] += eps
            minus[name][idx] -= eps
            fd = (loss(plus["q"], plus["k"], plus["v"], plus["s"]) -
                  loss(minus["q"], minus["k"], minus["v"], minus["s"])) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-9 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])


def test_backward_of_an_empty_sequence_passes_the_state_gradient():
    b, h, d = 1, 2, 3
    z = np.zeros((b, h, 0, d), np.float32)
    ds_out = _rand((b, h, d, d), 56)
    dq, dk, dv, ds_in = oracle.backward(z, z, z, z, SLOPES_MIX[:2], None, ds_out)
    assert dq.shape == (b, h, 0, d)
    np.testing.assert_array_equal(ds_in, ds_out.astype(np.float64))


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x.astype(np.float64)))


@pytest.mark.parametrize("per_head", [True, False])
def test_norm_gate_closed_forms(per_head):
    b, h, L, d = 2, 3, 5, 4
    g = _rand((b, L, h * d), 60)
    gamma = _rand((h * d,), 61)
    # constant channels c: every group's rms is |c|, so y = gamma * sign(c) * |c| / sqrt(c^2 + eps) * sigmoid(g)
    for c, eps in ((0.75, 0.0), (-2.0, 0.5)):
        o = np.full((b, h, L, d), c, np.float32)
        y = oracle.norm_gate(o, g, gamma, eps, per_head)
        want = gamma.astype(np.float64) * c / np.sqrt(c * c + eps) * _sigmoid(g)
        _close(y, want, 1e-12)
    # a zero gate halves; a large positive gate passes the normalised value through
    o = _rand((b, h, L, d), 62)
    y0 = oracle.norm_gate(o, np.zeros_like(g), gamma, 1e-6, per_head)
    y1 = oracle.norm_gate(o, np.full_like(g, 60.0), gamma, 1e-6, per_head)
    _close(y0, 0.5 * y1, 1e-12)


@pytest.mark.parametrize("per_head", [True, False])
def test_norm_gate_is_scale_invariant_and_groups_as_stated(per_head):
    b, h, L, d = 1, 4, 3, 8
    o = _rand((b, h, L, d), 63)
    g = _rand((b, L, h * d), 64)
    gamma = np.ones((h * d,), np.float32)
    y = oracle.norm_gate(o, g, gamma, 0.0, per_head)
    _close(oracle.norm_gate(o * np.float32(4.0), g, gamma, 0.0, per_head), y, 1e-12)
    # with gamma = 1 and eps = 0, every group of the normalised output has mean square 1
    x = y / _sigmoid(g)
    grp = d if per_head else h * d
    ms = np.mean(x.reshape(b, L, (h * d) // grp, grp) ** 2, axis=-1)
    _close(ms, np.ones_like(ms), 1e-12)
    # token channel n = head * dim + c reads o[b, head, l, c]
    if per_head:
        one = np.zeros_like(o)
        one[0, 2, 1, 5] = 3.0
        yy = oracle.norm_gate(one, np.full_like(g, 60.0), gamma, 1e-30, True)  # eps > 0: zero heads stay 0
        assert abs(yy[0, 1, 2 * d + 5] - np.sqrt(d)) < 1e-9
        assert np.count_nonzero(yy[0, 1]) == 1


def _gqa_case(b=2, h=8, hk=2, d=16, cap=12, seed=70):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((b, h, d)).astype(np.float32)
    kn = rng.standard_normal((b, hk, d)).astype(np.float32)
    vn = rng.standard_normal((b, hk, d)).astype(np.float32)
    kc = rng.standard_normal((b, hk, cap, d)).astype(np.float32)
    vc = rng.standard_normal((b, hk, cap, d)).astype(np.float32)
    return q, kn, vn, kc, vc


def test_rope_is_a_rotation_of_relative_position():
    rng = np.random.default_rng(71)
    x, y = rng.standard_normal(16), rng.standard_normal(16)
    np.testing.assert_allclose(oracle.rope(x, 0, 8, 1e4), x, rtol=0, atol=0)        # position 0: identity
    np.testing.assert_allclose(np.linalg.norm(oracle.rope(x, 777, 8, 1e4)), np.linalg.norm(x), rtol=1e-13)
    np.testing.assert_array_equal(oracle.rope(x, 55, 8, 1e4)[8:], x[8:])           # dims past rot untouched
    a = oracle.rope(x, 40, 8, 1e4) @ oracle.rope(y, 13, 8, 1e4)
    b = oracle.rope(x, 1040, 8, 1e4) @ oracle.rope(y, 1013, 8, 1e4)
    assert abs(a - b) < 1e-10                                                      # only m - n matters


def test_gqa_decode_special_cases():
    q, kn, vn, kc, vc = _gqa_case()
    b, h, d = q.shape
    hk = kn.shape[1]
    # position 0: the only key is the new one, so o is its value for every query head
    o = oracle.gqa_decode(q, kn, vn, kc, vc, np.zeros(b, np.int32), 8, 1e4, 0.25)
    for hh in range(h):
        np.testing.assert_allclose(o[:, hh], vn[:, hh // (h // hk)].astype(np.float64), rtol=0, atol=1e-14)
    # identical keys everywhere: softmax is uniform, o = mean of the values
    kcu = np.zeros_like(kc)
    knu = np.zeros_like(kn)
    pos = np.array([5, 9], np.int32)
    o = oracle.gqa_decode(q, knu, vn, kcu, vc, pos, 8, 1e4, 0.25)
    for bb in range(b):
        for hh in range(h):
            g = hh // (h // hk)
            want = (vc[bb, g, :pos[bb]].astype(np.float64).sum(0) + vn[bb, g]) / (pos[bb] + 1)
            np.testing.assert_allclose(o[bb, hh], want, rtol=1e-12, atol=1e-12)
    # one key aligned with a large query: softmax saturates on it
    qq = np.zeros_like(q)
    qq[:, :, 12] = 50.0                       # dim 12 lies past the rotated dims
    kca = np.zeros_like(kc)
    kca[:, :, 3, 12] = 50.0
    o = oracle.gqa_decode(qq, np.zeros_like(kn), vn, kca, vc, pos, 8, 1e4, 1.0)
    for hh in range(h):
        np.testing.assert_allclose(o[:, hh], vc[:, hh // (h // hk), 3].astype(np.float64), rtol=0, atol=1e-9)


def test_gqa_decode_matches_a_numpy_softmax_with_grouping():
    # brute force on a tiny case: numpy softmax over explicitly assembled keys
    q, kn, vn, kc, vc = _gqa_case(b=1, h=4, hk=2, d=8, cap=6, seed=72)
    pos = np.array([4], np.int32)
    o = oracle.gqa_decode(q, kn, vn, kc, vc, pos, 4, 100.0, 0.3)
    for hh in range(4):
        g = hh // 2
        keys = np.concatenate([kc[0, g, :4].astype(np.float64), oracle.rope(kn[0, g], 4, 4, 100.0)[None]], 0)
        vals = np.concatenate([vc[0, g, :4].astype(np.float64), vn[0, g].astype(np.float64)[None]], 0)
        s = 0.3 * keys @ oracle.rope(q[0, hh], 4, 4, 100.0)
        w = np.exp(s - s.max())
        np.testing.assert_allclose(o[0, hh], (w / w.sum()) @ vals, rtol=1e-12, atol=1e-12)


def test_gqa_decode_rotates_query_and_new_key_alike():
    # cached keys zero: only the new key scores, with rope(q, P) . rope(k, P) = q . k at any P,
    # so o = (sum_{p<P} v_p + e^{s} v_new) / (P + e^{s}), s = scale * q . k
    q, kn, vn, kc, vc = _gqa_case(b=1, h=4, hk=1, d=16, cap=40, seed=73)
    z = np.zeros_like(kc)
    for P in (0, 7, 39):
        o = oracle.gqa_decode(q, kn, vn, z, vc, np.array([P], np.int32), 16, 500.0, 0.2)
        for hh in range(4):
            s = 0.2 * float(q[0, hh].astype(np.float64) @ kn[0, 0].astype(np.float64))
            want = (vc[0, 0, :P].astype(np.float64).sum(0) + np.exp(s) * vn[0, 0]) / (P + np.exp(s))
            np.testing.assert_allclose(o[0, hh], want, rtol=1e-12, atol=1e-12)


def _gqa_prefill_case(b=2, h=4, hk=2, L=6, d=16, cap=20, seed=80):
    rng = np.random.default_rng(seed)
    f = lambda *s: rng.standard_normal(s).astype(np.float32)
    return f(b, h, L, d), f(b, hk, L, d), f(b, hk, L, d), f(b, hk, cap, d), f(b, hk, cap, d)


def test_gqa_prefill_matches_a_numpy_causal_softmax():
    # brute force: every key and value of the sequence assembled explicitly, one masked
    # score matrix per head, numpy softmax along keys
    q, kn, vn, kc, vc = _gqa_prefill_case()
    start, rot, base, scale = 5, 8, 100.0, 0.3
    o = oracle.gqa_prefill(q, kn, vn, kc, vc, start, rot, base, scale)
    b, h, L, d = q.shape
    hk = kn.shape[1]
    for bb in range(b):
        for hh in range(h):
            g = hh // (h // hk)
            keys = np.concatenate([kc[bb, g, :start].astype(np.float64),
                                   np.stack([oracle.rope(kn[bb, g, i], start + i, rot, base) for i in range(L)])])
            vals = np.concatenate([vc[bb, g, :start], vn[bb, g]]).astype(np.float64)
            qr = np.stack([oracle.rope(q[bb, hh, i], start + i, rot, base) for i in range(L)])
            s = scale * qr @ keys.T                                   # [L, start + L]
            s[np.arange(start + L)[None, :] > (start + np.arange(L))[:, None]] = -np.inf
            w = np.exp(s - s.max(1, keepdims=True))
            np.testing.assert_allclose(o[bb, hh], (w / w.sum(1, keepdims=True)) @ vals, rtol=1e-12, atol=1e-12)


def test_gqa_prefill_is_a_chain_of_decode_steps():
    # token i of a prefill is the decode step at position start + i over a cache that holds
    # the earlier new tokens (rotated keys) after the given prefix
    q, kn, vn, kc, vc = _gqa_prefill_case(b=1, h=4, hk=1, L=5, d=16, cap=12, seed=81)
    start, rot, base, scale = 3, 16, 500.0, 0.25
    o = oracle.gqa_prefill(q, kn, vn, kc, vc, start, rot, base, scale)
    kcc, vcc = kc.copy(), vc.copy()
    for i in range(q.shape[2]):
        od = oracle.gqa_decode(q[:, :, i], kn[:, :, i], vn[:, :, i], kcc, vcc, np.array([start + i], np.int32),
                               rot, base, scale)
        # the decode step reads the earlier keys back from a float32 cache
        np.testing.assert_allclose(o[:, :, i], od, rtol=0, atol=2e-6)
        kcc[0, 0, start + i] = oracle.rope(kn[0, 0, i], start + i, rot, base).astype(np.float32)
        vcc[0, 0, start + i] = vn[0, 0, i]
    # one token: exactly the decode step
    o1 = oracle.gqa_prefill(q[:, :, :1], kn[:, :, :1], vn[:, :, :1], kc, vc, start, rot, base, scale)
    od = oracle.gqa_decode(q[:, :, 0], kn[:, :, 0], vn[:, :, 0], kc, vc, np.array([start], np.int32), rot, base, scale)
    np.testing.assert_allclose(o1[:, :, 0], od, rtol=1e-13, atol=1e-13)


def test_gqa_prefill_is_causal_and_rows_are_independent():
    q, kn, vn, kc, vc = _gqa_prefill_case(seed=82)
    args = (4, 8, 1e4, 0.2)
    o = oracle.gqa_prefill(q, kn, vn, kc, vc, *args)
    q2, kn2, vn2 = q.copy(), kn.copy(), vn.copy()
    q2[:, :, 3:] += 1.0
    kn2[:, :, 3:] -= 2.0
    vn2[:, :, 3:] *= 3.0
    o2 = oracle.gqa_prefill(q2, kn2, vn2, kc, vc, *args)
    np.testing.assert_array_equal(o[:, :, :3], o2[:, :, :3])     # earlier tokens never see later ones
    assert np.abs(o[:, :, 3:] - o2[:, :, 3:]).max() > 1e-3
    b, h, L, d = q.shape
    rows = np.array([0, 7, L * 3 + 2, b * h * L - 1])
    np.testing.assert_array_equal(oracle.gqa_prefill(q, kn, vn, kc, vc, *args, rows=rows), o.reshape(-1, d)[rows])


def test_gqa_prefill_with_identical_keys_averages_the_prefix():
    q, kn, vn, kc, vc = _gqa_prefill_case(seed=83)
    start = 7
    o = oracle.gqa_prefill(q, np.zeros_like(kn), vn, np.zeros_like(kc), vc, start, 8, 1e4, 0.5)
    b, h, L, d = q.shape
    hk = kn.shape[1]
    for hh in range(h):
        g = hh // (h // hk)
        vals = np.concatenate([vc[:, g, :start], vn[:, g]], 1).astype(np.float64)
        for i in range(L):
            np.testing.assert_allclose(o[:, hh, i], vals[:, :start + i + 1].mean(1), rtol=1e-12, atol=1e-12)


def test_gqa_prefill_rejects_bad_arguments():
    q, kn, vn, kc, vc = _gqa_prefill_case(L=6, cap=20)
    with pytest.raises(RuntimeError):
        oracle.gqa_prefill(q, kn, vn, kc, vc, 15, 8, 1e4, 0.5)   # start + seq > cap
    with pytest.raises(RuntimeError):
        oracle.gqa_prefill(q, kn, vn, kc, vc, 0, 7, 1e4, 0.5)    # odd rot
    with pytest.raises(RuntimeError):
        oracle.gqa_prefill(q, kn, vn, kc, vc, 0, 8, 1e4, 0.5, rows=[10 ** 6])

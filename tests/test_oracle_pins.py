"""Pins of the float64 CPU oracle against what the mathematics fixes.

The pages print no worked numeric example for this layer, so the oracle is
pinned by: closed forms (RMSNorm of constant rows, sigmoid at ties),
brute-force enumeration of expert subsets, hand-computed end-to-end cases on
2x2 matrices whose arithmetic is written out below, exact reductions
(LatentMoE with identity fc1/fc2 is the direct layer; FP8 weights whose
dequantised values are BF16-exact give the BF16 result), and invariants
(weights sum to routed_scaling_factor, a zero-weight expert contributes
nothing, the sort is a stable bijection, tokens are independent).

Each hand case is chosen so that a transposed operand, a dropped term (norm
weight, residual, shared expert, scaling factor) or relu instead of relu^2
changes the result.
"""
import itertools
import math

import numpy as np
import pytest

import oracle
from tests.helpers import custom_inputs, exact_bf16
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.oracle


def sig(x):
    return 1.0 / (1.0 + math.exp(-x))


# ---------------------------------------------------------------- formats ---

def test_bf16_decode_known_values():
    assert oracle.bf16_value(0x3F80) == 1.0
    assert oracle.bf16_value(0xC000) == -2.0
    assert oracle.bf16_value(0x3E80) == 0.25
    assert oracle.bf16_value(0x0001) == 2.0 ** -133   # smallest subnormal
    assert oracle.bf16_value(0x7F7F) == (2 - 2 ** -7) * 2.0 ** 127


def test_e4m3_decode_known_values():
    # OCP FP8 E4M3 ("fn"): bias 7, no infinities, S.1111.111 is NaN.
    assert oracle.e4m3_value(0x38) == 1.0
    assert oracle.e4m3_value(0xB8) == -1.0
    assert oracle.e4m3_value(0x7E) == 448.0
    assert oracle.e4m3_value(0x08) == 2.0 ** -6      # smallest normal
    assert oracle.e4m3_value(0x01) == 2.0 ** -9      # smallest subnormal
    assert oracle.e4m3_value(0x07) == 7 * 2.0 ** -9
    assert oracle.e4m3_value(0x3C) == 1.5
    assert math.isnan(oracle.e4m3_value(0x7F))


# ---------------------------------------------------------------- RMSNorm ---

def _norm_only(H, norm_w, hidden, eps):
    inp = custom_inputs(H, 1, 1, 1, 1, eps=eps, norm_w=norm_w, gate_w=np.zeros(H),
                        up_w=np.zeros(H), down_w=np.zeros(H), shared_up_w=np.zeros(H),
                        shared_down_w=np.zeros(H), hidden=hidden)
    return oracle.Oracle(inp).rmsnorm(inp.hidden)


def test_rmsnorm_constant_row_closed_form():
    # x = c*1  =>  n_i = c / sqrt(c^2 + eps) * w_i
    H, c, eps = 8, 2.0, 1e-5
    w = np.array([0.5, 0.75, 1.0, 1.25, 1.5, 1.0, 0.625, 1.375])
    n = _norm_only(H, w, np.full((1, H), c), eps)
    np.testing.assert_allclose(n[0], c / math.sqrt(c * c + eps) * w, rtol=1e-15)


def test_rmsnorm_345_row():
    # x = [3, 4, 0, 0], eps = 0: mean square 25/4, r = 0.4, n = [1.2, 1.6, 0, 0] * w
    w = np.array([1.0, 0.5, 1.5, 1.0])
    n = _norm_only(4, w, np.array([[3.0, 4.0, 0.0, 0.0]]), 0.0)
    np.testing.assert_allclose(n[0], np.array([1.2, 0.8, 0.0, 0.0]), rtol=1e-15, atol=0)


def test_rmsnorm_scale_invariant_without_eps():
    rng = np.random.default_rng(7)
    x = exact_bf16(np.round(rng.standard_normal((3, 16)) * 8) / 8)
    xf = np.asarray(x, dtype=np.uint16)
    from workloads import bf16_to_f32
    v = bf16_to_f32(xf).astype(np.float64)
    w = np.linspace(0.5, 1.5, 16)
    w = np.round(w * 64) / 64
    n1 = _norm_only(16, w, v, 0.0)
    n2 = _norm_only(16, w, 4.0 * v, 0.0)
    np.testing.assert_allclose(n1, n2, rtol=1e-14)


# ------------------------------------------------------------ gate/route ---

def test_gate_hand_case():
    # n = [1, -0.5] (x = [1, -1], w = [1, 0.5], eps 0); G = [[0, 4], [-3, 0]]
    # logits = [0*1 + 4*(-0.5), -3*1 + 0] = [-2, -3]
    inp = custom_inputs(2, 2, 1, 1, 1, norm_w=[1, 0.5], gate_w=[[0, 4], [-3, 0]],
                        up_w=np.zeros(4), down_w=np.zeros(4), shared_up_w=[0, 0],
                        shared_down_w=[0, 0], hidden=[[1, -1]])
    lg = oracle.Oracle(inp).gate_logits(inp.hidden)
    np.testing.assert_array_equal(lg, [[-2.0, -3.0]])


def test_zero_gate_ties_pick_lowest_indices():
    # G = 0 => every score is sigmoid(0) = 1/2 => ties everywhere => experts
    # 0..k-1 in order, each weight rsf / k.
    s = WORKLOADS["tiny"].scaled(rsf=2.5)
    inp = make_inputs(s)
    inp.gate_w[:] = 0
    o = oracle.Oracle(inp)
    lg = o.gate_logits(inp.hidden)
    assert np.all(lg == 0.0)
    idx, w, keys = o.route(lg)
    assert np.all(keys == 0.5)
    np.testing.assert_array_equal(idx, np.tile(np.arange(s.k), (s.T, 1)))
    np.testing.assert_allclose(w, 2.5 / s.k, rtol=1e-15)


def _route_only(E, k, rsf, bias=None):
    inp = custom_inputs(2, E, k, 1, 1, rsf=rsf, norm_w=[1, 1], gate_w=np.zeros(2 * E),
                        up_w=np.zeros(2 * E), down_w=np.zeros(2 * E), shared_up_w=[0, 0],
                        shared_down_w=[0, 0], hidden=[[1, 1]], gate_bias=bias)
    return oracle.Oracle(inp)


def test_bias_selects_but_does_not_weight():
    # logits [2, 0, -1], bias [0, 0, 5]: keys = [s(2), s(0), s(-1) + 5] so the
    # selection is experts 2 then 0; the weights use the unbiased scores.
    o = _route_only(3, 2, 2.5, bias=[0.0, 0.0, 5.0])
    idx, w, keys = o.route(np.array([[2.0, 0.0, -1.0]]))
    np.testing.assert_array_equal(idx, [[2, 0]])
    den = sig(-1.0) + sig(2.0)
    np.testing.assert_allclose(w, [[2.5 * sig(-1.0) / den, 2.5 * sig(2.0) / den]], rtol=1e-14)
    np.testing.assert_allclose(keys, [[sig(2.0), 0.5, sig(-1.0) + 5.0]], rtol=1e-15)


def test_exact_ties_go_to_lower_index():
    # logits 0 (scores 1/2), bias [0, .25, .25, 0, .5] (exact): keys
    # [.5, .75, .75, .5, 1] -> slots 4, 1, 2 (1 before 2 on the tie).
    o = _route_only(5, 3, 1.0, bias=[0.0, 0.25, 0.25, 0.0, 0.5])
    idx, w, _ = o.route(np.zeros((1, 5)))
    np.testing.assert_array_equal(idx, [[4, 1, 2]])
    np.testing.assert_allclose(w, [[1 / 3, 1 / 3, 1 / 3]], rtol=1e-15)


@pytest.mark.parametrize("E,k", [(4, 1), (5, 2), (6, 3), (8, 4), (10, 4), (7, 7)])
def test_topk_matches_bruteforce_subset_enumeration(E, k):
    # The selected set maximises the sum of keys over all C(E, k) subsets;
    # slots come in descending key order; weights renormalise to rsf.
    rng = np.random.default_rng(E * 100 + k)
    rsf = 1.75
    bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    o = _route_only(E, k, rsf, bias=bias)
    logits = rng.standard_normal((50, E)) * 2
    idx, w, keys = o.route(logits)
    for t in range(logits.shape[0]):
        key = [sig(logits[t, e]) + float(bias[e]) for e in range(E)]
        best = max(itertools.combinations(range(E), k), key=lambda c: sum(key[e] for e in c))
        assert sorted(idx[t].tolist()) == list(best)
        got = [key[e] for e in idx[t]]
        assert got == sorted(got, reverse=True)
        s = [sig(logits[t, e]) for e in idx[t]]
        np.testing.assert_allclose(w[t], [rsf * x / sum(s) for x in s], rtol=1e-13)
        assert abs(w[t].sum() - rsf) < 1e-13


def test_weights_sum_to_scaling_factor_on_workload():
    s = WORKLOADS["tiny"].scaled(rsf=2.5)
    inp = make_inputs(s)
    o = oracle.Oracle(inp)
    _, w, _ = o.route(o.gate_logits(inp.hidden))
    np.testing.assert_allclose(w.sum(axis=1), 2.5, rtol=1e-14)
    assert np.all(w > 0)


# ------------------------------------------------------------------- sort ---

def _random_routing(rng, T, E, k):
    return np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)


@pytest.mark.parametrize("T,E,k", [(1, 4, 2), (16, 8, 2), (37, 128, 6), (300, 5, 3), (64, 128, 8)])
def test_sort_is_stable_bijection(T, E, k):
    rng = np.random.default_rng(T + E + k)
    idx = _random_routing(rng, T, E, k)
    perm, inv, off = oracle.sort(idx, E)
    flat = idx.reshape(-1)
    R = T * k
    # brute force: Python's stable sort of the flat rows by expert id
    expect = sorted(range(R), key=lambda f: (int(flat[f]), f))
    assert perm.tolist() == expect
    assert sorted(perm.tolist()) == list(range(R))             # bijection
    assert np.array_equal(inv[perm], np.arange(R))               # inverse
    cnt = np.bincount(flat, minlength=E)
    assert off[0] == 0 and off[-1] == R
    assert np.array_equal(np.diff(off), cnt)
    for e in range(E):                                           # bucket content
        assert np.all(flat[perm[off[e]:off[e + 1]]] == e)


def test_sort_empty_and_invalid():
    perm, inv, off = oracle.sort(np.zeros((0, 3), dtype=np.int32), 4)
    assert perm.size == 0 and np.all(off == 0)
    with pytest.raises(ValueError):
        oracle.sort(np.array([[0, 4]], dtype=np.int32), 4)


# ----------------------------------------------------- hand-computed layer ---

def test_hand_case_direct_single_expert():
    # x = [1, -1]; norm w = [1, 0.5]; eps = 0 -> r = 1, n = [1, -0.5]
    # up  [[1, 2], [3, -1]]: [1 - 1, 3 + 0.5] = [0, 3.5] -> relu^2 = [0, 12.25]
    # down [[1, 1], [0.5, -1]]: [12.25, -12.25]; rsf 2 (k = 1, weight = rsf)
    #   routed = [24.5, -24.5]
    # shared up [[1, 1], [2, 0]]: [0.5, 2] -> relu^2 [0.25, 4]
    # shared down [[2, 3], [1, 1]]: [0.5 + 12, 0.25 + 4] = [12.5, 4.25]
    # out = x + routed + shared = [38, -21.25]
    inp = custom_inputs(2, 1, 1, 2, 2, rsf=2.0, eps=0.0, norm_w=[1, 0.5], gate_w=[0.5, 0.5],
                        up_w=[[1, 2], [3, -1]], down_w=[[1, 1], [0.5, -1]],
                        shared_up_w=[[1, 1], [2, 0]], shared_down_w=[[2, 3], [1, 1]],
                        hidden=[[1, -1]])
    out, idx, w = oracle.Oracle(inp).forward(inp.hidden)
    np.testing.assert_array_equal(out, [[38.0, -21.25]])
    np.testing.assert_array_equal(idx, [[0]])
    np.testing.assert_array_equal(w, [[2.0]])


def test_hand_case_gate_picks_expert():
    # n = [1, -0.5]; G = [[0, 4], [-3, 0]] -> logits [-2, -3] -> expert 0 (k=1)
    # (a transposed gate gives logits [1.5, 4] and would pick expert 1)
    # expert 0: up [[2, 2], [1, 0]] -> [1, 1] -> relu^2 [1, 1];
    #           down [[1, -1], [3, 0.5]] -> [0, 3.5]; rsf 0.5 -> [0, 1.75]
    # expert 1 (identity up and down) would give [0.5, 0]
    # shared expert zero.  out = [1, -1] + [0, 1.75] = [1, 0.75]
    inp = custom_inputs(2, 2, 1, 2, 2, rsf=0.5, eps=0.0, norm_w=[1, 0.5],
                        gate_w=[[0, 4], [-3, 0]],
                        up_w=[[[2, 2], [1, 0]], [[1, 0], [0, 1]]],
                        down_w=[[[1, -1], [3, 0.5]], [[1, 0], [0, 1]]],
                        shared_up_w=np.zeros((2, 2)), shared_down_w=np.zeros((2, 2)),
                        hidden=[[1, -1]])
    out, idx, _ = oracle.Oracle(inp).forward(inp.hidden)
    np.testing.assert_array_equal(idx, [[0]])
    np.testing.assert_array_equal(out, [[1.0, 0.75]])


def test_hand_case_latent():
    # n = [1, -0.5]; fc1 [[2, 1], [0, 1]] -> z = [1.5, -0.5]
    # up [[2, 1]] -> 2.5 -> relu^2 6.25; down [[1], [-2]] -> [6.25, -12.5]
    # fc2 [[1, 0.5], [0, 1]] -> [0, -12.5]
    # shared up [[1, -2]] -> 2 -> 4; shared down [[0.25], [1]] -> [1, 4]
    # out = [1, -1] + [0, -12.5] + [1, 4] = [2, -9.5]
    inp = custom_inputs(2, 1, 1, 1, 1, L=2, rsf=1.0, eps=0.0, norm_w=[1, 0.5], gate_w=[1, 1],
                        up_w=[2, 1], down_w=[1, -2], shared_up_w=[1, -2],
                        shared_down_w=[0.25, 1], fc1_w=[[2, 1], [0, 1]],
                        fc2_w=[[1, 0.5], [0, 1]], hidden=[[1, -1]])
    out, _, _ = oracle.Oracle(inp).forward(inp.hidden)
    np.testing.assert_array_equal(out, [[2.0, -9.5]])


# ------------------------------------------------- reductions, invariants ---

def _tiny(**kw):
    return make_inputs(WORKLOADS["tiny"].scaled(**kw))


def test_latent_with_identity_projections_is_direct():
    d = _tiny(T=6)
    s = d.shape
    eye = np.eye(s.H)
    lat = custom_inputs(s.H, s.E, s.k, s.I, s.S, L=s.H, rsf=s.rsf, eps=s.eps,
                        norm_w=np.zeros(s.H), gate_w=np.zeros(s.E * s.H), up_w=np.zeros(s.E * s.I * s.H),
                        down_w=np.zeros(s.E * s.H * s.I), shared_up_w=np.zeros(s.S * s.H),
                        shared_down_w=np.zeros(s.H * s.S), fc1_w=eye, fc2_w=eye,
                        hidden=np.zeros((6, s.H)))
    for name in ("norm_w", "gate_w", "up_w", "down_w", "shared_up_w", "shared_down_w", "hidden"):
        setattr(lat, name, getattr(d, name))
    o_d, i_d, _ = oracle.Oracle(d).forward(d.hidden)
    o_l, i_l, _ = oracle.Oracle(lat).forward(lat.hidden)
    np.testing.assert_array_equal(i_d, i_l)
    np.testing.assert_array_equal(o_d, o_l)


def test_fp8_weights_equal_bf16_when_dequantised_values_are_exact():
    # E4M3 codes times power-of-two row scales are exact in BF16, so the FP8
    # oracle must reproduce the BF16 oracle on those dequantised values.
    d = _tiny(T=5)
    s = d.shape
    rng = np.random.default_rng(3)
    codes = np.array([c for c in range(256) if (c & 0x7F) not in (0x7F,)], dtype=np.uint8)

    def q(shape):
        return rng.choice(codes, size=shape).astype(np.uint8)

    from workloads import e4m3_to_f32
    up_q, down_q = q(d.up_w.shape), q(d.down_w.shape)
    up_s = (2.0 ** -rng.integers(4, 9, size=(s.E, s.I))).astype(np.float32)
    down_s = (2.0 ** -rng.integers(4, 9, size=(s.E, s.H))).astype(np.float32)
    f8 = make_inputs(s.scaled(expert_fp8=True))
    for name in ("norm_w", "gate_w", "gate_bias", "shared_up_w", "shared_down_w", "hidden"):
        setattr(f8, name, getattr(d, name))
    f8.up_w, f8.down_w, f8.up_scale, f8.down_scale = up_q, down_q, up_s, down_s
    d.up_w = exact_bf16(e4m3_to_f32(up_q).astype(np.float64) * up_s[..., None])
    d.down_w = exact_bf16(e4m3_to_f32(down_q).astype(np.float64) * down_s[..., None])
    o8, i8, _ = oracle.Oracle(f8).forward(f8.hidden)
    ob, ib, _ = oracle.Oracle(d).forward(d.hidden)
    np.testing.assert_array_equal(i8, ib)
    np.testing.assert_array_equal(o8, ob)


def test_zero_weight_expert_contributes_nothing():
    # An expert whose gate logit is below -800 has score 1/(1+exp(800)) == 0
    # in float64, so its routing weight is exactly 0 and its weights cannot
    # matter.  Gate row of the dead expert: -128 * sign(n) of the token.
    d = _tiny(T=1)
    s = d.shape
    dead = s.E - 1
    n = oracle.Oracle(d).rmsnorm(d.hidden)
    d.gate_w = d.gate_w.reshape(s.E, s.H).copy()
    d.gate_w[dead] = exact_bf16(-np.sign(n[0]) * 128.0)
    lg = oracle.Oracle(d).gate_logits(d.hidden)
    assert lg[0, dead] < -800
    forced = np.array([[0, dead]], dtype=np.int32)
    out1, _, w1 = oracle.Oracle(d).forward(d.hidden, forced_idx=forced)
    assert w1[0, 1] == 0.0 and w1[0, 0] == s.rsf
    d.down_w = d.down_w.copy()
    d.down_w[dead] = exact_bf16(np.full(d.down_w[dead].shape, 3.0))
    d.up_w = d.up_w.copy()
    d.up_w[dead] = exact_bf16(np.full(d.up_w[dead].shape, 1.0))
    out2, _, _ = oracle.Oracle(d).forward(d.hidden, forced_idx=forced)
    np.testing.assert_array_equal(out1, out2)


def test_routed_part_is_linear_in_scaling_factor():
    d1, d2 = _tiny(T=8, rsf=1.0), _tiny(T=8, rsf=2.5)
    z = _tiny(T=8, rsf=1.0)
    z.down_w = np.zeros_like(z.down_w)          # routed part removed
    o1, i1, _ = oracle.Oracle(d1).forward(d1.hidden)
    o2, i2, _ = oracle.Oracle(d2).forward(d2.hidden)
    oz, _, _ = oracle.Oracle(z).forward(z.hidden)
    np.testing.assert_array_equal(i1, i2)
    np.testing.assert_allclose(o2 - oz, 2.5 * (o1 - oz), rtol=1e-12, atol=1e-12)


def test_shared_and_routed_parts_add():
    base = _tiny(T=8)
    no_shared = _tiny(T=8)
    no_shared.shared_down_w = np.zeros_like(no_shared.shared_down_w)
    no_routed = _tiny(T=8)
    no_routed.down_w = np.zeros_like(no_routed.down_w)
    from workloads import bf16_to_f32
    x = bf16_to_f32(base.hidden).astype(np.float64)
    o, _, _ = oracle.Oracle(base).forward(base.hidden)
    a, _, _ = oracle.Oracle(no_shared).forward(no_shared.hidden)
    b, _, _ = oracle.Oracle(no_routed).forward(no_routed.hidden)
    np.testing.assert_allclose(o, a + b - x, rtol=1e-12, atol=1e-12)


def test_tokens_are_independent_and_threading_is_exact():
    d = _tiny(T=16)
    o = oracle.Oracle(d)
    out1, idx1, w1 = o.forward(d.hidden, nthreads=1)
    out8, idx8, w8 = o.forward(d.hidden, nthreads=8)
    np.testing.assert_array_equal(out1, out8)
    p = np.random.default_rng(0).permutation(16)
    outp, idxp, _ = o.forward(d.hidden[p], nthreads=3)
    np.testing.assert_array_equal(outp, out1[p])
    np.testing.assert_array_equal(idxp, idx1[p])
    # one token at a time gives the same rows
    for t in (0, 7, 15):
        ot, _, _ = o.forward(d.hidden[t:t + 1])
        np.testing.assert_array_equal(ot[0], out1[t])


def test_forced_routing_recomputes_weights_from_scores():
    d = _tiny(T=4, rsf=2.0)
    o = oracle.Oracle(d)
    lg = o.gate_logits(d.hidden)
    forced = np.array([[3, 1], [0, 7], [5, 2], [6, 4]], dtype=np.int32)
    _, idx, w = o.forward(d.hidden, forced_idx=forced)
    np.testing.assert_array_equal(idx, forced)
    s = 1.0 / (1.0 + np.exp(-np.take_along_axis(lg, forced, axis=1)))
    np.testing.assert_allclose(w, 2.0 * s / s.sum(axis=1, keepdims=True), rtol=1e-14)


def test_route_weights_of_forced_sets_match_the_scores():
    # the weights of a given expert set: rsf * sigmoid(logit_e) / sum over
    # the set, in the set's own slot order; forward with the same forced
    # sets reports the same weights
    d = _tiny(T=4, rsf=2.5)
    o = oracle.Oracle(d)
    lg = o.gate_logits(d.hidden)
    forced = np.array([[6, 2], [1, 0], [7, 3], [4, 5]], dtype=np.int32)
    w = o.route_weights(lg, forced)
    s = 1.0 / (1.0 + np.exp(-np.take_along_axis(lg, forced, axis=1)))
    np.testing.assert_allclose(w, 2.5 * s / s.sum(axis=1, keepdims=True), rtol=1e-14)
    _, _, fw = o.forward(d.hidden, forced_idx=forced)
    np.testing.assert_array_equal(w, fw)
    # the oracle's own choice gives its own weights
    idx, ow, _ = o.route(lg)
    np.testing.assert_array_equal(o.route_weights(lg, idx), ow)


@pytest.mark.parametrize("which", ["shared", "latent"])
def test_fp8_dense_weights_equal_bf16_when_dequantised_values_are_exact(which):
    # Shared expert (up, down) or LatentMoE fc1 / fc2 stored as E4M3 codes
    # with power-of-two row scales: the dequantised values are exact in
    # BF16, so the FP8 oracle must reproduce the BF16 oracle run on them.
    # A missing row scale or a transposed scale index changes the result.
    from workloads import e4m3_to_f32
    base = WORKLOADS["tiny"].scaled(T=6, L=64 if which == "latent" else 0)
    d = make_inputs(base)
    rng = np.random.default_rng(11)
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    names = ("shared_up", "shared_down") if which == "shared" else ("fc1", "fc2")
    f8 = make_inputs(base.scaled(**{f"{which}_fp8": True}))
    for name in ("norm_w", "gate_w", "gate_bias", "up_w", "down_w", "hidden",
                 "shared_up_w", "shared_down_w", "fc1_w", "fc2_w"):
        setattr(f8, name, getattr(d, name))
    for n in names:
        w = getattr(d, f"{n}_w")
        qc = rng.choice(codes, size=w.shape).astype(np.uint8)
        sc = (2.0 ** -rng.integers(3, 8, size=w.shape[0])).astype(np.float32)
        setattr(f8, f"{n}_w", qc)
        setattr(f8, f"{n}_scale", sc)
        setattr(d, f"{n}_w", exact_bf16(e4m3_to_f32(qc).astype(np.float64) * sc[:, None]))
    o8, i8, _ = oracle.Oracle(f8).forward(f8.hidden)
    ob, ib, _ = oracle.Oracle(d).forward(d.hidden)
    np.testing.assert_array_equal(i8, ib)
    np.testing.assert_array_equal(o8, ob)
    # and the FP8 weights do matter: a changed row scale changes the output
    sc = getattr(f8, f"{names[1]}_scale").copy()
    sc[0] *= 2.0
    setattr(f8, f"{names[1]}_scale", sc)
    o8b, _, _ = oracle.Oracle(f8).forward(f8.hidden)
    assert not np.array_equal(o8b, o8)

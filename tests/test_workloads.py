"""The seeded input recipe on CPU: determinism, the token-prefix property,
the value distributions each array is drawn from, the FP8 storage format,
and the stored Zipf calibration of the skewed workload (re-derived with the
oracle's routing)."""
import dataclasses
import json
import os

import numpy as np
import pytest

import oracle
from workloads import WORKLOADS, bf16_to_f32, e4m3_to_f32, make_inputs, skew_alpha

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _arrays(inp):
    return {f.name: getattr(inp, f.name) for f in dataclasses.fields(inp) if f.name != "shape"}


def test_same_seed_gives_the_same_bits():
    a, b = make_inputs(WORKLOADS["tiny"]), make_inputs(WORKLOADS["tiny"])
    for name, x in _arrays(a).items():
        y = getattr(b, name)
        assert (x is None) == (y is None), name
        if x is not None:
            assert x.dtype == y.dtype and np.array_equal(x, y), name


def test_other_seed_gives_other_bits():
    a = make_inputs(WORKLOADS["tiny"])
    b = make_inputs(WORKLOADS["tiny"].scaled(seed=7))
    assert not np.array_equal(a.hidden, b.hidden)
    assert not np.array_equal(a.up_w, b.up_w)


def test_fewer_tokens_give_a_prefix():
    s = WORKLOADS["decode"].scaled(H=512, I=128, S=256, E=16)
    a = make_inputs(s, T=2, experts=False)
    b = make_inputs(s, T=8, experts=False)
    assert np.array_equal(a.hidden, b.hidden[:2])
    assert np.array_equal(a.residual, b.residual[:2])
    assert np.array_equal(a.gate_w, b.gate_w) and np.array_equal(a.gate_bias, b.gate_bias)


def _std(bits):
    return float(np.std(bf16_to_f32(bits).astype(np.float64)))


def test_value_distributions():
    s = WORKLOADS["decode"].scaled(T=64, H=512, I=256, S=384, E=16)
    inp = make_inputs(s)
    H, I, S = s.H, s.I, s.S
    # weights ~ N(0, 1/fan_in), fan_in = the input width of each matrix
    for bits, fan_in in ((inp.gate_w, H), (inp.up_w, H), (inp.down_w, I),
                         (inp.shared_up_w, H), (inp.shared_down_w, S)):
        assert _std(bits) == pytest.approx(1 / np.sqrt(fan_in), rel=0.03)
        assert abs(float(np.mean(bf16_to_f32(bits)))) < 3 / np.sqrt(fan_in) / np.sqrt(bits.size)
    assert inp.up_w.shape == (s.E, I, H) and inp.down_w.shape == (s.E, H, I)
    # tokens ~ N(0, 1); the norm weight ~ U(0.5, 1.5); the uniform bias ~ U(-0.1, 0.1)
    assert _std(inp.hidden) == pytest.approx(1.0, rel=0.03)
    g = bf16_to_f32(inp.norm_w)
    assert g.min() >= 0.5 and g.max() <= 1.5 and abs(g.mean() - 1.0) < 0.05
    b = inp.gate_bias
    assert b.dtype == np.float32 and b.min() >= -0.1 and b.max() <= 0.1
    assert WORKLOADS["prefill"].bias == "none" and WORKLOADS["latent"].bias == "none"


def test_latent_projection_shapes_and_scale():
    s = WORKLOADS["latent"].scaled(T=8, H=512, I=128, S=256, L=128, E=8)
    inp = make_inputs(s)
    assert inp.fc1_w.shape == (s.L, s.H) and inp.fc2_w.shape == (s.H, s.L)
    assert inp.up_w.shape == (s.E, s.I, s.L) and inp.down_w.shape == (s.E, s.L, s.I)
    assert _std(inp.fc1_w) == pytest.approx(1 / np.sqrt(s.H), rel=0.05)
    assert _std(inp.fc2_w) == pytest.approx(1 / np.sqrt(s.L), rel=0.05)


def test_fp8_rows_span_the_e4m3_range():
    s = WORKLOADS["skew_fp8"].scaled(T=4, H=512, I=256, S=256, E=4)
    inp = make_inputs(s)
    for q, sc, fan_in in ((inp.up_w, inp.up_scale, s.H), (inp.down_w, inp.down_scale, s.I)):
        assert q.dtype == np.uint8 and sc.dtype == np.float32 and sc.shape == q.shape[:2]
        v = e4m3_to_f32(q).astype(np.float64)
        assert np.all(np.isfinite(v))
        # scale = row amax / 448: every row's largest code is +-448 exactly
        assert np.array_equal(np.abs(v).max(axis=-1), np.full(q.shape[:2], 448.0))
        deq = v * sc[..., None]
        assert float(np.std(deq)) == pytest.approx(1 / np.sqrt(fan_in), rel=0.05)


def test_zipf_bias_profile():
    s = WORKLOADS["skew_fp8"]
    b = make_inputs(s, T=1, experts=False).gate_bias.astype(np.float64)
    a = skew_alpha()
    with open(os.path.join(ROOT, "tests", "golden", "skew_alpha.json")) as f:
        assert a == json.load(f)["alpha"]
    ranks = np.arange(1, s.E + 1)
    np.testing.assert_allclose(np.sort(b)[::-1], -a * 1.1 * np.log(ranks), rtol=1e-6, atol=1e-7)


def test_zipf_calibration_reproduces_with_the_oracle():
    """The stored scale gives the hottest expert 20x the mean token count
    when the workload's 8192 tokens are routed by the oracle."""
    s = WORKLOADS["skew_fp8"]
    inp = make_inputs(s, experts=False)
    z = np.zeros(1, dtype=np.uint16)
    view = dataclasses.replace(inp, shape=s.scaled(expert_fp8=False), up_w=z, down_w=z,
                               shared_up_w=z, shared_down_w=z)
    o = oracle.Oracle(view)
    idx, _, _ = o.route(o.gate_logits(inp.hidden))
    cnt = np.bincount(idx.reshape(-1), minlength=s.E)
    assert cnt.sum() == s.T * s.k
    assert cnt.max() / (s.T * s.k / s.E) == pytest.approx(20.0, abs=0.05)

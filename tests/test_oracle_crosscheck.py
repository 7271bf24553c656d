"""Cross-check of the C++ oracle against an independent NumPy float64
restatement of the layer (written from the layer's definition, not from
the oracle's code): matching results rule out coding slips in either (an
index, a transposed operand, a loop bound).  This is a check of the
implementation, not a pin of the definition; the definition is pinned by
tests/test_oracle_pins.py.
"""
import numpy as np
import pytest

import oracle
from workloads import WORKLOADS, bf16_to_f32, e4m3_to_f32, make_inputs


def _f64_bf16(bits):
    return bf16_to_f32(bits).astype(np.float64)


def numpy_layer(inp, hidden_bits):
    """(out [T,H] f64, idx [T,k], w [T,k]) of the layer, all in float64."""
    s = inp.shape
    T, E, k = hidden_bits.shape[0], s.E, s.k
    x = _f64_bf16(hidden_bits)
    n = x / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + s.eps) * _f64_bf16(inp.norm_w)
    score = 1.0 / (1.0 + np.exp(-(n @ _f64_bf16(inp.gate_w).T)))
    bias = np.zeros(E) if inp.gate_bias is None else inp.gate_bias.astype(np.float64)
    key = score + bias
    # k largest keys, lower expert index first among equal keys
    idx = np.stack([np.lexsort((np.arange(E), -key[t]))[:k] for t in range(T)])
    sel = np.take_along_axis(score, idx, axis=1)
    w = s.rsf * sel / sel.sum(axis=1, keepdims=True)

    def expert(m, scale):  # weights of one expert as float64 [out, in]
        if s.expert_fp8:
            return e4m3_to_f32(m).astype(np.float64) * scale[:, None]
        return _f64_bf16(m)

    def dense(m, scale, fp8):  # shared expert / fc1 / fc2 weights as float64 [out, in]
        return e4m3_to_f32(m).astype(np.float64) * scale[:, None] if fp8 else _f64_bf16(m)

    z = n if not s.L else n @ dense(inp.fc1_w, inp.fc1_scale, s.latent_fp8).T
    m = np.zeros_like(z)
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            up = expert(inp.up_w[e], None if inp.up_scale is None else inp.up_scale[e])
            dn = expert(inp.down_w[e], None if inp.down_scale is None else inp.down_scale[e])
            u = np.maximum(up @ z[t], 0.0) ** 2
            m[t] += w[t, j] * (dn @ u)
    if s.L:
        m = m @ dense(inp.fc2_w, inp.fc2_scale, s.latent_fp8).T
    v = np.maximum(n @ dense(inp.shared_up_w, inp.shared_up_scale, s.shared_fp8).T, 0.0) ** 2
    return x + m + v @ dense(inp.shared_down_w, inp.shared_down_scale, s.shared_fp8).T, idx, w


@pytest.mark.parametrize("name,T,over", [
    ("tiny", 16, {}),
    ("decode", 8, {}),
    ("latent", 6, dict(H=512, I=256, S=512, L=256)),
    ("skew_fp8", 8, dict(H=512, I=256, S=512, E=32)),
    ("skew_fp8", 8, dict(H=512, I=256, S=512, E=32, shared_fp8=True)),
    ("latent", 6, dict(H=512, I=256, S=512, L=256, shared_fp8=True, latent_fp8=True)),
])
def test_oracle_matches_numpy_restatement(name, T, over):
    shape = WORKLOADS[name].scaled(**over) if over else WORKLOADS[name]
    inp = make_inputs(shape, T=T)
    h = inp.hidden[:T]
    out_o, idx_o, w_o = oracle.Oracle(inp).forward(h)
    out_n, idx_n, w_n = numpy_layer(inp, h)
    assert np.array_equal(idx_o, idx_n)
    np.testing.assert_allclose(w_o, w_n, rtol=1e-12, atol=0)
    scale = np.max(np.abs(out_n))
    np.testing.assert_allclose(out_o, out_n, rtol=0, atol=1e-12 * scale)

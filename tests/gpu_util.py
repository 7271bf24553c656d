"""Helpers for the GPU parity tests: run the library through its C ABI and
compare with the CPU oracle (no layer arithmetic here)."""
from __future__ import annotations

import numpy as np

import oracle
from tests.helpers import check_output
from workloads import bf16_to_f32

TIE_WINDOW = 1e-5  # routing sets may differ only where the oracle's k-th and (k+1)-th keys are this close


def to_dev(a, dtype=np.int16):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(dtype)).cuda()


def run_forward(layer, hidden_bits, path, residual_bits=None):
    """Returns (out f32 [T,H], residual_out bits [T,H], idx [T,k], w [T,k])."""
    import torch
    T = hidden_bits.shape[0]
    k = layer.cfg.top_k
    hid = to_dev(hidden_bits)
    res = to_dev(residual_bits if residual_bits is not None
                 else np.full_like(hidden_bits, 0x7FC0))          # NaN fill: must be ignored
    layer.forward(hid, res, path=path)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    layer.copy_routing(idx, w)
    torch.cuda.synchronize()
    out = bf16_to_f32(hid.cpu().numpy().view(np.uint16))
    return out, res.cpu().numpy().view(np.uint16), idx.cpu().numpy(), w.cpu().numpy()


def check_routing(orc: oracle.Oracle, hidden_bits, gpu_idx, gpu_w, rows=None):
    """Routing sets equal the oracle's except inside the tie window; weights of
    the GPU's set match the oracle's weights for that set.  Returns the number
    of tokens routed differently (all inside the window)."""
    rows = np.arange(hidden_bits.shape[0]) if rows is None else np.asarray(rows)
    s = orc.shape
    logits = orc.gate_logits(hidden_bits[rows])
    oidx, _, keys = orc.route(logits)
    flips = 0
    for n, t in enumerate(rows):
        g = gpu_idx[t]
        assert len(set(g.tolist())) == s.k and g.min() >= 0 and g.max() < s.E, (t, g)
        if set(g.tolist()) != set(oidx[n].tolist()):
            kk = np.sort(keys[n])[::-1]
            gap = kk[s.k - 1] - kk[s.k]
            assert gap < TIE_WINDOW, f"token {t}: routing differs with key gap {gap}"
            flips += 1
    # weights of the GPU's chosen set, recomputed by the oracle
    _, _, fw = orc.forward(hidden_bits[rows[:64]], forced_idx=gpu_idx[rows[:64]])
    np.testing.assert_allclose(gpu_w[rows[:64]], fw, rtol=2e-5, atol=2e-6 * s.rsf)
    np.testing.assert_allclose(gpu_w[rows].sum(axis=1), s.rsf, rtol=1e-5)
    return flips


def check_layer(orc: oracle.Oracle, hidden_bits, out, gpu_idx, rows, expert_fp8=False):
    """Layer output on `rows` against the oracle run with the GPU's routing
    (identical to the oracle's own except for tie-window tokens)."""
    rows = np.asarray(rows)
    ref, _, _ = orc.forward(hidden_bits[rows], forced_idx=gpu_idx[rows])
    err, bound = check_output(out[rows], ref, expert_fp8)
    assert np.all(np.isfinite(out[rows]))
    assert err <= bound, f"max|gpu - oracle| = {err:.4g} > bound {bound:.4g}"
    return err, bound


def sample_rows(T, n, seed=0):
    """First, last, tile-boundary and random rows (sorted, unique)."""
    rng = np.random.default_rng(seed)
    fixed = [0, 1, T - 1] + [r for r in (127, 128, 129, 255, 256, T // 2) if r < T]
    extra = rng.choice(T, size=min(n, T), replace=False).tolist()
    return np.array(sorted(set(fixed + extra)))

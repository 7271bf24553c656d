"""Helpers for the GPU parity tests: run the library through its C ABI and
compare with the CPU oracle (no layer arithmetic here)."""
from __future__ import annotations

import numpy as np

import oracle
from tests.helpers import check_output
from workloads import bf16_to_f32

TIE_WINDOW = 1e-5  # routing sets may differ only where the oracle's k-th and (k+1)-th keys are this close

# Routing report, printed at the end of the pytest run (tests/conftest.py):
# case -> (tokens checked, tokens routed differently from the oracle, tokens
# whose k-th and (k+1)-th oracle keys lie inside the tie window).
ROUTING_REPORT = {}


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


def check_routing(orc: oracle.Oracle, hidden_bits, gpu_idx, gpu_w, rows=None, case=None):
    """Routing sets equal the oracle's except inside the tie window, and the
    GPU's weights equal the oracle's weights of the GPU's own set, on every
    row checked.  Returns the number of tokens routed differently (all inside
    the window); with `case` the counts go into ROUTING_REPORT."""
    rows = np.arange(hidden_bits.shape[0]) if rows is None else np.asarray(rows)
    s = orc.shape
    logits = orc.gate_logits(hidden_bits[rows])
    oidx, _, keys = orc.route(logits)
    g = gpu_idx[rows]
    assert g.min() >= 0 and g.max() < s.E, "expert id out of range"
    gs = np.sort(g, axis=1)
    assert np.all(gs[:, 1:] != gs[:, :-1]), "an expert chosen twice for one token"
    kk = -np.sort(-keys, axis=1)
    gap = kk[:, s.k - 1] - kk[:, s.k] if s.k < s.E else np.full(len(rows), np.inf)
    differ = np.any(gs != np.sort(oidx, axis=1), axis=1)
    bad = differ & ~(gap < TIE_WINDOW)
    assert not bad.any(), (f"tokens {rows[bad][:8].tolist()} routed differently with key gaps "
                           f"{gap[bad][:8].tolist()}")
    # weights of the GPU's chosen set, recomputed by the oracle, every row
    fw = orc.route_weights(logits, g)
    np.testing.assert_allclose(gpu_w[rows], fw, rtol=2e-5, atol=2e-6 * s.rsf)
    np.testing.assert_allclose(gpu_w[rows].sum(axis=1), s.rsf, rtol=1e-5)
    flips = int(differ.sum())
    if case is not None:
        ROUTING_REPORT[case] = (len(rows), flips, int((gap < TIE_WINDOW).sum()))
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


def check_forward_sort(layer, gpu_idx, E):
    """The forward pass's own sort by expert (perm, inv, off) equals the
    oracle's counting sort of the routing that pass used, bit for bit."""
    import torch
    T, k = gpu_idx.shape
    R = T * k
    perm = torch.full((R,), -7, dtype=torch.int32, device="cuda")
    inv = torch.full((R,), -7, dtype=torch.int32, device="cuda")
    off = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    layer.copy_sort(perm, inv, off, T)
    torch.cuda.synchronize()
    perm_o, inv_o, off_o = oracle.sort(gpu_idx, E)
    assert np.array_equal(off.cpu().numpy(), off_o)
    assert np.array_equal(perm.cpu().numpy(), perm_o)
    assert np.array_equal(inv.cpu().numpy(), inv_o)

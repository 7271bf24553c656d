"""Writes tests/golden/skew_alpha.json: the Zipf gate-bias scale of the skewed
FP8 workload (T=8192, H=2688, E=128, top_k=6).

The workload asks for a Zipf(s=1.1) bias profile over a random expert
permutation, scaled so the hottest expert receives about 20x the mean token
count.  This script routes the workload's tokens with the CPU oracle only
(norm, gate, sigmoid top-k) and bisects on the scale alpha of
bias[rank r] = -alpha * 1.1 * ln(r) until max_e count_e / (T*k/E) is 20.

Run:  python tests/golden/calibrate_skew.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from workloads import WORKLOADS, make_inputs  # noqa: E402

TARGET = 20.0


def skew_of(o, logits, bias, s):
    idx, _, _ = o.route(logits, bias=bias)
    cnt = np.bincount(idx.reshape(-1), minlength=s.E)
    return cnt.max() / (s.T * s.k / s.E)


def main():
    s = WORKLOADS["skew_fp8"]
    inp = make_inputs(s, alpha=1.0, experts=False)
    # the oracle only needs the routing arrays; give it the bf16 path
    o = oracle.Oracle(_routing_view(inp))
    logits = o.gate_logits(inp.hidden)
    unit = inp.gate_bias.astype(np.float64)           # bias at alpha = 1
    lo, hi = 0.0, 4.0
    for _ in range(60):
        mid = 0.5 * (lo + hi)
        if skew_of(o, logits, (mid * unit).astype(np.float32), s) < TARGET:
            lo = mid
        else:
            hi = mid
    alpha = hi
    bias = make_inputs(s, T=1, alpha=alpha, experts=False).gate_bias
    ratio = skew_of(o, logits, bias, s)
    out = {"alpha": alpha, "hottest_over_mean": float(ratio), "target": TARGET,
           "workload": "skew_fp8 T=8192 H=2688 E=128 k=6 seed 4",
           "written_by": "tests/golden/calibrate_skew.py (CPU oracle routing only)"}
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "skew_alpha.json"), "w") as f:
        json.dump(out, f, indent=1)
    print(out)


def _routing_view(inp):
    import dataclasses
    z = np.zeros(1, dtype=np.uint16)
    return dataclasses.replace(inp, shape=inp.shape.scaled(expert_fp8=False), up_w=z, down_w=z,
                               shared_up_w=z, shared_down_w=z)


if __name__ == "__main__":
    main()

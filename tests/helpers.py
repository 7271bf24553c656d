"""Shared test helpers: hand-built inputs and tolerance checks (no layer math)."""
from __future__ import annotations

import numpy as np

from workloads import Inputs, MoEShape, bf16_bits, bf16_to_f32


def exact_bf16(a) -> np.ndarray:
    """float values -> bf16 bits, asserting each value is exactly representable."""
    a = np.asarray(a, dtype=np.float64)
    b = bf16_bits(a.astype(np.float32))
    assert np.array_equal(bf16_to_f32(b).astype(np.float64), a), "value not exact in bf16"
    return b


def custom_inputs(H, E, k, I, S, L=0, rsf=1.0, eps=0.0, *, norm_w, gate_w, up_w, down_w,
                  shared_up_w, shared_down_w, hidden, fc1_w=None, fc2_w=None,
                  gate_bias=None) -> Inputs:
    """Inputs from explicit float matrices (all exactly representable in bf16)."""
    hidden = np.atleast_2d(np.asarray(hidden, dtype=np.float64))
    shape = MoEShape("custom", T=hidden.shape[0], H=H, E=E, k=k, I=I, S=S, L=L,
                     rsf=rsf, eps=eps)
    return Inputs(
        shape=shape,
        norm_w=exact_bf16(norm_w),
        gate_w=exact_bf16(np.reshape(gate_w, (E, H))),
        gate_bias=None if gate_bias is None else np.asarray(gate_bias, dtype=np.float32),
        up_w=exact_bf16(np.reshape(up_w, (E, I, L or H))),
        down_w=exact_bf16(np.reshape(down_w, (E, L or H, I))),
        up_scale=None, down_scale=None,
        shared_up_w=exact_bf16(np.reshape(shared_up_w, (S, H))),
        shared_down_w=exact_bf16(np.reshape(shared_down_w, (H, S))),
        fc1_w=None if fc1_w is None else exact_bf16(np.reshape(fc1_w, (L, H))),
        fc2_w=None if fc2_w is None else exact_bf16(np.reshape(fc2_w, (H, L))),
        hidden=exact_bf16(hidden),
        residual=exact_bf16(np.zeros_like(hidden)),
    )


def output_tolerance(expert_fp8: bool) -> float:
    """Relative coefficient c of the layer-output bound c*max|oracle| + 1e-3."""
    return 5e-2 if expert_fp8 else 1e-2


def check_output(gpu_out: np.ndarray, oracle_out: np.ndarray, expert_fp8: bool):
    """max|gpu - oracle| <= c*max|oracle| + 1e-3 over the whole output."""
    err = float(np.max(np.abs(gpu_out.astype(np.float64) - oracle_out)))
    bound = output_tolerance(expert_fp8) * float(np.max(np.abs(oracle_out))) + 1e-3
    return err, bound

"""Seeded synthetic inputs for the Nemotron-H MoE FFN layer.

This module only draws random numbers and stores them in the layer's storage
formats (BF16 bits, FP8 E4M3 bits plus an FP32 per-row scale).  It holds none
of the layer's arithmetic: no norm, gate, routing, expert or reduction math.
Both the CPU oracle and the CUDA library consume exactly the arrays produced
here, so the two sides see bit-identical inputs.

Shapes follow the layer as described on the NemotronMoeLayer pages
(nemotron_moe.rs, module documentation): hidden ``[T, H]``; gate ``[E, H]``;
routed expert up ``[E, I, D]`` and down ``[E, D, I]`` where ``D = H`` for the
direct layer and ``D = L`` (``moe_latent_size``) for LatentMoE; shared expert
up ``[S, H]`` and down ``[H, S]``; latent fc1 ``[L, H]`` and fc2 ``[H, L]``.
Every weight is stored ``[out, in]`` (row-major, ``in`` contiguous).

Streams: the workload seed is split (numpy SeedSequence.spawn) into one
independent PCG64 stream per array, in this fixed order: norm_w, gate_w,
gate_bias, up, down, shared_up, shared_down, fc1, fc2, hidden, residual; the
up and down streams are split once more, one child per expert.  Any array can therefore be drawn without the
others, and a smaller token count gives a prefix of a larger one.
"""
from __future__ import annotations

import dataclasses
import json
import os
from typing import Dict, Optional

import numpy as np

__all__ = ["MoEShape", "WORKLOADS", "Inputs", "make_inputs", "bf16_bits",
           "bf16_to_f32", "e4m3_to_f32", "skew_alpha"]


@dataclasses.dataclass(frozen=True)
class MoEShape:
    """One synthetic workload: layer sizes plus the recipe for its values."""
    name: str
    T: int            # tokens
    H: int            # hidden size
    E: int            # routed experts
    k: int            # experts per token (top_k)
    I: int            # routed-expert intermediate size (moe_inter)
    S: int            # shared-expert intermediate size
    L: int = 0        # moe_latent_size (0 = direct layer)
    rsf: float = 1.0  # routed_scaling_factor
    eps: float = 1e-5
    expert_fp8: bool = False   # routed up/down stored as FP8 E4M3 + FP32 row scale
    shared_fp8: bool = False   # shared expert up/down stored the same way
    latent_fp8: bool = False   # fc1 / fc2 stored the same way
    bias: str = "none"         # "none" | "uniform" (U(-0.1,0.1)) | "zipf"
    gate_scale: float = 1.0    # gate ~ N(0, gate_scale / H)
    seed: int = 0

    @property
    def D(self) -> int:
        """Width the routed experts work on: H (direct) or L (LatentMoE)."""
        return self.L if self.L > 0 else self.H

    def with_tokens(self, T: int) -> "MoEShape":
        return dataclasses.replace(self, T=T)

    def scaled(self, **kw) -> "MoEShape":
        return dataclasses.replace(self, **kw)


# The five workloads.  Where a workload's description is silent: rsf is 2.5
# for the three Nemotron-H-sized direct layers (decode, prefill, skew_fp8) and
# 1.0 for tiny and latent; the selection bias is zero unless given (uniform
# for decode, Zipf for skew_fp8); the latent layer's shared expert works on
# the hidden width H.
WORKLOADS: Dict[str, MoEShape] = {
    "tiny": MoEShape("tiny", T=16, H=256, E=8, k=2, I=128, S=256, L=0,
                     rsf=1.0, bias="none", seed=0),
    "decode": MoEShape("decode", T=8, H=2688, E=128, k=6, I=1856, S=3712,
                       L=0, rsf=2.5, bias="uniform", seed=1),
    "prefill": MoEShape("prefill", T=1024, H=2688, E=128, k=6, I=1856,
                        S=3712, L=0, rsf=2.5, bias="none", seed=2),
    "latent": MoEShape("latent", T=4096, H=4096, E=128, k=8, I=2688, S=5376,
                       L=1024, rsf=1.0, bias="none", seed=3),
    "skew_fp8": MoEShape("skew_fp8", T=8192, H=2688, E=128, k=6, I=1856,
                         S=3712, L=0, rsf=2.5, expert_fp8=True, bias="zipf",
                         seed=4),
}

_GOLDEN = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                       "tests", "golden", "skew_alpha.json")


def skew_alpha() -> float:
    """Zipf bias scale for the skewed workload.

    The value is written by ``tests/golden/calibrate_skew.py``, which routes
    the seed-4 tokens with the oracle and bisects for the scale at which the
    hottest expert receives about 20x the mean token count.  Until that file
    exists a provisional 0.5 is used.
    """
    try:
        with open(_GOLDEN) as f:
            return float(json.load(f)["alpha"])
    except FileNotFoundError:
        return 0.5


# ---------------------------------------------------------------------------
# storage-format conversions (bit packing only)
# ---------------------------------------------------------------------------

def bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> BF16 bit pattern (uint16), round to nearest even."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    if a.size >= (1 << 16):
        try:  # torch's CPU cast is the same RNE rounding, multi-threaded
            import torch
            return torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        except ImportError:
            pass
    u = a.view(np.uint32)
    r = (u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """BF16 bit pattern (uint16) -> float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _e4m3_table() -> np.ndarray:
    """All 256 OCP FP8 E4M3 (fn) values, NaN for 0x7F / 0xFF."""
    t = np.zeros(256, dtype=np.float64)
    for b in range(256):
        s = -1.0 if b & 0x80 else 1.0
        ex = (b >> 3) & 0xF
        m = b & 0x7
        if ex == 0xF and m == 0x7:
            t[b] = np.nan
        elif ex == 0:
            t[b] = s * (m / 8.0) * 2.0 ** -6
        else:
            t[b] = s * (1.0 + m / 8.0) * 2.0 ** (ex - 7)
    return t


_E4M3 = _e4m3_table()


def e4m3_to_f32(q: np.ndarray) -> np.ndarray:
    return _E4M3[np.asarray(q, dtype=np.uint8)].astype(np.float32)


def _quantize_rows_e4m3(w: np.ndarray):
    """Per-output-row symmetric FP8 E4M3 quantisation of a float32 matrix.

    scale_row = amax_row / 448; q = RNE(w / scale_row) in E4M3 (torch's CPU
    float8_e4m3fn cast).  Returns (q uint8 bits, scale float32).
    """
    import torch
    amax = np.abs(w).max(axis=-1, keepdims=True).astype(np.float32)
    scale = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    q = torch.from_numpy(np.ascontiguousarray(w / scale)).to(torch.float8_e4m3fn)
    return q.view(torch.uint8).numpy().copy(), scale[..., 0].copy()


# ---------------------------------------------------------------------------
# generator
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class Inputs:
    """Host arrays of one workload, in the layer's storage formats."""
    shape: MoEShape
    norm_w: np.ndarray                   # [H] bf16 bits
    gate_w: np.ndarray                   # [E,H] bf16 bits
    gate_bias: Optional[np.ndarray]      # [E] float32 or None
    up_w: np.ndarray                     # [E,I,D] bf16 bits (uint16) or e4m3 bits (uint8)
    down_w: np.ndarray                   # [E,D,I]
    up_scale: Optional[np.ndarray]       # [E,I] float32 (fp8 only)
    down_scale: Optional[np.ndarray]     # [E,D] float32 (fp8 only)
    shared_up_w: np.ndarray              # [S,H] bf16 bits
    shared_down_w: np.ndarray            # [H,S] bf16 bits
    fc1_w: Optional[np.ndarray]          # [L,H] bf16 bits
    fc2_w: Optional[np.ndarray]          # [H,L] bf16 bits
    hidden: np.ndarray                   # [T,H] bf16 bits
    residual: np.ndarray                 # [T,H] bf16 bits (ignored by the layer)
    shared_up_scale: Optional[np.ndarray] = None    # [S] float32 (shared_fp8 only)
    shared_down_scale: Optional[np.ndarray] = None  # [H] float32 (shared_fp8 only)
    fc1_scale: Optional[np.ndarray] = None          # [L] float32 (latent_fp8 only)
    fc2_scale: Optional[np.ndarray] = None          # [H] float32 (latent_fp8 only)


def _normal(rng, shape, std):
    x = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def _expert_stack(seq, E, rows, cols, fp8):
    """E matrices [rows, cols] ~ N(0, 1/cols); expert e draws from child e of
    the array's seed sequence, so experts are generated in parallel threads."""
    import concurrent.futures as cf
    std = 1.0 / np.sqrt(cols)
    kids = seq.spawn(E)
    out = np.empty((E, rows, cols), dtype=np.uint8 if fp8 else np.uint16)
    sc = np.empty((E, rows), dtype=np.float32) if fp8 else None

    def one(e):
        x = _normal(np.random.Generator(np.random.PCG64(kids[e])), (rows, cols), std)
        if fp8:
            out[e], sc[e] = _quantize_rows_e4m3(x)
        else:
            out[e] = bf16_bits(x)

    with cf.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
        list(ex.map(one, range(E)))
    return out, sc


_STREAMS = ("norm_w", "gate_w", "gate_bias", "up", "down", "shared_up", "shared_down",
            "fc1", "fc2", "hidden", "residual")


def _streams(seed: int):
    kids = np.random.SeedSequence(seed).spawn(len(_STREAMS))
    return ({n: np.random.Generator(np.random.PCG64(k)) for n, k in zip(_STREAMS, kids)},
            dict(zip(_STREAMS, kids)))


def make_inputs(shape: MoEShape, T: Optional[int] = None,
                alpha: Optional[float] = None, experts: bool = True) -> Inputs:
    """Draw every array of a workload from its seed.

    ``T`` overrides the token count (hidden rows are a prefix of a larger T).
    ``alpha`` overrides the Zipf bias scale (used by the calibration script).
    ``experts=False`` skips the routed/shared/latent weights (left None), for
    callers that only route tokens.
    """
    if T is not None:
        shape = shape.with_tokens(T)
    s = shape
    rng, seqs = _streams(s.seed)
    norm_w = bf16_bits(rng["norm_w"].uniform(0.5, 1.5, size=s.H).astype(np.float32))
    gate_w = bf16_bits(_normal(rng["gate_w"], (s.E, s.H), np.sqrt(s.gate_scale / s.H)))
    if s.bias == "none":
        gate_bias = None
    elif s.bias == "uniform":
        gate_bias = rng["gate_bias"].uniform(-0.1, 0.1, size=s.E).astype(np.float32)
    elif s.bias == "zipf":
        # Zipf(s=1.1) profile over a random expert permutation: the expert of
        # popularity rank r (1-based) gets bias -alpha * 1.1 * ln(r).
        perm = rng["gate_bias"].permutation(s.E)
        a = skew_alpha() if alpha is None else alpha
        gate_bias = np.empty(s.E, dtype=np.float32)
        gate_bias[perm] = (-a * 1.1 * np.log(np.arange(1, s.E + 1))).astype(np.float32)
    else:
        raise ValueError(s.bias)
    D = s.D
    up_w = down_w = up_scale = down_scale = None
    shared_up_w = shared_down_w = fc1_w = fc2_w = None
    shared_up_scale = shared_down_scale = fc1_scale = fc2_scale = None
    if experts:
        up_w, up_scale = _expert_stack(seqs["up"], s.E, s.I, D, s.expert_fp8)
        down_w, down_scale = _expert_stack(seqs["down"], s.E, D, s.I, s.expert_fp8)
        def dense(name, rows, cols, fp8):
            x = _normal(rng[name], (rows, cols), 1.0 / np.sqrt(cols))
            return _quantize_rows_e4m3(x) if fp8 else (bf16_bits(x), None)
        shared_up_w, shared_up_scale = dense("shared_up", s.S, s.H, s.shared_fp8)
        shared_down_w, shared_down_scale = dense("shared_down", s.H, s.S, s.shared_fp8)
        if s.L > 0:
            fc1_w, fc1_scale = dense("fc1", s.L, s.H, s.latent_fp8)
            fc2_w, fc2_scale = dense("fc2", s.H, s.L, s.latent_fp8)
    hidden = bf16_bits(_normal(rng["hidden"], (s.T, s.H), 1.0))
    residual = bf16_bits(_normal(rng["residual"], (s.T, s.H), 1.0))
    return Inputs(s, norm_w, gate_w, gate_bias, up_w, down_w, up_scale,
                  down_scale, shared_up_w, shared_down_w, fc1_w, fc2_w,
                  hidden, residual, shared_up_scale, shared_down_scale, fc1_scale, fc2_scale)

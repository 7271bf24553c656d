"""Python binding of the B200 MoE FFN layer library (libmoe_b200.so).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels (include/moe_b200.h).  PyTorch provides device memory and streams.
There is no fallback: if the shared library is missing or cannot be loaded,
``load_library`` raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

__all__ = ["load_library", "sort_static", "MoEConfig", "MoELayer", "MoEError", "STATUS",
           "PATH_AUTO", "PATH_DECODE", "PATH_PREFILL", "EXPORTED_SYMBOLS", "LIB_PATH"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_b200.so")

STATUS = {
    0: "MOE_OK", 1: "MOE_ERR_INVALID_CONFIG", 2: "MOE_ERR_NULL_POINTER",
    3: "MOE_ERR_MISALIGNED", 4: "MOE_ERR_TOKENS_OUT_OF_RANGE", 5: "MOE_ERR_OUT_OF_MEMORY",
    6: "MOE_ERR_CUDA", 7: "MOE_ERR_DEVICE", 8: "MOE_ERR_INVALID_HANDLE",
}
PATH_AUTO, PATH_DECODE, PATH_PREFILL = 0, 1, 2
WEIGHTS_BF16, WEIGHTS_FP8 = 0, 1

EXPORTED_SYMBOLS = ("moe_create", "moe_forward", "moe_forward_path", "moe_forward_host",
                    "moe_destroy", "moe_status_string", "moe_route", "moe_sort",
                    "moe_get_device_status", "moe_last_launch_count", "moe_copy_routing",
                    "moe_set_stage_events", "moe_sort_static", "moe_copy_sort",
                    "moe_last_path")


class MoEError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


class MoEConfig(ctypes.Structure):
    _fields_ = [("hidden_size", ctypes.c_int32), ("num_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("moe_inter", ctypes.c_int32),
                ("shared_inter", ctypes.c_int32), ("latent_size", ctypes.c_int32),
                ("max_tokens", ctypes.c_int32), ("rms_eps", ctypes.c_float),
                ("routed_scaling_factor", ctypes.c_float), ("expert_wdtype", ctypes.c_int32),
                ("shared_wdtype", ctypes.c_int32), ("latent_wdtype", ctypes.c_int32)]


class MoEWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("norm_w", "gate_w", "gate_bias", "up_w", "down_w", "up_scale", "down_scale",
                 "shared_up_w", "shared_down_w", "fc1_w", "fc2_w", "shared_up_scale",
                 "shared_down_scale", "fc1_scale", "fc2_scale")]


_lib = None


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libmoe_b200.so (building it first if it is absent and nvcc exists).

    The MOE_B200_LIBRARY environment variable names another build of the same
    library to load instead (e.g. one compiled with different tile sizes).
    """
    global _lib
    if _lib is not None:
        return _lib
    p = path or os.environ.get("MOE_B200_LIBRARY") or LIB_PATH
    if not os.path.exists(p):
        if p != LIB_PATH:  # an explicit library that is not there: no substitute
            raise FileNotFoundError(f"libmoe_b200: {p} does not exist")
        from . import build as _build
        _build.build()  # raises when nvcc fails; there is no fallback implementation
    lib = ctypes.CDLL(p)
    V, I32 = ctypes.c_void_p, ctypes.c_int32
    sig = {
        "moe_create": ([V, V, V], ctypes.c_int),
        "moe_forward": ([V, V, V, I32, V], ctypes.c_int),
        "moe_forward_path": ([V, V, V, I32, I32, V], ctypes.c_int),
        "moe_forward_host": ([V, V, V, I32, V], ctypes.c_int),
        "moe_destroy": ([V], ctypes.c_int),
        "moe_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "moe_route": ([V, V, I32, V, V, V], ctypes.c_int),
        "moe_sort": ([V, V, I32, V, V, V, V], ctypes.c_int),
        "moe_get_device_status": ([V, V, V], ctypes.c_int),
        "moe_last_launch_count": ([V], I32),
        "moe_copy_routing": ([V, V, V, I32, V], ctypes.c_int),
        "moe_set_stage_events": ([V, V, I32], ctypes.c_int),
        "moe_sort_static": ([V, I32, I32, I32, V, V, V, V, V], ctypes.c_int),
        "moe_copy_sort": ([V, V, V, V, I32, V], ctypes.c_int),
        "moe_last_path": ([V], I32),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    _lib = lib
    return lib


def _ptr(t) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def _stream_ptr(stream) -> Optional[int]:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream) or None


def sort_static(idx, top_k, num_experts, perm, inv, off, status=None, stream=None):
    """moe_sort_static: sort-by-expert of idx [T, top_k] (CUDA int32) into
    perm, inv, off without a handle and without device allocation (scratch
    in a fixed array of the library, at most MOE_SORT_STATIC_MAX_TOKENS
    tokens; overlapping calls on one device race on it)."""
    lib = load_library()
    st = lib.moe_sort_static(_ptr(idx), idx.shape[0], top_k, num_experts, _ptr(perm), _ptr(inv),
                             _ptr(off), _ptr(status), _stream_ptr(stream))
    if st != 0:
        raise MoEError(st, "moe_sort_static")


class MoELayer:
    """One layer instance bound to device weight tensors (torch, on CUDA).

    The tensors are kept referenced for the lifetime of the layer because the
    library borrows their memory.
    """

    def __init__(self, *, hidden_size, num_experts, top_k, moe_inter, shared_inter,
                 latent_size=0, max_tokens, rms_eps=1e-5, routed_scaling_factor=1.0,
                 expert_fp8=False, shared_fp8=False, latent_fp8=False, norm_w, gate_w,
                 gate_bias=None, up_w, down_w, up_scale=None, down_scale=None, shared_up_w,
                 shared_down_w, fc1_w=None, fc2_w=None, shared_up_scale=None,
                 shared_down_scale=None, fc1_scale=None, fc2_scale=None):
        self.lib = load_library()
        dt = lambda f: WEIGHTS_FP8 if f else WEIGHTS_BF16  # noqa: E731
        self.cfg = MoEConfig(hidden_size, num_experts, top_k, moe_inter, shared_inter,
                             latent_size, max_tokens, rms_eps, routed_scaling_factor,
                             dt(expert_fp8), dt(shared_fp8), dt(latent_fp8))
        self._tensors = dict(norm_w=norm_w, gate_w=gate_w, gate_bias=gate_bias, up_w=up_w,
                             down_w=down_w, up_scale=up_scale, down_scale=down_scale,
                             shared_up_w=shared_up_w, shared_down_w=shared_down_w,
                             fc1_w=fc1_w, fc2_w=fc2_w, shared_up_scale=shared_up_scale,
                             shared_down_scale=shared_down_scale, fc1_scale=fc1_scale,
                             fc2_scale=fc2_scale)
        self.w = MoEWeights(**{k: _ptr(v) for k, v in self._tensors.items()})
        self.handle = ctypes.c_void_p()
        st = self.lib.moe_create(ctypes.byref(self.cfg), ctypes.byref(self.w),
                                 ctypes.byref(self.handle))
        if st != 0:
            raise MoEError(st, "moe_create")

    # -- calls ---------------------------------------------------------------
    def _check(self, st, what):
        if st != 0:
            raise MoEError(st, what)

    def forward(self, hidden, residual, num_tokens=None, path=PATH_AUTO, stream=None):
        """In place: hidden <- layer(hidden); residual <- pre-layer hidden."""
        T = hidden.shape[0] if num_tokens is None else num_tokens
        self._check(self.lib.moe_forward_path(self.handle, _ptr(hidden), _ptr(residual), T,
                                              path, _stream_ptr(stream)), "moe_forward")

    def forward_host(self, hidden_host, residual_host=None, stream=None):
        """Host (preferably pinned) CPU tensors; enqueue only, sync the stream to read."""
        T = hidden_host.shape[0]
        self._check(self.lib.moe_forward_host(self.handle, _ptr(hidden_host),
                                              _ptr(residual_host), T, _stream_ptr(stream)),
                    "moe_forward_host")

    def route(self, hidden, idx, w, stream=None):
        self._check(self.lib.moe_route(self.handle, _ptr(hidden), hidden.shape[0], _ptr(idx),
                                       _ptr(w), _stream_ptr(stream)), "moe_route")

    def sort(self, idx, perm, inv, off, stream=None):
        self._check(self.lib.moe_sort(self.handle, _ptr(idx), idx.shape[0], _ptr(perm),
                                      _ptr(inv), _ptr(off), _stream_ptr(stream)), "moe_sort")

    def copy_routing(self, idx, w, stream=None):
        """Routing (idx, w) the last forward used; tensors [T, k] on the device."""
        self._check(self.lib.moe_copy_routing(self.handle, _ptr(idx), _ptr(w), idx.shape[0],
                                              _stream_ptr(stream)), "moe_copy_routing")

    def copy_sort(self, perm, inv, off, num_tokens, stream=None):
        """Sort by expert (perm [R], inv [R], off [E+1]) of the last forward
        (prefill path); int32 tensors on the device."""
        self._check(self.lib.moe_copy_sort(self.handle, _ptr(perm), _ptr(inv), _ptr(off),
                                           num_tokens, _stream_ptr(stream)), "moe_copy_sort")

    def device_status(self, stream=None) -> int:
        v = ctypes.c_int32(0)
        self._check(self.lib.moe_get_device_status(self.handle, ctypes.byref(v),
                                                   _stream_ptr(stream)), "moe_get_device_status")
        return int(v.value)

    def set_stage_events(self, events):
        """Record torch.cuda.Event objects around each kernel of later forwards
        (events[0] before the first launch, events[i] after the i-th); None
        disables.  The events must already exist (recorded once)."""
        if not events:
            self._events = None
            self._check(self.lib.moe_set_stage_events(self.handle, None, 0), "moe_set_stage_events")
            return
        arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
        self._events = (arr, list(events))
        self._check(self.lib.moe_set_stage_events(self.handle, arr, len(events)),
                    "moe_set_stage_events")

    def last_launch_count(self) -> int:
        return int(self.lib.moe_last_launch_count(self.handle))

    def last_path_decode(self) -> bool:
        """Whether the last forward took the decode path."""
        return int(self.lib.moe_last_path(self.handle)) == PATH_DECODE

    def close(self):
        if self.handle:
            self.lib.moe_destroy(self.handle)
            self.handle = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- construction from host arrays -----------------------------------------
    @classmethod
    def from_inputs(cls, inp, max_tokens=None, device="cuda"):
        """Upload a workloads.Inputs weight set to the device and bind it."""
        import numpy as np
        import torch

        def up(a, dtype):
            if a is None:
                return None
            return torch.from_numpy(np.ascontiguousarray(a).view(dtype)).to(device)

        s = inp.shape
        b16 = np.int16
        sf8, lf8 = getattr(s, "shared_fp8", False), getattr(s, "latent_fp8", False)
        wd = np.uint8 if s.expert_fp8 else b16
        sd = np.uint8 if sf8 else b16
        ld = np.uint8 if lf8 else b16
        f32 = np.float32
        return cls(hidden_size=s.H, num_experts=s.E, top_k=s.k, moe_inter=s.I,
                   shared_inter=s.S, latent_size=s.L, max_tokens=max_tokens or s.T,
                   rms_eps=s.eps, routed_scaling_factor=s.rsf, expert_fp8=s.expert_fp8,
                   shared_fp8=sf8, latent_fp8=lf8,
                   norm_w=up(inp.norm_w, b16), gate_w=up(inp.gate_w, b16),
                   gate_bias=up(inp.gate_bias, f32), up_w=up(inp.up_w, wd),
                   down_w=up(inp.down_w, wd), up_scale=up(inp.up_scale, f32),
                   down_scale=up(inp.down_scale, f32),
                   shared_up_w=up(inp.shared_up_w, sd), shared_down_w=up(inp.shared_down_w, sd),
                   fc1_w=up(inp.fc1_w, ld), fc2_w=up(inp.fc2_w, ld),
                   shared_up_scale=up(getattr(inp, "shared_up_scale", None), f32),
                   shared_down_scale=up(getattr(inp, "shared_down_scale", None), f32),
                   fc1_scale=up(getattr(inp, "fc1_scale", None), f32),
                   fc2_scale=up(getattr(inp, "fc2_scale", None), f32))

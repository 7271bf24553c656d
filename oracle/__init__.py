"""ctypes front end of the float64 CPU oracle (oracle/oracle.cpp).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only users.  The CUDA library and its
Python binding never import this package.

Parity status of each function (pins in tests/test_oracle_pins.py):
  rmsnorm, gate_logits, route, route_weights, sort, forward - pinned (closed forms,
  brute-force enumeration, hand-computed cases, invariants).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (plain IEEE float64, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", _LIB])
    return _LIB


class _Cfg(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("E", ctypes.c_int32), ("k", ctypes.c_int32),
                ("I", ctypes.c_int32), ("S", ctypes.c_int32), ("L", ctypes.c_int32),
                ("eps", ctypes.c_double), ("rsf", ctypes.c_double),
                ("expert_fp8", ctypes.c_int32), ("shared_fp8", ctypes.c_int32),
                ("latent_fp8", ctypes.c_int32)]


class _W(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("norm_w", "gate_w", "gate_bias", "up_w", "down_w", "up_scale",
                 "down_scale", "shared_up_w", "shared_down_w", "fc1_w", "fc2_w",
                 "shared_up_scale", "shared_down_scale", "fc1_scale", "fc2_scale")]


_lib = None


def _L():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        for name, args in {
            "oracle_rmsnorm": [P, P, P, ctypes.c_int32, P],
            "oracle_gate_logits": [P, P, P, ctypes.c_int32, P, ctypes.c_int32],
            "oracle_route": [P, P, P, ctypes.c_int32, P, P, P],
            "oracle_route_forced": [P, P, P, ctypes.c_int32, P],
            "oracle_sort": [P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, P, P, P],
            "oracle_forward": [P, P, P, ctypes.c_int32, P, P, P, P, ctypes.c_int32],
        }.items():
            f = getattr(_lib, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        _lib.oracle_bf16_value.argtypes = [ctypes.c_uint16]
        _lib.oracle_bf16_value.restype = ctypes.c_double
        _lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        _lib.oracle_e4m3_value.restype = ctypes.c_double
        _lib.oracle_default_threads.restype = ctypes.c_int
    return _lib


def default_threads() -> int:
    return int(_L().oracle_default_threads())


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """Binds one set of host weights (workloads.Inputs-like object).

    Keeps references to the arrays it was given so their buffers outlive the
    raw pointers stored in the C struct.
    """

    def __init__(self, inp):
        s = inp.shape
        self.shape = s
        self._keep = {}

        def c(name, a, dtype):
            if a is None:
                return None
            a = np.ascontiguousarray(a, dtype=dtype)
            self._keep[name] = a
            return a

        wd = np.uint8 if s.expert_fp8 else np.uint16
        sd = np.uint8 if getattr(s, "shared_fp8", False) else np.uint16
        ld = np.uint8 if getattr(s, "latent_fp8", False) else np.uint16
        arrs = dict(
            norm_w=c("norm_w", inp.norm_w, np.uint16),
            gate_w=c("gate_w", inp.gate_w, np.uint16),
            gate_bias=c("gate_bias", inp.gate_bias, np.float32),
            up_w=c("up_w", inp.up_w, wd),
            down_w=c("down_w", inp.down_w, wd),
            up_scale=c("up_scale", inp.up_scale, np.float32),
            down_scale=c("down_scale", inp.down_scale, np.float32),
            shared_up_w=c("shared_up_w", inp.shared_up_w, sd),
            shared_down_w=c("shared_down_w", inp.shared_down_w, sd),
            fc1_w=c("fc1_w", inp.fc1_w, ld),
            fc2_w=c("fc2_w", inp.fc2_w, ld),
            shared_up_scale=c("shared_up_scale", getattr(inp, "shared_up_scale", None), np.float32),
            shared_down_scale=c("shared_down_scale", getattr(inp, "shared_down_scale", None),
                                np.float32),
            fc1_scale=c("fc1_scale", getattr(inp, "fc1_scale", None), np.float32),
            fc2_scale=c("fc2_scale", getattr(inp, "fc2_scale", None), np.float32),
        )
        self.cfg = _Cfg(s.H, s.E, s.k, s.I, s.S, s.L, float(s.eps), float(s.rsf),
                        1 if s.expert_fp8 else 0, 1 if sd is np.uint8 else 0,
                        1 if ld is np.uint8 else 0)
        self.w = _W(**{k: (None if v is None else v.ctypes.data) for k, v in arrs.items()})
        self.bias = arrs["gate_bias"]

    def _hidden(self, hidden):
        h = np.ascontiguousarray(hidden, dtype=np.uint16)
        assert h.ndim == 2 and h.shape[1] == self.shape.H
        return h

    def rmsnorm(self, hidden) -> np.ndarray:
        h = self._hidden(hidden)
        out = np.empty(h.shape, dtype=np.float64)
        assert _L().oracle_rmsnorm(ctypes.byref(self.cfg), ctypes.byref(self.w), _ptr(h),
                                   h.shape[0], _ptr(out)) == 0
        return out

    def gate_logits(self, hidden, nthreads: int = 0) -> np.ndarray:
        h = self._hidden(hidden)
        out = np.empty((h.shape[0], self.shape.E), dtype=np.float64)
        assert _L().oracle_gate_logits(ctypes.byref(self.cfg), ctypes.byref(self.w), _ptr(h),
                                       h.shape[0], _ptr(out), nthreads) == 0
        return out

    def route(self, logits, bias=None) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
        """(idx [T,k] int32, weights [T,k] f64, selection keys [T,E] f64)."""
        lg = np.ascontiguousarray(logits, dtype=np.float64)
        T = lg.shape[0]
        b = self.bias if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
        idx = np.empty((T, self.shape.k), dtype=np.int32)
        w = np.empty((T, self.shape.k), dtype=np.float64)
        keys = np.empty((T, self.shape.E), dtype=np.float64)
        assert _L().oracle_route(ctypes.byref(self.cfg), _ptr(lg), _ptr(b), T, _ptr(idx),
                                 _ptr(w), _ptr(keys)) == 0
        return idx, w, keys

    def route_weights(self, logits, forced_idx) -> np.ndarray:
        """Routing weights [T,k] f64 of the given expert sets (slot order
        kept): rsf * sigmoid(logit_e) / sum over the set."""
        lg = np.ascontiguousarray(logits, dtype=np.float64)
        T = lg.shape[0]
        f = np.ascontiguousarray(forced_idx, dtype=np.int32)
        assert f.shape == (T, self.shape.k)
        w = np.empty((T, self.shape.k), dtype=np.float64)
        rc = _L().oracle_route_forced(ctypes.byref(self.cfg), _ptr(lg), _ptr(f), T, _ptr(w))
        assert rc == 0, "oracle_route_forced rejected its arguments"
        return w

    def forward(self, hidden, forced_idx=None, nthreads: int = 0):
        """(out [T,H] f64, idx [T,k] int32, weights [T,k] f64)."""
        h = self._hidden(hidden)
        T = h.shape[0]
        out = np.empty((T, self.shape.H), dtype=np.float64)
        idx = np.empty((T, self.shape.k), dtype=np.int32)
        w = np.empty((T, self.shape.k), dtype=np.float64)
        f = None
        if forced_idx is not None:
            f = np.ascontiguousarray(forced_idx, dtype=np.int32)
            assert f.shape == (T, self.shape.k)
        rc = _L().oracle_forward(ctypes.byref(self.cfg), ctypes.byref(self.w), _ptr(h), T,
                                 _ptr(f), _ptr(out), _ptr(idx), _ptr(w), nthreads)
        assert rc == 0, "oracle_forward rejected its arguments"
        return out, idx, w


def sort(idx: np.ndarray, E: int):
    """Counting sort of routed rows by expert: (perm, inv, off)."""
    i = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = i.shape
    R = T * k
    perm = np.empty(R, dtype=np.int32)
    inv = np.empty(R, dtype=np.int32)
    off = np.empty(E + 1, dtype=np.int32)
    rc = _L().oracle_sort(_ptr(i), T, k, E, _ptr(perm), _ptr(inv), _ptr(off))
    if rc != 0:
        raise ValueError("expert id out of range")
    return perm, inv, off


def bf16_value(b: int) -> float:
    return float(_L().oracle_bf16_value(b))


def e4m3_value(b: int) -> float:
    return float(_L().oracle_e4m3_value(b))

"""CPU-side checks of the C ABI: the library builds and loads without a GPU,
exports every function include/*.h declares, and its host-side validation
answers before touching a device."""
import ctypes
import glob
import os
import re

import pytest

import mixture_experts_ffn_rmsnorm_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names += re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("moe_create", "moe_forward", "moe_destroy"):
        assert required in names
    assert set(names) == set(moe.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol():
    lib = moe.load_library()
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings():
    lib = moe.load_library()
    for code in range(9):
        s = lib.moe_status_string(code)
        assert s and s != b"unknown status"
    assert lib.moe_status_string(99) == b"unknown status"


def _cfg(**kw):
    base = dict(hidden_size=256, num_experts=8, top_k=2, moe_inter=128, shared_inter=256,
                latent_size=0, max_tokens=16, rms_eps=1e-5, routed_scaling_factor=1.0,
                expert_wdtype=0)
    base.update(kw)
    return moe.MoEConfig(**base)


def _create(cfg, w):
    lib = moe.load_library()
    h = ctypes.c_void_p(1234)
    st = lib.moe_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h))
    return st, h


ALL16 = dict(norm_w=16, gate_w=32, gate_bias=None, up_w=48, down_w=64, up_scale=None,
             down_scale=None, shared_up_w=80, shared_down_w=96, fc1_w=None, fc2_w=None)


@pytest.mark.parametrize("bad", [dict(top_k=0), dict(top_k=9), dict(top_k=17, num_experts=32),
                                 dict(num_experts=257, top_k=2), dict(hidden_size=100),
                                 dict(moe_inter=96), dict(shared_inter=0), dict(latent_size=-64),
                                 dict(latent_size=32), dict(max_tokens=0), dict(rms_eps=-1.0),
                                 dict(expert_wdtype=5), dict(shared_wdtype=3),
                                 dict(latent_wdtype=-1),
                                 dict(routed_scaling_factor=float("inf"))])
def test_invalid_configs_rejected_on_host(bad):
    # NemotronMoeLayer `new`: top_k must be in 1..=num_experts and within the
    # routing kernels' bounds; plus this library's layout requirements.
    st, h = _create(_cfg(**bad), moe.MoEWeights(**ALL16))
    assert st == 1 and h.value is None


def test_null_and_misaligned_weights_rejected():
    w = dict(ALL16)
    w["up_w"] = None
    st, h = _create(_cfg(), moe.MoEWeights(**w))
    assert st == 2 and h.value is None
    w = dict(ALL16)
    w["gate_w"] = 34
    st, _ = _create(_cfg(), moe.MoEWeights(**w))
    assert st == 3
    # FP8 needs the row scales; LatentMoE needs fc1/fc2
    st, _ = _create(_cfg(expert_wdtype=1), moe.MoEWeights(**ALL16))
    assert st == 2
    st, _ = _create(_cfg(latent_size=128), moe.MoEWeights(**ALL16))
    assert st == 2
    # FP8 shared expert / fc1 / fc2 need their row scales too
    st, _ = _create(_cfg(shared_wdtype=1), moe.MoEWeights(**ALL16))
    assert st == 2
    lat = dict(ALL16, fc1_w=112, fc2_w=128)
    st, _ = _create(_cfg(latent_size=128, latent_wdtype=1), moe.MoEWeights(**lat))
    assert st == 2
    # FP8 routed experts are wired for the direct layer only
    st, _ = _create(_cfg(latent_size=128, expert_wdtype=1),
                    moe.MoEWeights(**dict(lat, up_scale=144, down_scale=160)))
    assert st == 1


def test_invalid_handle_rejected():
    lib = moe.load_library()
    assert lib.moe_forward(None, None, None, 1, None) == 8
    assert lib.moe_destroy(None) == 8
    bogus = ctypes.create_string_buffer(64)
    assert lib.moe_forward(ctypes.addressof(bogus), None, None, 1, None) == 8
    assert lib.moe_last_launch_count(None) == -1


def test_static_sort_validates_on_host():
    # every rejection happens before the device is touched
    lib = moe.load_library()
    p = 256  # any non-NULL value: nothing is dereferenced on these paths
    assert lib.moe_sort_static(None, 10, 2, 8, p, p, p, None, None) == 2
    assert lib.moe_sort_static(p, 10, 2, 8, p, None, p, None, None) == 2
    assert lib.moe_sort_static(p, 8193, 2, 8, p, p, p, None, None) == 4
    assert lib.moe_sort_static(p, 0, 2, 8, p, p, p, None, None) == 4
    assert lib.moe_sort_static(p, 10, 0, 8, p, p, p, None, None) == 1
    assert lib.moe_sort_static(p, 10, 17, 64, p, p, p, None, None) == 1
    assert lib.moe_sort_static(p, 10, 4, 257, p, p, p, None, None) == 1
    assert lib.moe_sort_static(p, 10, 9, 8, p, p, p, None, None) == 1


def test_missing_library_fails_loudly():
    # no fallback: a library path that does not exist is an error, in a fresh
    # interpreter (the loaded library is cached per process)
    import subprocess
    import sys
    code = ("import mixture_experts_ffn_rmsnorm_b200 as m\n"
            "try:\n"
            "    m.load_library()\n"
            "except FileNotFoundError as e:\n"
            "    print('raised', e)\n"
            "else:\n"
            "    print('loaded')\n")
    env = dict(os.environ, MOE_B200_LIBRARY="/nonexistent/libmoe_b200.so")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.startswith("raised"), r.stdout

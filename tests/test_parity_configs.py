"""GPU parity on layer shapes the five workloads do not reach: more experts
than one 128-wide router tile (E = 160, 256; E not a power of two), the
top_k bounds (1 and 16), and a hidden size that is a multiple of 64 but not
of 128.  Every token of every case is compared with the oracle, through the
prefill path and, where the decode path covers the shape, the decode path
at T = 1, 3 and 8.

Weights and tokens come from the workload generator with the decode
workload's distributions (uniform selection bias, rsf 2.5) at these sizes.
"""
import numpy as np
import pytest

import oracle
from tests.gpu_util import check_layer, check_routing, run_forward
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - collected on CPU machines too
    pytest.skip("needs a CUDA device", allow_module_level=True)

import mixture_experts_ffn_rmsnorm_b200 as moe  # noqa: E402

CASES = {
    # name: (H, E, k, I, S, T)
    "E256_k8": (512, 256, 8, 256, 512, 300),
    "E160_k16": (384, 160, 16, 192, 320, 200),
    "E96_k1": (256, 96, 1, 128, 128, 150),
    "H192_E64_k4": (192, 64, 4, 64, 128, 130),
}

_CACHE = {}


def setup(name):
    if name not in _CACHE:
        H, E, k, I, S, T = CASES[name]
        shape = WORKLOADS["decode"].scaled(name=name, T=T, H=H, E=E, k=k, I=I, S=S,
                                           seed=11 + len(_CACHE))
        inp = make_inputs(shape)
        layer = moe.MoELayer.from_inputs(inp, max_tokens=T)
        _CACHE[name] = (inp, layer, oracle.Oracle(inp))
    return _CACHE[name]


def teardown_module(module):
    for _, layer, _ in _CACHE.values():
        layer.close()
    _CACHE.clear()


@pytest.mark.parametrize("name", sorted(CASES))
def test_prefill_all_tokens(name):
    inp, layer, orc = setup(name)
    h = inp.hidden
    out, res, idx, w = run_forward(layer, h, moe.PATH_PREFILL)
    assert np.array_equal(res, h)
    flips = check_routing(orc, h, idx, w)
    check_layer(orc, h, out, idx, np.arange(h.shape[0]))
    assert layer.device_status() == 0
    print(f"{name}: flips={flips}")


@pytest.mark.parametrize("T", [1, 3, 8])
@pytest.mark.parametrize("name", sorted(CASES))
def test_decode_small_batches(name, T):
    inp, layer, orc = setup(name)
    h = inp.hidden[:T]
    out, res, idx, w = run_forward(layer, h, moe.PATH_DECODE)
    assert np.array_equal(res, h)
    check_routing(orc, h, idx, w)
    check_layer(orc, h, out, idx, np.arange(T))
    assert layer.device_status() == 0

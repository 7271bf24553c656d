"""GPU parity with FP8 copies of the shared expert and of LatentMoE fc1 / fc2
(E4M3 bytes with one float32 scale per output row, as the pages keep them:
nemotron_moe.rs `new`), alone and together with FP8 routed experts.

The library runs these as W8A8 on the tensor cores (the normed tokens, the
shared relu^2 rows and the latent sums quantised to E4M3 with one scale per
row); the oracle dequantises the weights exactly and never quantises
activations, so the FP8 bound applies: max|gpu - oracle| <= 5e-2 * max|oracle|
+ 1e-3, over every token.  Decode-sized batches take the prefill path for
these weight types.
"""
import numpy as np
import pytest

import oracle
from tests.gpu_util import check_forward_sort, check_layer, check_routing, run_forward
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - collected on CPU machines too
    pytest.skip("needs a CUDA device", allow_module_level=True)

import mixture_experts_ffn_rmsnorm_b200 as moe  # noqa: E402

# name: (base workload, shape overrides, tokens)
CASES = {
    "tiny_shared_fp8": ("tiny", dict(shared_fp8=True), 200),
    "direct_fp8_experts_and_shared": ("skew_fp8", dict(H=512, I=256, S=512, E=32, k=4,
                                                       shared_fp8=True), 300),
    "latent_fp8_fc": ("latent", dict(H=512, I=256, S=512, E=32, L=256, latent_fp8=True), 260),
    "latent_fp8_fc_and_shared": ("latent", dict(H=512, I=256, S=512, E=32, L=256,
                                                latent_fp8=True, shared_fp8=True), 260),
}

_CACHE = {}


def setup(name):
    if name not in _CACHE:
        base, over, T = CASES[name]
        shape = WORKLOADS[base].scaled(name=name, T=T, **over)
        inp = make_inputs(shape)
        layer = moe.MoELayer.from_inputs(inp, max_tokens=T)
        _CACHE[name] = (inp, layer, oracle.Oracle(inp))
    return _CACHE[name]


def teardown_module(module):
    for _, layer, _ in _CACHE.values():
        layer.close()
    _CACHE.clear()


@pytest.mark.parametrize("T", [4, 129, None])
@pytest.mark.parametrize("name", sorted(CASES))
def test_fp8_dense_weights_every_token(name, T):
    inp, layer, orc = setup(name)
    h = inp.hidden if T is None else inp.hidden[:T]
    n = h.shape[0]
    out, res, idx, w = run_forward(layer, h, moe.PATH_AUTO)
    assert np.array_equal(res, h)
    check_routing(orc, h, idx, w, case=f"{name} T={n}")
    err, bound = check_layer(orc, h, out, idx, np.arange(n), expert_fp8=True)
    check_forward_sort(layer, idx, inp.shape.E)
    assert layer.device_status() == 0
    print(f"{name} T={n}: err {err:.3g} bound {bound:.3g} ({err / bound:.2f} of it)")


def test_fp8_dense_weights_change_the_result():
    # the FP8 copies are what the library reads: the same layer with the
    # BF16 originals gives a different (nearby) output
    inp, layer, orc = setup("tiny_shared_fp8")
    h = inp.hidden[:64]
    out8 = run_forward(layer, h, moe.PATH_AUTO)[0]
    bf = make_inputs(WORKLOADS["tiny"].scaled(name="tiny_bf16", T=200))
    lb = moe.MoELayer.from_inputs(bf, max_tokens=200)
    try:
        outb = run_forward(lb, bf.hidden[:64], moe.PATH_AUTO)[0]
    finally:
        lb.close()
    assert not np.array_equal(out8, outb)
    assert np.max(np.abs(out8 - outb)) < 0.2 * np.max(np.abs(outb))

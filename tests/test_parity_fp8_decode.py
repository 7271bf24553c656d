"""GPU parity of the single-launch decode path with FP8 routed experts (E4M3
weights, one float32 scale per weight row; nemotron_moe.rs `new` keeps FP8
expert copies and decodes through W8A16 kernels).  The launch streams the
E4M3 boxes and dequantises them to BF16 in shared memory (value times its
row's scale, rounded once), so the activations stay BF16; the oracle
dequantises exactly.  The FP8 bound applies: max|gpu - oracle| <= 5e-2 *
max|oracle| + 1e-3, over every token.
"""
import numpy as np
import pytest

import oracle
from tests.gpu_util import check_layer, check_routing, run_forward, to_dev
from workloads import WORKLOADS, bf16_to_f32, make_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - collected on CPU machines too
    pytest.skip("needs a CUDA device", allow_module_level=True)

import mixture_experts_ffn_rmsnorm_b200 as moe  # noqa: E402

# name: (base workload, shape overrides)
SHAPES = {
    # the skewed FP8 workload's layer (H=2688, E=128, k=6, I=1856 with a
    # 64-row last unit per expert, Zipf bias), at decode sizes
    "skew_fp8_decode": ("skew_fp8", dict(T=8)),
    # H = 192: the last FP8 box of an up row is half past the matrix
    "tiny_fp8_h192": ("tiny", dict(T=8, H=192, expert_fp8=True)),
}

_CACHE = {}


def setup(name):
    if name not in _CACHE:
        base, over = SHAPES[name]
        shape = WORKLOADS[base].scaled(name=name, **over)
        inp = make_inputs(shape)
        layer = moe.MoELayer.from_inputs(inp, max_tokens=inp.shape.T)
        _CACHE[name] = (inp, layer, oracle.Oracle(inp))
    return _CACHE[name]


def teardown_module(module):
    for _, layer, _ in _CACHE.values():
        layer.close()
    _CACHE.clear()


@pytest.mark.parametrize("T", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("name", sorted(SHAPES))
def test_fp8_experts_decode_path_every_token(name, T):
    inp, layer, orc = setup(name)
    h = inp.hidden[:T]
    out, res, idx, w = run_forward(layer, h, moe.PATH_DECODE)
    assert layer.last_path_decode()
    assert np.array_equal(res, h)
    check_routing(orc, h, idx, w, case=f"{name} T={T} (decode)")
    err, bound = check_layer(orc, h, out, idx, np.arange(T), expert_fp8=True)
    assert layer.device_status() == 0
    print(f"{name} T={T} decode: err {err:.3g} bound {bound:.3g} ({err / bound:.2f} of it)")


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_fp8_experts_decode_and_prefill_paths_agree_with_the_oracle(name):
    inp, layer, orc = setup(name)
    h = inp.hidden[:8]
    for path in (moe.PATH_DECODE, moe.PATH_PREFILL):
        out, res, idx, w = run_forward(layer, h, path)
        check_routing(orc, h, idx, w)
        check_layer(orc, h, out, idx, np.arange(8), expert_fp8=True)
    assert layer.device_status() == 0


def test_fp8_experts_decode_graph_replay_is_bit_exact():
    inp, layer, orc = setup("skew_fp8_decode")
    hb = inp.hidden[:1]
    ref = run_forward(layer, hb, moe.PATH_DECODE)[0]
    s = torch.cuda.Stream()
    hid = to_dev(hb)
    res = torch.empty_like(hid)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        layer.forward(hid, res, path=moe.PATH_DECODE, stream=s)
    for _ in range(3):
        hid.copy_(to_dev(hb))
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(bf16_to_f32(hid.cpu().numpy().view(np.uint16)), ref)
    assert layer.device_status() == 0


@pytest.mark.parametrize("T,decode", [(1, True), (2, False), (8, False)])
def test_fp8_experts_auto_path_choice(T, decode):
    # the decode launch is chosen for FP8 experts where it is the faster
    # path: one token (each routed unit then has a CTA to itself)
    inp, layer, orc = setup("skew_fp8_decode")
    h = inp.hidden[:T]
    out, res, idx, w = run_forward(layer, h, moe.PATH_AUTO)
    assert layer.last_path_decode() == decode
    check_layer(orc, h, out, idx, np.arange(T), expert_fp8=True)

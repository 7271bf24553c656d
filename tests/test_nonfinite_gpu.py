"""GPU: a token whose gate logits are NaN (one NaN in its hidden row makes
its RMSNorm factor NaN) chooses no expert.  No comparison with a NaN
selection key holds, so the sigmoid top-k of NemotronMoeLayer (nemotron_moe.rs
module documentation) never picks one; the layer reports the out-of-range
ids in bit 2 of the device status word and routes the token nowhere.  Every
other token of the batch is unaffected: its routing and its output match the
oracle, on the single-launch decode path and on the prefill path (whose sort
gives such a row inv = -1 and whose combine skips it).
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

BAD_INDEX_BIT = 2
NAN_BF16 = 0x7FC0
_CACHE = {}


def setup():
    if "decode" not in _CACHE:
        inp = make_inputs(WORKLOADS["decode"].scaled(T=16))
        layer = moe.MoELayer.from_inputs(inp, max_tokens=16)
        _CACHE["decode"] = (inp, layer, oracle.Oracle(inp))
    return _CACHE["decode"]


def teardown_module(module):
    for _, layer, _ in _CACHE.values():
        layer.close()
    _CACHE.clear()


@pytest.mark.parametrize("T,path", [(1, "decode"), (4, "decode"), (8, "decode"),
                                    (8, "prefill"), (16, "prefill")])
def test_nan_token_routes_nowhere_and_leaves_the_others_exact(T, path):
    inp, layer, orc = setup()
    p = moe.PATH_DECODE if path == "decode" else moe.PATH_PREFILL
    bad = min(2, T - 1)
    h = inp.hidden[:T].copy()
    h[bad, 5] = NAN_BF16
    assert layer.device_status() == 0
    out, res, idx, w = run_forward(layer, h, p)
    assert layer.last_path_decode() == (path == "decode")
    status = layer.device_status()  # (reading clears it)
    assert status & BAD_INDEX_BIT, f"status {status}"
    E = inp.shape.E
    assert np.all((idx[bad] < 0) | (idx[bad] >= E)), idx[bad]
    others = np.array([t for t in range(T) if t != bad], dtype=np.int64)
    if len(others):
        check_routing(orc, h, idx, w, rows=others)
        check_layer(orc, h, out, idx, others)
    # the next clean pass reports nothing
    run_forward(layer, inp.hidden[:T], p)
    assert layer.device_status() == 0

"""moe_sort_static (sort-by-expert with scratch in a fixed device array, no
allocation) against the handle-based moe_sort and the oracle.

Integer outputs, so the tolerance is zero: perm, inv and off must be equal.
Two calls in a row with different routing check that nothing from the
first call leaks into the second.  The file name makes pytest collect it
last; it also passes alone.
"""
import numpy as np
import pytest

import oracle
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - collected on CPU machines too
    pytest.skip("needs a CUDA device", allow_module_level=True)

import mixture_experts_ffn_rmsnorm_b200 as moe  # noqa: E402

MAX_T = 8192          # MOE_SORT_STATIC_MAX_TOKENS
BAD_INDEX_BIT = 2     # device status bit: an id outside [0, E) was skipped


@pytest.fixture(scope="module")
def layer():
    # E = 128, top_k = 6 as the prefill workload, narrow matrices (only the
    # sort runs here); max_tokens covers the static entry point's limit.
    shape = WORKLOADS["prefill"].scaled(H=256, I=128, S=256)
    inp = make_inputs(shape, T=16)
    lay = moe.MoELayer.from_inputs(inp, max_tokens=MAX_T)
    yield lay
    lay.close()


def _routing(T, E, k, seed, skew):
    rng = np.random.default_rng(seed)
    if skew:  # one hot expert in every token, groups of every size elsewhere
        rest = np.delete(np.arange(E), 5)
        idx = np.stack([np.concatenate([[5], rng.choice(rest, k - 1, replace=False)])
                        for _ in range(T)])
    else:
        idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
    return idx.astype(np.int32)


def _outs(R, E):
    z = lambda n: torch.full((n,), -7, dtype=torch.int32, device="cuda")  # noqa: E731
    return z(R), z(R), z(E + 1)


def test_static_sort_matches_handle_sort_two_calls_in_a_row(layer):
    E, k = layer.cfg.num_experts, layer.cfg.top_k
    status = torch.full((1,), 99, dtype=torch.int32, device="cuda")
    for T, seed, skew in ((1000, 11, False), (MAX_T, 12, True)):
        idx = _routing(T, E, k, seed, skew)
        d_idx = torch.from_numpy(idx).cuda()
        R = T * k
        ps, is_, os_ = _outs(R, E)
        ph, ih, oh = _outs(R, E)
        moe.sort_static(d_idx, k, E, ps, is_, os_, status=status)
        layer.sort(d_idx, ph, ih, oh)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(ps, ph) and torch.equal(is_, ih) and torch.equal(os_, oh)
        perm_o, inv_o, off_o = oracle.sort(idx, E)
        assert np.array_equal(ps.cpu().numpy(), perm_o)
        assert np.array_equal(is_.cpu().numpy(), inv_o)
        assert np.array_equal(os_.cpu().numpy(), off_o)


def test_static_sort_without_status_and_tiny_config():
    # no handle at all: E = 8, top_k = 2, a ragged single tile, status word
    # from the scratch; run twice so the second call reuses the scratch
    E, k = 8, 2
    for T, seed in ((37, 1), (5, 2)):
        idx = _routing(T, E, k, seed, False)
        perm, inv, off = _outs(T * k, E)
        moe.sort_static(torch.from_numpy(idx).cuda(), k, E, perm, inv, off)
        torch.cuda.synchronize()
        perm_o, inv_o, off_o = oracle.sort(idx, E)
        assert np.array_equal(perm.cpu().numpy(), perm_o)
        assert np.array_equal(inv.cpu().numpy(), inv_o)
        assert np.array_equal(off.cpu().numpy(), off_o)


def test_static_sort_status_is_cleared_between_calls():
    # an out-of-range id is skipped by the kernels' bounds checks and flagged;
    # the next call starts from a cleared status word
    E, k, T = 16, 2, 40
    idx = _routing(T, E, k, 3, False)
    bad = idx.copy()
    bad[7, 1] = E
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    perm, inv, off = _outs(T * k, E)
    moe.sort_static(torch.from_numpy(bad).cuda(), k, E, perm, inv, off, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & BAD_INDEX_BIT
    # the skipped row goes nowhere (inv = -1); every other row is placed
    inv_b, perm_b = inv.cpu().numpy(), perm.cpu().numpy()
    assert inv_b[7 * k + 1] == -1
    good = np.array([f for f in range(T * k) if f != 7 * k + 1])
    assert np.array_equal(perm_b[inv_b[good]], good)
    moe.sort_static(torch.from_numpy(idx).cuda(), k, E, perm, inv, off, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert np.array_equal(perm.cpu().numpy(), oracle.sort(idx, E)[0])


def test_static_sort_rejects_sizes_beyond_its_scratch():
    E, k = 128, 6
    idx = torch.zeros((MAX_T + 1, k), dtype=torch.int32, device="cuda")
    perm, inv, off = _outs((MAX_T + 1) * k, E)
    with pytest.raises(moe.MoEError) as ei:
        moe.sort_static(idx, k, E, perm, inv, off)
    assert ei.value.status == 4  # MOE_ERR_TOKENS_OUT_OF_RANGE
    with pytest.raises(moe.MoEError) as ei:
        moe.sort_static(idx[:4], 17, E, perm, inv, off)
    assert ei.value.status == 1  # MOE_ERR_INVALID_CONFIG (top_k above 16)

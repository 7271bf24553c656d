"""bench.py's work model on CPU: the algorithmic bytes and flops it divides
by each kernel's time, against closed forms written out here from the
layer's shapes, and the committed DRAM captures against that model.

The closed forms count what the layer must move or compute once: every
touched expert's weights, the shared expert, the gate, and the token rows
(NemotronMoeLayer `prefill` / `decode`; grouped GEMM loading each expert's
weights once, MoeLayer `forward_prefill`).
"""
import json
import os

import pytest

import bench
from workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _sum(stages, i):
    return sum(st[i] for st in stages)


def test_decode_T1_bytes_match_the_weight_stream():
    s = WORKLOADS["decode"]
    H, E, k, I, S = s.H, s.E, s.k, s.I, s.S
    U, T = k, 1  # one token touches k distinct experts
    weights = U * 2 * H * I * 2 + 2 * H * S * 2 + E * H * 2
    tokens = H * 2 + 3 * T * H * 2
    closed = weights + tokens
    assert closed == 160_355_328  # 160.4 MB: a 24.5 us roofline at 6.53 TB/s
    model = bench.stage_model(s, T, "decode", U)
    assert [m[0] for m in model] == ["decode_fused"]  # the decode path is one launch
    assert model[0][1] == closed
    assert model[0][2] == 2 * T * H * E + 4 * T * k * H * I + 4 * T * H * S


@pytest.mark.parametrize("name,T,gflop", [
    ("prefill", 1024, 164.2),   # 48 rows per expert: HBM-bound
    ("latent", 4096, 794.6),    # tensor-bound
])
def test_prefill_flops_closed_form(name, T, gflop):
    s = WORKLOADS[name]
    H, E, k, I, S, L, D = s.H, s.E, s.k, s.I, s.S, s.L, s.D
    R = T * k
    closed = 2 * T * H * E + 4 * R * D * I + 4 * T * H * S + 4 * T * H * L
    assert closed / 1e9 == pytest.approx(gflop, abs=0.05)
    for split in (False, True):
        model = bench.stage_model(s, T, "prefill", E, router_split=split)
        assert _sum(model, 2) == closed


def test_skew_fp8_splits_fp8_and_bf16_work():
    s = WORKLOADS["skew_fp8"]
    T = 8192
    H, E, k, I, S = s.H, s.E, s.k, s.I, s.S
    R = T * k
    fp8 = 4 * R * H * I
    bf16 = 2 * T * H * E + 4 * T * H * S
    assert fp8 / 1e9 == pytest.approx(980.9, abs=0.05)
    assert bf16 / 1e9 == pytest.approx(332.6, abs=0.05)
    model = bench.stage_model(s, T, "prefill", E, router_split=True)
    assert _sum(model, 2) == fp8 + bf16
    names = [m[0] for m in model]
    assert "quantize_rows" in names and "combine" in names
    # FP8 expert weights stream one byte per element plus one fp32 scale per row
    up = dict((m[0], m) for m in model)["grouped_up_gemm"]
    assert up[1] >= E * I * H * 1 + E * I * 4 + S * H * 2


def test_prefill_T1024_weight_bytes():
    s = WORKLOADS["prefill"]
    H, E, I, S = s.H, s.E, s.I, s.S
    weights = E * 2 * H * I * 2 + 2 * H * S * 2 + E * H * 2
    assert weights / 1e9 == pytest.approx(2.595, abs=0.001)
    model = bench.stage_model(s, 1024, "prefill", E, router_split=True)
    gemms = [m for m in model if "gemm" in m[0]]
    assert _sum(gemms, 1) > weights
    assert _sum(gemms, 1) < weights * 1.1


def test_roofline_picks_the_binding_bound():
    peaks = {"hbm_gbs": 6530.0, "bf16_tflops": 1626.0, "bf16_tflops_sustained": 1399.0,
             "source": "measured"}
    # 80 MB in 30 us: HBM-bound, 2.67 TB/s
    r = bench.roofline_of("decode_down_gemm", 80e6, 1e6, 0.030, peaks)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(80e6 / 30e-6 / 1e9, rel=1e-3)
    assert r["frac"] == pytest.approx(r["achieved"] / 6530.0, rel=1e-3)
    # 800 GFLOP in 1 ms over 1.6 GB: tensor-bound
    r = bench.roofline_of("grouped_up_gemm", 1.6e9, 800e9, 1.0, peaks)
    assert r["bound"] == "tensor" and r["peak"] == 1626.0
    assert r["frac"] == pytest.approx(800e9 / 1626e12 / 1e-3, rel=1e-3)
    # all of it on FP8 operands: twice the peak, half the bound time
    r8 = bench.roofline_of("grouped_up_gemm", 1.6e9, 800e9, 1.0, peaks, 800e9)
    assert r8["peak"] == 2 * 1626.0 and r8["frac"] == pytest.approx(r["frac"] / 2, rel=1e-3)
    # kernels without flops are HBM-bound
    r = bench.roofline_of("combine", 1e8, 0, 0.02, peaks)
    assert r["bound"] == "hbm"


def test_mixed_fp8_bf16_launch_takes_each_class_at_its_own_peak():
    # the skew workload's up launch at T = 8192: routed experts FP8, shared
    # expert BF16 (same launch); the bound is the sum of the two classes'
    # times, not all flops at the FP8 rate
    peaks = {"hbm_gbs": 6530.0, "bf16_tflops": 1626.0, "source": "measured"}
    s = WORKLOADS["skew_fp8"]
    T = 8192
    up = dict((m[0], m) for m in bench.stage_model(s, T, "prefill", s.E, router_split=True))[
        "grouped_up_gemm"]
    fp8 = 2 * T * s.k * s.H * s.I
    bf16 = 2 * T * s.H * s.S
    assert up[2] == fp8 + bf16 and up[3] == fp8
    t_bound = fp8 / (2 * 1626e12) + bf16 / 1626e12
    r = bench.roofline_of("grouped_up_gemm", up[1], up[2], 0.430, peaks, up[3])
    assert r["bound"] == "tensor"
    assert r["frac"] == pytest.approx(t_bound / 0.430e-3, rel=1e-3)
    assert 0.55 < r["frac"] < 0.6   # 58 % at 430 us, where all-FP8 would say 47 %


def test_gather_moves_each_token_row_once_and_writes_each_slot():
    for name, T in (("prefill", 1024), ("skew_fp8", 8192), ("latent", 4096)):
        s = WORKLOADS[name]
        wb = 1 if s.expert_fp8 else 2
        R = T * s.k
        g = dict((m[0], m) for m in bench.stage_model(s, T, "prefill", s.E, True))["gather"]
        assert g[1] == T * s.D * wb + R * s.D * wb + R * 4


def test_step_work_closed_forms():
    s = WORKLOADS["decode"]
    nb, fl, f8 = bench.step_work(s, 1, 6)
    assert nb == 160_355_328 and f8 == 0
    assert fl == 2 * s.H * s.E + 4 * 6 * s.H * s.I + 4 * s.H * s.S
    s = WORKLOADS["skew_fp8"]
    nb, fl, f8 = bench.step_work(s, 8192, s.E)
    assert f8 / 1e9 == pytest.approx(980.9, abs=0.05)
    assert (fl - f8) / 1e9 == pytest.approx(332.6, abs=0.05)
    s = WORKLOADS["latent"]
    nb, fl, f8 = bench.step_work(s, 4096, s.E)
    assert fl / 1e9 == pytest.approx(794.6, abs=0.05) and f8 == 0


def test_committed_dram_captures_are_close_to_the_model():
    """Every capture in profiles/traffic.json moves within 10 % of the
    algorithmic bytes the benchmark divides by: no wasted re-reads."""
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        recs = json.load(f)["kernels"]
    assert recs
    for key, rec in recs.items():
        stage, workload = key.split("@")
        name, tok = workload.split(" T=")
        T = int(tok)
        s = WORKLOADS[name]
        path = "decode" if stage == "decode_fused" else "prefill"
        # touched experts: as captured (decode), all of them (prefill)
        U = rec.get("distinct_experts", s.k * T) if path == "decode" else s.E
        model = dict((m[0], m) for m in bench.stage_model(s, T, path, U, router_split=True))
        stage_bytes = model[stage][1] if stage in model else model[stage.replace("_gemm", "_gemm_topk")][1]
        got = rec["dram_bytes_per_launch"]
        assert abs(got - stage_bytes) <= 0.10 * stage_bytes, (key, got, stage_bytes)
        assert rec["capture"].startswith("profiles/") and os.path.exists(
            os.path.join(ROOT, rec["capture"]))


def test_sources_hash_is_stable_and_detects_change(tmp_path):
    a = tmp_path / "a.cu"
    a.write_text("x")
    rel = os.path.relpath(a, bench.ROOT)
    h1 = bench.sources_hash([rel])
    assert h1 == bench.sources_hash([rel]) and len(h1) == 16
    a.write_text("y")
    assert bench.sources_hash([rel]) != h1
    assert bench.sources_hash(["no/such/file.cu"]) is None
    assert bench.kernel_traffic("no_such_stage", "decode T=1") is None

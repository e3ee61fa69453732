"""Host-side arithmetic of the benchmark's roofline object (no GPU)."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

PEAKS = {"bf16_tflops_sustained": 1400.0, "source": "fallback"}


def test_dominant_stage_and_its_flop_model():
    # 5 launches of attn_bwd at 2 ms each dominate 5 launches of attn_fwd at 1 ms
    stages = {"attn_bwd": (10.0, 5), "attn_fwd": (5.0, 5)}
    r = bench.stage_roofline(stages, 8, 24, 4096, 64, PEAKS)
    assert r["kernel"] == "attn_bwd" and r["bound"] == "tensor"
    L, d, nh = 4096, 64, 8 * 24
    flop = (5.0 * L * L * d + 2.0 * L * L * d * d / 128) * nh
    assert r["achieved"] == pytest.approx(flop / 2e-3 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / 1400.0)
    assert r["traffic"] is None  # no capture given


def test_traffic_scales_with_the_heads_processed():
    stages = {"attn_bwd": (5.75, 1)}
    per_head = {k: v / 6.0 for k, v in bench.DRAM_BYTES_FOX_B1H6.items()}
    r = bench.stage_roofline(stages, 1, 24, 16384, 64, PEAKS, per_head)
    assert r["traffic"] == pytest.approx(4.0 * bench.DRAM_BYTES_FOX_B1H6["attn_bwd"])
    assert r["traffic_unit"] == "bytes per launch"
    # a stage without a capture reports none
    r = bench.stage_roofline({"chain": (1.0, 1)}, 1, 24, 16384, 64, PEAKS, per_head)
    assert r["kernel"] == "chain" and r["traffic"] is None


def test_ut_stage_models_count_the_issued_products():
    # per 128-block: 36 (prep) and 52 (adjoint) products of 64 x 64 x 64 at d = 64
    f, bound = bench.stage_model("ut_prep", 1, 1, 4096, 64)
    assert bound == "tensor" and f == pytest.approx(32 * 36 * 2.0 * 64 ** 3)
    f, bound = bench.stage_model("ut_adj", 2, 3, 4096, 128)
    assert bound == "tensor" and f == pytest.approx(6 * 32 * 124 * 2.0 * 64 ** 3)
    # other head dims: fp32 recurrences on the ALUs
    assert bench.stage_model("ut_prep", 1, 1, 4096, 32)[1] == "alu"

"""The rho-aware weight-group selector (apex_select_weight_group), host only.

"APEX4: Efficient Pure W4A4 LLM Inference via Intra-SM Compute Rebalancing" (abstract): the
tensor-core to CUDA-core throughput ratio rho governs the group-dequantisation bottleneck --
the W4A4-g128 kernel speeds up on the RTX 3090 (rho = 16) but degrades on the A100 (rho = 64)
in compute-bound cases, which the mixed-granularity mode recovers.  The selector's speed-side
rule is checked against those statements and against a table measured on a B200
(tests/data/weight_group_sweep_b200.json, written from `bench.py --sweep`).
"""
import json
import os

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def apex():
    import group_quantized_w4a4_b200 as m
    m.load_library()
    return m


B200_FP32_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12   # 128 fp32 fma per SM per clock
B200_HBM_GBS = 6551.4                                # measured copy bandwidth


def test_low_rho_keeps_128_wide_groups(apex):
    # rho = 8 (L40S), 16 (RTX 3090, A40): g128 is the viable kernel, even compute-bound
    for rho in (8, 16):
        for M in (16, 4096, 65536):
            assert apex.apex_select_weight_group(M, 8192, 8192, rho, 300.0) == 128


def test_high_rho_compute_bound_takes_per_channel_groups(apex):
    # rho = 64 (A100): compute-bound W4A4-g128 degrades; the coarse mode is chosen there ...
    for M in (1024, 4096, 65536):
        assert apex.apex_select_weight_group(M, 8192, 8192, 64, 300.0) == 8192
    # ... but not where the weight stream bounds the GEMM (a few tokens)
    for M in (1, 16, 64):
        assert apex.apex_select_weight_group(M, 8192, 8192, 64, 300.0) == 128


def test_ridge_sets_the_boundary(apex):
    # intensity of M x 8192 x 8192 with packed operands is about 4*M ops per byte for small M
    assert apex.apex_select_weight_group(100, 8192, 8192, 64, 500.0) == 128
    assert apex.apex_select_weight_group(200, 8192, 8192, 64, 500.0) == 8192
    assert apex.apex_select_weight_group(200, 8192, 8192, 64, 1000.0) == 128


def test_invalid_arguments_return_zero(apex):
    assert apex.apex_select_weight_group(0, 8192, 8192, 64, 300.0) == 0
    assert apex.apex_select_weight_group(16, 8192, 8000, 64, 300.0) == 0
    assert apex.apex_select_weight_group(16, 8192, 8192, 0, 300.0) == 0
    assert apex.apex_select_weight_group(16, 8192, 8192, 64, -1.0) == 0


def test_choice_is_the_fastest_measured_mode_on_b200(apex):
    with open(os.path.join(HERE, "data", "weight_group_sweep_b200.json")) as f:
        table = json.load(f)
    i8 = table["int8_peak_tops"]
    rho = i8 / B200_FP32_TFLOPS                # about 41 with the measured int8 rate
    ridge = i8 * 1e12 / (B200_HBM_GBS * 1e9)   # int8 ops per HBM byte
    for M, times in table["gemm_us"].items():
        gw = apex.apex_select_weight_group(int(M), 8192, 8192, rho, ridge)
        assert gw in (128, 8192)
        best = min(times.values())
        assert times[str(gw)] <= 1.03 * best, (M, gw, times)
    # the table itself shows the effect the selector relies on: per-channel groups win big
    # once compute-bound, and nothing is lost at a few tokens
    t = table["gemm_us"]
    assert t["4096"]["8192"] < 0.8 * t["4096"]["128"]
    assert abs(t["16"]["8192"] - t["16"]["128"]) < 0.05 * t["16"]["128"]

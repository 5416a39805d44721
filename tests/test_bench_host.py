"""Host-side logic of bench.py on CPU: the counted FLOPs, the workload table,
the machine-read profile lines and the reference arm's JSON line."""
import json
import math

import pytest

import bench
import seeded_inputs as si


def test_forward_flops_match_the_stated_counts():
    # additive: 4 N^2 d + 2 N^2 R per head, halved when causal
    assert bench.flops(1, 1, 8, 4, 2, False) == 4 * 64 * 4 + 2 * 64 * 2
    assert bench.flops(2, 3, 8, 4, 2, True) == 6 * (4 * 64 * 4 + 2 * 64 * 2) / 2
    # multiplicative: 2 N^2 d R + 2 N^2 d
    assert bench.flops(1, 1, 8, 4, 3, False, multiplicative=True) == 2 * 64 * 4 * 3 + 2 * 64 * 4


def test_backward_flops_count_the_five_products():
    N, d, R = 16, 8, 4
    s_, dq_, dk_ = (2 * N * N * (d + R),) * 3          # S, dQ', dK' over the concatenated width
    dp_, dv_ = 2 * N * N * d, 2 * N * N * d            # dP, dV
    assert bench.bwd_flops(1, 1, N, d, R, False) == s_ + dq_ + dk_ + dp_ + dv_
    fixed = 2 * N * N * (d + R) + 4 * 2 * N * N * d   # no factor gradients: dQ and dK over d only
    assert bench.bwd_flops(1, 1, N, d, R, False, factor_grads=False) == fixed
    assert bench.bwd_flops(2, 2, N, d, R, True) == 4 * (s_ + dq_ + dk_ + dp_ + dv_) / 2


@pytest.mark.parametrize("idx", range(len(si.CONFIGS)))
def test_every_workload_has_positive_counted_flops(idx):
    c = bench.workload(idx)
    assert c["flops"] > 0 and c["index"] == idx
    json.dumps(bench.config_json(c, "n/a"))


def test_profile_lines_match_current_sources_or_are_ignored():
    # the forward headline and the backward line read DRAM traffic only from a
    # summary taken on the current kernel sources
    for idx in (1, 7):
        t = bench.profiled_traffic(idx)
        assert t is None or (t > 0 and math.isfinite(t))
    assert bench.profiled_traffic(0) is None  # no summary for the fp32 workload


@pytest.mark.parametrize("cfg", [1, 7])
def test_reference_arm_json_line(cfg):
    out = bench.run_reference(bench.parse_args(["--impl", "reference", "--config", str(cfg), "--steps", "1",
                                                "--warmup", "1"]), 0, 1)
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in out, key
    assert out["impl"] == "reference" and out["value"] > 0
    assert out["e2e"]["h2d_bytes_per_step"] == 0 and out["e2e"]["d2h_bytes_per_step"] == 0
    assert out["cpu_baseline"]["kind"] == "oracle" and out["cpu_baseline"]["value"] == out["value"]
    json.dumps(out)


def test_fp32_peak_and_exp2_counts():
    """The fp32 path's roofline peak (148 SMs x 128 FMA lanes x 2 FLOP per
    clock) and the exp2 counts behind the special-function-unit floor."""
    assert abs(bench.fp32_fma_peak_tflops({"sm_max_mhz": 1965.0}) - 74.45) < 0.01
    assert abs(bench.fp32_fma_peak_tflops(None) - 74.45) < 0.01
    c1 = bench.workload(1)  # causal: half of B H N^2
    assert bench.exp2_elements(c1) == 8 * 12 * 2048 * 2048 / 2
    c3 = bench.workload(3)  # no mask: all of them
    assert bench.exp2_elements(c3) == 4 * 8 * 4096 * 4096

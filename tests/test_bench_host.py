"""Host-side bookkeeping of bench.py (no GPU): the roofline peak rule and the forward's
exponential-unit roof, checked against numbers worked out by hand."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from attention_kl_divergence_02_b200 import inputs  # noqa: E402

PEAKS = {"bf16_tflops": 1694.5, "bf16_tflops_sustained": 1420.9}


def test_burst_peak_for_a_short_region_at_the_maximum_clock():
    peak, label, why = bench.choose_peak(PEAKS, "measured", 0.25, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0})
    assert peak == 1694.5 and "burst" in label and "0.25 s" in why


@pytest.mark.parametrize("timed_s, clk", [
    (4.0, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0}),      # seconds-long region
    (0.25, {"sm_mhz": 1380.0, "sm_max_mhz": 1965.0}),     # clock held below its maximum
    (0.25, {"sm_mhz": None, "sm_max_mhz": None}),         # no clock record
])
def test_sustained_peak_otherwise(timed_s, clk):
    peak, label, why = bench.choose_peak(PEAKS, "measured", timed_s, clk)
    assert peak == 1420.9 and "sustained" in label and why


def test_effective_clock_decides_over_the_sampled_one():
    """nvidia-smi may report the maximum clock while the power cap holds the SMs lower; the
    clock probe's cycles-over-time figure then decides."""
    clk = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "sm_mhz_effective": 1725.0}
    peak, label, why = bench.choose_peak(PEAKS, "measured", 0.25, clk)
    assert peak == 1420.9 and "sustained" in label and "1725" in why and "power cap" in why
    clk["sm_mhz_effective"] = 1950.0
    peak, label, why = bench.choose_peak(PEAKS, "measured", 0.25, clk)
    assert peak == 1694.5 and "clock probe" in why


def test_exp_roofline_of_the_headline_forward():
    w = inputs.WORKLOADS["headline"]
    # 16 ex2 per clock per SM on 148 SMs at 2000 MHz -> 4.736e12 exp2/s; the forward spends 2
    # per unmasked pair (causal pairs halved: 32 * 16384^2 / 2 = 4.295e9 pairs), 75 % of them on
    # the exponential unit -> 6.442e9 exp2 -> 1.3602 ms; over a 2.72 ms forward: 0.5001
    rates = {"mufu_ex2": {"per_sm_per_clk": 16.0}, "fma_poly": {"per_sm_per_clk": 12.0}, "sms": 148}
    r = bench.exp_roofline(w, 2.72, rates, 2000.0)
    assert r["exps_per_call"] == 2 * 32 * 16384 * 16384 / 2
    assert abs(r["t_mufu_ms"] - 0.75 * r["exps_per_call"] / (16 * 148 * 2e9) * 1e3) < 1e-9
    assert abs(r["frac"] - 1.36022 / 2.72) < 1e-4
    assert abs(r["t_all_on_mufu_ms"] - r["t_mufu_ms"] / 0.75) < 1e-9

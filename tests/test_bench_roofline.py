"""Host-side checks of bench.py's roofline bookkeeping (no GPU): the algorithmic work per
kernel class, the peak each one is divided by, and which kernels carry measured DRAM
traffic.  The numbers are the 4096 x 4096 layer's (n = 2048 tokens, 4-bit g128)."""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

BF16 = 1635.2     # TFLOP/s
TF32 = 744.0      # TFLOP/s
HBM = 6535.7      # GB/s


def _roof(kernel_ms):
    launches = {k: 1 for k in kernel_ms}
    return bench.kernel_rooflines(kernel_ms, launches, HBM, BF16, "measured", tf32=TF32)


def test_trailing_updates_are_measured_against_a_third_of_bf16():
    r = _roof({"trailing_update": 0.4, "trailing_update_sb": 0.2})["trailing_update"]
    # sum over the 31 block ends of 2 d_out (d_in - e) 128 flops
    flops = sum(2.0 * 4096 * (4096 - 128 * (b + 1)) * 128 for b in range(31))
    assert flops == pytest.approx(66.57e9, rel=1e-3)
    assert r["peak"] == pytest.approx(BF16 / 3)
    assert r["achieved"] == pytest.approx(flops / 0.6e-3 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"])


def test_factorization_counts_two_thirds_d_cubed_against_a_third_of_tf32():
    r = _roof({"chol_dag": 1.4})["chol_dag"]
    assert r["peak"] == pytest.approx(TF32 / 3)
    assert r["achieved"] == pytest.approx(2.0 / 3.0 * 4096 ** 3 / 1.4e-3 / 1e12)
    # the only kernel whose DRAM traffic is reported: measured on the current code
    assert r["traffic"] == 39034112 + 311716096


def test_hessian_and_column_loop_units():
    r = _roof({"hessian_syrk": 0.1, "colloop": 0.5})
    h, c = r["hessian_syrk"], r["colloop"]
    assert h["unit"] == "TFLOP/s" and h["peak"] == BF16
    assert h["achieved"] == pytest.approx(2048 * 4096 * 4097 / 0.1e-3 / 1e12)
    assert c["unit"] == "GB/s" and c["peak"] == HBM and c["bound"] == "hbm"
    # W read once, codes and group metadata written
    col_bytes = 4.0 * 4096 * 4096 + 0.5 * 4096 * 4096 + (2 + 0.5) * 4096 * 32
    assert c["achieved"] == pytest.approx(col_bytes / 0.5e-3 / 1e9)
    assert h["traffic"] is None and c["traffic"] is None


def test_without_a_measured_tf32_peak_the_nominal_ratio_is_used():
    r = bench.kernel_rooflines({"chol_dag": 1.0}, {"chol_dag": 1}, HBM, BF16, "measured")["chol_dag"]
    assert r["peak"] == pytest.approx(BF16 * 1.1 / 2.25 / 3)


def test_end_to_end_bound_is_the_sum_of_the_stage_bounds():
    assert bench.END_TO_END_BOUND_MS == pytest.approx((21.0 + 168.1 + 244.3 + 11.6) / 1e3, abs=1e-3)

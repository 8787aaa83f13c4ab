"""Host-side arithmetic of bench.py's report (no GPU): the mask-stage
roofline object and the per-scorer launch counts."""
import math

import bench
import workloads as W


def test_mask_roofline_sampling_counts_one_exp2_per_score_element():
    w = W.PRESETS["wan14b"]
    r = bench.mask_roofline(w, mask_ms=10.0, hbm=6541.5, clocks={"sm_mhz": 1800.0}, elem=2)
    exps = (-(-75600 // 128) * 8) * 75600 * 40
    assert r["bound"] == "alu" and r["unit"] == "Gexp2/s"
    assert math.isclose(r["achieved"], exps / 10e-3 / 1e9)
    assert math.isclose(r["peak"], 16 * 148 * 1800e6 / 1e9)
    assert math.isclose(r["frac"], r["achieved"] / r["peak"])


def test_mask_roofline_antidiag_causal_halves():
    w = W.PRESETS["qwen2.5vl"]
    r = bench.mask_roofline(w, mask_ms=1.0, hbm=6541.5, clocks=None, elem=2)
    n = 32768 // 8
    assert math.isclose(r["achieved"], n * n * 28 * 0.5 / 1e-3 / 1e9)


def test_mask_roofline_meankey_reads_q_and_k_once():
    w = W.PRESETS["wan14b"].replace(mask_mode="meankey")
    r = bench.mask_roofline(w, mask_ms=2.0, hbm=6541.5, clocks=None, elem=2)
    byts = (40 + 40) * 75600 * 128 * 2
    assert r["bound"] == "hbm" and math.isclose(r["achieved"], byts / 2e-3 / 1e9)
    assert bench.mask_roofline(W.PRESETS["tiny"], 1.0, 6541.5, None, 4) is None


def test_launch_counts_per_scorer():
    assert bench.MASK_KERNELS == {"sample": 2, "antidiag": 2, "meankey": 5, "given": 0}

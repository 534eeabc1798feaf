"""bench.py's host-side arithmetic (CPU only): the GEMM roofline object and its choice of
bound, checked against numbers worked out by hand."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

PEAKS = {"hbm_gbs": 6443.2, "tflops": 1671.8, "tflops_sustained": 1410.0, "source": "measured"}


def test_tensor_bound_at_4096_tokens():
    H, T = 12288, 4096
    # 12 layers x 4 GEMMs in 10 steps taking 1430 ms of GEMM time in all
    r = bench.gemm_roofline(H, T, 2, 480, 1430.0, PEAKS, 123)
    flops_per_launch = 24 * H * H * T / 4           # 6 H^2 T = 3.71e12
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["traffic"] == 123
    assert r["algorithmic_flops_per_launch"] == pytest.approx(3.7108517e12, rel=1e-6)
    assert r["achieved"] == pytest.approx(flops_per_launch * 480 / 1.430 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / 1410.0)
    assert r["ms_per_launch"] == pytest.approx(1430.0 / 480)


def test_weight_streaming_bound_at_32_tokens():
    H, T = 12288, 32
    # 2 T flop per weight element = T = 32 flop per 16-bit weight byte, under the ridge
    # 1410e12 / 6443.2e9 = 218.8
    r = bench.gemm_roofline(H, T, 2, 40, 6.4, PEAKS, 123)
    bytes_per_launch = 12 * H * H * 2 / 4            # 906 MB: one quarter of a layer's weights
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["traffic"] is None
    assert r["algorithmic_bytes_per_launch"] == pytest.approx(905969664)
    assert r["achieved"] == pytest.approx(bytes_per_launch * 40 / 0.0064 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6443.2)


def test_bound_switches_at_the_ridge():
    H = 1024
    ridge = 1410.0e12 / 6443.2e9                      # flop per byte
    below, above = int(ridge), int(ridge) + 1          # T flop per 16-bit weight byte
    assert bench.gemm_roofline(H, below, 2, 4, 1.0, PEAKS, None)["bound"] == "hbm"
    assert bench.gemm_roofline(H, above, 2, 4, 1.0, PEAKS, None)["bound"] == "tensor"
    assert bench.gemm_roofline(H, 100, 2, 0, 0.0, PEAKS, None)["achieved"] is None

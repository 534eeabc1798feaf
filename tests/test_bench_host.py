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


def test_step_roofline_matches_the_worked_figures():
    # 12 layers, batch 32 of length 128 at H 12288: 1.783e14 flop; 126.4 ms at 1410 TFLOP/s
    r = bench.step_roofline(12288, 12, [128] * 32, 2, 148.5, PEAKS)
    assert r["algorithmic_flop"] == 12 * (24 * 12288 ** 2 * 4096 + 4 * 12288 * 32 * 128 * 129 // 2)
    assert r["algorithmic_flop"] == pytest.approx(1.783e14, rel=1e-3)
    assert r["bound"] == "tensor" and r["t_roof_ms"] == pytest.approx(126.4, rel=2e-3)
    assert r["frac"] == pytest.approx(r["t_roof_ms"] / 148.5)
    # one layer at T = 32: the weights (3.62 GB) bound it, 0.562 ms at 6443 GB/s
    r = bench.step_roofline(12288, 1, [32], 2, 0.727, PEAKS)
    assert r["bound"] == "hbm" and r["weight_bytes"] == 12 * 12288 ** 2 * 2
    assert r["t_roof_ms"] == pytest.approx(0.5624, rel=2e-3)


def test_fractions_of_burst_and_datasheet():
    r = bench.gemm_roofline(12288, 4096, 2, 480, 1430.0, PEAKS, None)
    assert r["frac_of_burst"] == pytest.approx(r["achieved"] / 1671.8)
    assert r["frac_of_datasheet"] == pytest.approx(r["achieved"] / 2250.0)
    r = bench.gemm_roofline(12288, 32, 2, 40, 6.4, PEAKS, None)
    assert r["frac_of_datasheet"] == pytest.approx(r["achieved"] / 8000.0)


def test_batching_cost_table_interpolates_the_measured_points():
    pts = [(1024, 0.04), (256, 0.016), (4096, 0.15), (16384, 0.63)]
    t = bench.cost_table(pts, 64, 256)
    assert t[7][31] == pytest.approx(0.016)                 # 8 x 32 = 256 tokens: a measured point
    assert t[0][0] == pytest.approx(0.016)                  # below the first point: its cost
    assert t[31][127] == pytest.approx(0.15)                # 32 x 128 = 4096
    assert t[15][159] == pytest.approx(0.04 + (2560 - 1024) / (4096 - 1024) * (0.15 - 0.04))   # 16 x 160
    assert t[63][255] == pytest.approx(0.63)
    # monotone in the padded token count, as the measured points are
    flat = sorted(((b + 1) * (s + 1), t[b][s]) for b in range(64) for s in range(256))
    assert all(flat[i][1] <= flat[i + 1][1] + 1e-15 for i in range(len(flat) - 1))


def test_batching_pool_has_every_position_a_batch_claims():
    """The dynamic-batching section cuts batches of up to 256 positions from the workload's
    padded input; a workload padded to 64 positions (gpt3_layer) repeats its positions so that
    no batch is shorter than the pad length passed with it."""
    import torch
    pool = torch.arange(2 * 64 * 3, dtype=torch.float32).reshape(2, 64, 3)
    ext = bench.extend_positions(pool, 256)
    assert ext.shape == (2, 256, 3) and ext.is_contiguous()
    assert torch.equal(ext[:, :64], pool) and torch.equal(ext[:, 64:128], pool)
    assert bench.extend_positions(pool, 64) is pool


def test_binding_refuses_tensors_smaller_than_the_call_needs():
    """The C ABI takes sizes on trust; the binding checks every tensor argument against the
    bytes the call will touch before anything reaches a kernel."""
    import torch
    from padding_free_varlen_b200 import capi
    cfg = capi.make_config(256, 2, 1024, capi.ENERGON_F16)
    w = capi.energon_layer_weights(*([0] * 13))
    small = torch.zeros((2, 4, 256), dtype=torch.float16)          # 4 positions, the call claims 8
    with pytest.raises(ValueError, match="padded_in"):
        capi.energon_stack_forward(cfg, [w], 1, small, torch.zeros(2, dtype=torch.int32), 2, 8, 1, small,
                                   torch.zeros(1, dtype=torch.int32), torch.zeros(1, dtype=torch.uint8), 1, stream=0)
    with pytest.raises(ValueError, match="packed"):
        capi.energon_rce_remove_padding(torch.zeros((2, 8, 16), dtype=torch.float16), torch.zeros(3, dtype=torch.int32),
                                        2, 8, 16, 2, torch.zeros((8, 16), dtype=torch.float16), stream=0)


def test_gemm_traffic_record_applies_to_its_own_workload_only(monkeypatch):
    """The committed DRAM count was taken on one launch configuration (the half-padded GPT-3
    stack); the roofline of another workload must not report it."""
    import json
    with open(os.path.join(os.path.dirname(os.path.abspath(bench.__file__)), "profiles", "gemm_tc_traffic.json")) as f:
        rec = json.load(f)
    monkeypatch.setattr(bench, "gemm_device_code_hash", lambda: rec["device_code_sha256_16"])
    assert bench.traffic_from_profile(rec["workload"]) == rec["dram_bytes_per_launch_scaled"]
    assert bench.traffic_from_profile("gpt3_stack_dynbatch") is None
    monkeypatch.setattr(bench, "gemm_device_code_hash", lambda: "0" * 16)
    assert bench.traffic_from_profile(rec["workload"]) is None

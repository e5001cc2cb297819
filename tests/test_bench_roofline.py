"""bench.py's roofline object for the GEMM launch (host logic, no GPU):
which kernel a workload runs and which bound its algorithmic bytes and
flops put it under at the measured peaks."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

HBM, FP4 = 6551.4, 6621.2   # GB/s, TFLOP/s


def test_kernel_by_token_count():
    assert bench.gemm_kernel_name(1) == "w4a4_linear_small_kernel"
    assert bench.gemm_kernel_name(64) == "w4a4_linear_small_kernel"
    assert bench.gemm_kernel_name(65) == "w4a4_linear_kernel"
    assert bench.gemm_kernel_name(128) == "w4a4_linear_kernel"
    assert bench.gemm_kernel_name(129) == "w4a4_linear_pair_kernel"
    assert bench.gemm_kernel_name(4352) == "w4a4_linear_pair_kernel"


def test_few_tokens_are_hbm_bound():
    # out-projection at 64 tokens: 9.94 MB of operands and output against
    # 1.95 GFLOP -> the bytes take longer at the measured peaks
    r = bench.gemm_roofline(64, 9938946, 1950351360, 0.015, HBM, FP4, "measured", None)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["kernel"] == "w4a4_linear_small_kernel"
    assert abs(r["achieved"] - 9938946 / 15e-6 / 1e9) < 0.1
    assert abs(r["frac"] - r["achieved"] / HBM) < 1e-4
    assert r["algorithmic_bytes_per_launch"] == 9938946


def test_dit_shape_is_tensor_bound():
    # qkv at 4352 tokens: 398 GFLOP against 139 MB
    r = bench.gemm_roofline(4352, 138662914, 397871677440, 0.121, HBM, FP4, "measured",
                            90749184.0)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["kernel"] == "w4a4_linear_pair_kernel"
    assert abs(r["achieved"] - 397871677440 / 121e-6 / 1e12) < 0.1
    assert abs(r["frac"] - r["achieved"] / FP4) < 1e-4
    assert r["traffic"] == 90749184.0
    assert r["avg_launch_ms"] == 0.121


def test_flops_per_step_counts_both_products():
    M, K, N, R = 4352, 3840, 11520, 128
    assert bench.flops_per_step(M, K, N, R) == 2 * M * N * K + 2 * M * R * (K + N)
    assert bench.flops_per_step(M, K, N, 0) == 2 * M * N * K

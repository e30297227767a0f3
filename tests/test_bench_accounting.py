"""The bench's algorithmic work and byte counts (the numerators of its roofline
fractions), pinned to values worked out by hand from the workload sizes.

Per-launch figures the bench reports (`roofline.algorithmic_per_launch`) are the
means of these over a workload's layers."""
import dataclasses
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
from w4a4_rank_assisted_b200.synth import WORKLOADS  # noqa: E402


def test_gemm_bytes_flux_mlp_up():
    # M = 4608, K = 3072, N = 12288, r = 4, groups of 64 (48 groups):
    # x codes 7 077 888 + x scales 884 736 + U 73 728
    # + w codes 18 874 368 + w scales 2 359 296 + L2 98 304 + Y (bf16) 113 246 208
    spec = WORKLOADS["flux_block_r4"][1]
    assert (spec.M, spec.K, spec.N, spec.r, spec.group) == (4608, 3072, 12288, 4, 64)
    assert bench.layer_gemm_bytes(spec) == 142_614_528


def test_gemm_bytes_mean_over_the_flux_block():
    # qkv 108 969 984, MLP up 142 614 528, MLP down 81 494 016
    specs = WORKLOADS["flux_block_r4"]
    got = [bench.layer_gemm_bytes(s) for s in specs]
    assert got == [108_969_984, 142_614_528, 81_494_016]
    assert sum(got) // 3 == 111_026_176


def test_bias_is_read_once():
    spec = WORKLOADS["flux_block_r4"][1]
    with_bias = dataclasses.replace(spec, bias=True)
    assert bench.layer_gemm_bytes(with_bias) - bench.layer_gemm_bytes(spec) == 2 * spec.N
    one = WORKLOADS["qwen3_8b_m1"][0]
    assert bench.layer_fused_bytes(dataclasses.replace(one, bias=True)) - bench.layer_fused_bytes(one) == 2 * one.N


def test_groups_of_128_and_padded_k():
    # K = 200 pads to 256 at groups of 128: 2 groups, Kp = 256
    spec = dataclasses.replace(WORKLOADS["qwen3_8b_m1_g128"][0], M=3, K=200, N=16, r=2)
    # x codes 384 + x scales 24 + U 24 + w codes 2048 + w scales 128 + L2 64 + Y 96
    assert bench.layer_gemm_bytes(spec) == 2768


def test_layer_ops():
    # 2MNK + 2MKr + 2MNr for M = 3, K = 64, N = 8, r = 2
    spec = dataclasses.replace(WORKLOADS["flux_block_r4"][0], M=3, K=64, N=8, r=2)
    assert bench.layer_ops(spec) == 3072 + 768 + 96


def test_activation_bytes_flux_mlp_up():
    # X 28 311 552 + codes 7 077 888 + scales 884 736 + U 73 728 + s 12 288 + L1 24 576
    assert bench.layer_act_bytes(WORKLOADS["flux_block_r4"][1]) == 36_384_768


def test_single_launch_bytes_qwen3_8b_m1():
    # gate/up: X 8 192 + s 16 384 + L1 32 768 + w codes 25 165 824 + w scales 3 145 728 + L2 98 304 + Y 24 576
    # down:    X 24 576 + s 49 152 + L1 98 304 + w codes 25 165 824 + w scales 3 145 728 + L2 32 768 + Y 8 192
    got = [bench.layer_fused_bytes(s) for s in WORKLOADS["qwen3_8b_m1"]]
    assert got == [28_491_776, 28_524_544]
    assert sum(got) // 2 == 28_508_160

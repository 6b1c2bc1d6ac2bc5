"""Host-side pieces of the benchmark (no GPU): the algorithmic byte and flop
counts the roofline divides by, the launch count it reports, and the argument
parser."""
import bench
from combine_moe_route_12_b200.workload import WORKLOADS


def test_algorithmic_counts_bf16_qwen3_shape():
    wl = WORKLOADS["qwen3_30b_a3b"]
    N = 32768
    a = bench.algorithmic(wl, [N], [128], tokens_read=4096)
    H, I, T, b = 2048, 768, 4096, 2
    assert a["N"] == N
    assert a["ffn_flops"] == 6.0 * H * I * N
    # weights of 128 experts once, the receive rows, h written and read, y written
    assert a["ffn_bytes"] == 128 * 3 * H * I * b + N * H * b + 2 * N * I * b + N * H * b
    assert a["permute_bytes"] == T * H * b + N * H * b
    assert a["combine_bytes"] == N * H * b + T * H * b


def test_algorithmic_counts_only_needed_x_rows_and_fp8_bytes():
    wl = WORKLOADS["skew_capacity"]
    full = bench.algorithmic(wl, [14137], [14], tokens_read=None)
    part = bench.algorithmic(wl, [14137], [14], tokens_read=8812)
    assert full["permute_bytes"] - part["permute_bytes"] == (16384 - 8812) * 2048 * 2
    f8 = bench.algorithmic(WORKLOADS["qwen3_30b_a3b_fp8"], [32768], [128], tokens_read=4096)
    bf = bench.algorithmic(WORKLOADS["qwen3_30b_a3b"], [32768], [128], tokens_read=4096)
    # one byte per weight (+ a scale byte per weight row) instead of two
    H, I = 2048, 768
    assert f8["ffn_flops"] == bf["ffn_flops"]
    w8 = 128 * (3 * H * I + 2 * I + H)
    assert f8["ffn_bytes"] == w8 + 32768 * H + 32768 * I * (2 * 2 + 2) + 32768 * H * 2
    # the fused quantise-and-permute reads the kept tokens' bf16 rows, writes codes
    assert f8["permute_bytes"] == 4096 * H * 2 + 32768 * H


def test_kernels_per_step():
    assert bench.kernels_per_step(WORKLOADS["qwen3_30b_a3b"]) == 1 + 2 + 6
    assert bench.kernels_per_step(WORKLOADS["skew_capacity"]) == 1 + 4 + 6
    assert bench.kernels_per_step(WORKLOADS["dsv3_prefill"]) == 1 + 2 + 2 * 6
    assert bench.kernels_per_step(WORKLOADS["dsv3_grouped"]) == 1 + 2 + 6 + 3
    assert bench.kernels_per_step(WORKLOADS["qwen3_30b_a3b_fp8"]) == 1 + 2 + 6 + 1
    assert bench.kernels_per_step(WORKLOADS["dsv3_prefill_fp8"]) == 1 + 2 + 2 * (6 + 1)


def test_default_arguments_finish_within_minutes():
    a = bench.parse_args([])
    assert a.gpus == 1 and a.config == "qwen3_30b_a3b" and a.impl == "ours"
    assert a.warmup >= 3 and a.steps <= 100
    assert not a.backward

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
    # no capacity: the clip is one pass
    assert bench.kernels_per_step(WORKLOADS["qwen3_30b_a3b"]) == 1 + 1 + 6
    assert bench.kernels_per_step(WORKLOADS["skew_capacity"]) == 1 + 4 + 6
    assert bench.kernels_per_step(WORKLOADS["dsv3_prefill"]) == 1 + 1 + 2 * 6
    assert bench.kernels_per_step(WORKLOADS["dsv3_grouped"]) == 1 + 1 + 6 + 3
    assert bench.kernels_per_step(WORKLOADS["qwen3_30b_a3b_fp8"]) == 1 + 1 + 6 + 1
    assert bench.kernels_per_step(WORKLOADS["dsv3_prefill_fp8"]) == 1 + 1 + 2 * (6 + 1)
    assert bench.kernels_per_step(WORKLOADS["qwen3_30b_a3b"].with_(capacity=0)) == 1 + 2 + 6


def test_default_arguments_finish_within_minutes():
    a = bench.parse_args([])
    assert a.gpus == 1 and a.config == "dsv3_prefill" and a.impl == "ours"
    assert a.warmup >= 3 and a.steps <= 100
    assert not a.backward


def test_reference_steps_are_ep_aligned_sub_batches():
    for name in ("tiny", "qwen3_30b_a3b", "skew_capacity", "dsv3_prefill", "dsv3_decode"):
        wl = WORKLOADS[name]
        ts = bench.reference_tokens(wl, 2.0)
        assert ts % wl.ep == 0 and wl.ep <= ts <= wl.T


def test_ffn_roofline_picks_the_binding_roof():
    peaks = {"hbm_gbs": 6500.0, "bf16_tflops": 1650.0, "bf16_tflops_sustained": 1370.0}
    wl = WORKLOADS["dsv3_prefill"]
    # two chunks: every expert's weights twice, HBM-bound
    a2 = bench.algorithmic(wl, [32768, 32768], [256, 256], tokens_read=8192)
    r2 = bench.ffn_roofline(wl, a2, 8.0, peaks, "measured", None)
    assert r2["bound"] == "hbm" and abs(r2["frac"] - r2["hbm_frac"]) < 1e-12
    # one chunk: one weight read; at 231 flop/B it still sits below this ridge
    # (254 flop/B), and above a lower one, where the tensor roof binds
    a1 = bench.algorithmic(wl.with_(n_chunks=1), [65536], [256], tokens_read=8192)
    assert 230 < a1["ffn_flops"] / a1["ffn_bytes"] < 232
    r1 = bench.ffn_roofline(wl.with_(n_chunks=1), a1, 6.0, peaks, "measured", None)
    assert r1["bound"] == "hbm"
    low = dict(peaks, bf16_tflops=1400.0)
    r1 = bench.ffn_roofline(wl.with_(n_chunks=1), a1, 6.0, low, "measured", None)
    assert r1["bound"] == "tensor" and abs(r1["frac"] - r1["tensor_frac"]) < 1e-12
    assert r1["tensor_frac_sustained"] > r1["tensor_frac"]


def test_block_scaled_fp8_counts():
    mx = WORKLOADS["dsv3_prefill_mxfp8"]
    bf = WORKLOADS["dsv3_prefill"]
    # x quantised inside the permute, h inside GEMM1: the bf16 layer's launches
    assert bench.kernels_per_step(mx) == bench.kernels_per_step(bf)
    a = bench.algorithmic(mx, [32768, 32768], [256, 256], tokens_read=8192)
    H, I, N = 7168, 2048, 65536
    # one byte per weight plus a scale byte per 32; h's codes and scales written and read
    assert a["ffn_bytes"] == 2 * 256 * 3 * H * I * 33 // 32 + N * H * 33 // 32 + 2 * N * I * 33 // 32 + N * H * 2
    assert a["permute_bytes"] == 8192 * H * 2 + N * H * 33 // 32


def test_oracle_rows_visits_every_row_once_in_threads():
    """The CPU baseline's threaded runner calls the row function once per row,
    whatever the thread count, and only with the row's own expert."""
    import threading
    rows_by_expert = {e: list(range(10 * e, 10 * e + e % 4)) for e in range(32)}
    for threads in (1, 3, 8):
        seen = []
        lock = threading.Lock()

        def row(p, e):
            with lock:
                seen.append((p, e))
        bench.oracle_rows(row, rows_by_expert, threads)
        want = sorted((p, e) for e, ps in rows_by_expert.items() for p in ps)
        assert sorted(seen) == want
    assert bench.host_threads() >= 1

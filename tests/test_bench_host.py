"""Host-side arithmetic of bench.py that every roofline figure rests on: the
algorithmic bytes of a decode call, the step total, and the per-launch DRAM
traffic looked up from the committed ncu summaries."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_gemv_bytes_is_codes_scales_biases_and_vectors():
    # 4-bit, gs 64: 0.5 B of codes + 4 / 64 B of bf16 scale and bias per weight = 0.5625 B
    N, K = 128256, 2048
    assert bench.gemv_bytes(N, K, 4) == N * K * 9 // 16 + 2 * K + 2 * N
    assert bench.gemv_bytes(N, K, 4) == 148011520             # the lm_head figure the profiles quote
    assert bench.gemv_bytes(8192, 2048, 8, M=4) == 8192 * 2048 + 4 * 8192 * 32 + 2 * 4 * 2048 + 2 * 4 * 8192


def test_step_bytes_sum_the_decode_layers():
    assert bench.STEP_BYTES == sum(bench.gemv_bytes(N, K, b) for N, K, b in bench.DECODE)
    assert bench.STEP_BYTES > 126 * 2 ** 20                   # the step's inputs exceed the 126 MB L2


def test_traffic_entries_resolve():
    assert bench.traffic_for("k_gemv_pipe_lmhead") == 154382080
    assert bench.traffic_for("k_tc2_w8a8_m4096") == 524822784
    assert bench.traffic_for("no_such_kernel") is None
    # every entry names a summary that exists
    with open(os.path.join(ROOT, "profiles", "traffic.txt")) as f:
        for line in f:
            parts = line.split()
            if parts and not parts[0].startswith("#"):
                assert os.path.exists(os.path.join(ROOT, "profiles", parts[2])), parts[2]


def test_job_throughput_scales_with_ranks():
    assert bench.job_gbs(1, 10 ** 9, 1, 1000.0) == 1.0
    assert bench.job_gbs(8, 10 ** 9, 1, 1000.0) == 8.0

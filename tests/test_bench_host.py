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
    # the lm_head's traffic is its algorithmic bytes within 10 % (no re-reads)
    assert abs(bench.traffic_for("k_gemv_pipe_lmhead") / bench.gemv_bytes(*bench.LMHEAD) - 1) < 0.10
    assert bench.traffic_entry("k_tc2_w8a8_m4096")[1] == "gemm_tc2_w8a8_14336x4096_m4096.md"
    assert bench.traffic_for("no_such_kernel") is None
    # every entry names a summary that exists
    with open(os.path.join(ROOT, "profiles", "traffic.txt")) as f:
        for line in f:
            parts = line.split()
            if parts and not parts[0].startswith("#"):
                assert os.path.exists(os.path.join(ROOT, "profiles", parts[2])), parts[2]


def test_every_traffic_key_the_bench_quotes_resolves():
    """Every traffic key bench.py passes to a roofline object has a committed ncu figure, so
    no `traffic` in the bench line is null."""
    import re
    src = open(os.path.join(ROOT, "bench.py")).read()
    keys = set(re.findall(r'traffic_for\("(k_[A-Za-z0-9_]+)"\)', src))
    keys |= set(re.findall(r'"(k_tc2_affine[0-9a-z_]+)"', src))
    # every plain key on a line that passes one (f-strings are expanded below)
    for line in src.splitlines():
        if "traffic_key=" in line:
            keys |= set(re.findall(r'(?<![{f])"(k_[A-Za-z0-9_]+)"', line))
    for M in bench.PREFILL_M:
        keys.add(f"k_tc2_affine4_m{M}")
    for fmt in ("w4a8", "w8a8"):
        for M in bench.INT8_M:
            keys.add(f"k_gemv_pipe_i8w8_m{M}" if fmt == "w8a8" and M <= 8 else f"k_tc2_{fmt}_m{M}")
    assert len(keys) > 20, keys
    missing = sorted(k for k in keys if bench.traffic_for(k) is None)
    assert not missing, missing
    # the fused MLP's traffic is the sum of its two launches
    assert bench.mlp_traffic() == bench.traffic_for("k_gemv_pipe_dual") + bench.traffic_for("k_gemv_pipe_silu")


def test_token_tile_labels():
    assert [bench.tc2_tile(M) for M in (9, 32, 33, 64, 65, 128, 129, 4096)] == \
        ["32", "32", "64", "64", "128", "128", "256,pair", "256,pair"]


def test_job_throughput_scales_with_ranks():
    assert bench.job_gbs(1, 10 ** 9, 1, 1000.0) == 1.0
    assert bench.job_gbs(8, 10 ** 9, 1, 1000.0) == 8.0


# ---------------------------------------------------------------- the bench's parity check before timing
import numpy as np  # noqa: E402
import pytest  # noqa: E402
import torch  # noqa: E402

import gwb_synth as synth  # noqa: E402
import oracle  # noqa: E402


def _affine_item(N=64, K=256, M=5, bits=4, gs=64):
    w = synth.weights(N, K, seed=3)
    wq, sc, bi, _ = oracle.qpack_affine(w.numpy(), bits, gs)
    x = synth.activations(M, K, seed=4)
    y = oracle.qmm_affine(synth.bits16(x), wq, sc, bi, N, K, bits, gs)
    wt = (torch.from_numpy(wq.view(np.int32)), synth.from_bits16(sc, torch.bfloat16),
          synth.from_bits16(bi, torch.bfloat16))
    return ("affine", dict(x=x, w=wt, y=torch.from_numpy(y).to(torch.bfloat16), N=N, K=K, M=M, bits=bits, gs=gs))


def _int8_item(kind, N=48, K=256, M=4):
    w = synth.weights(N, K, seed=5)
    x = synth.activations(M, K, seed=6)
    qx, sx = oracle.quant_per_token_i8(synth.bits16(x))
    if kind == "w4a8":
        wq, sw, _ = oracle.qpack_sym_i4(w.numpy())
        acc, y, _ = oracle.gemm_i8i4(qx, sx, wq, sw, N, K)
        wt = (torch.from_numpy(wq.view(np.int32)), torch.from_numpy(sw))
    else:
        wq, sw = oracle.qpack_sym_i8(w.numpy())
        acc, y, _ = oracle.gemm_i8i8(qx, sx, wq, sw, N, K)
        wt = (torch.from_numpy(wq), torch.from_numpy(sw))
    return (kind, dict(x=x, qx=torch.from_numpy(qx), sx=torch.from_numpy(sx), w=wt,
                       y=torch.from_numpy(y).to(torch.bfloat16), acc=torch.from_numpy(acc.astype(np.int32)), N=N, K=K))


def _gptq_items(K=256, N=64, gs=64, M=3):
    qw, sc, qz, gi = synth.gptq_quartet(K, N, gs, seed=7, permuted=True)
    h = (qw.numpy(), synth.bits16(sc), qz.numpy(), gi.numpy())
    x = synth.activations(M, K, seed=8, dtype=torch.float16)
    y = oracle.gptq_qmm(synth.bits16(x), *h, K, N, gs)
    wd = oracle.gptq_dequant_f16(*h, K, N, gs)
    return [("gptq", dict(x=x, h=(qw, sc, qz, gi), y=torch.from_numpy(y).to(torch.float16), K=K, N=N, gs=gs, M=M)),
            ("gptq_dequant", dict(h=(qw, sc, qz, gi), y=synth.from_bits16(wd, torch.float16), K=K, N=N, gs=gs))]


def test_bench_check_accepts_oracle_outputs_and_rejects_a_planted_error():
    items = [_affine_item(), _int8_item("w4a8"), _int8_item("w8a8")] + _gptq_items()
    for it in items:
        assert bench.check_item(it)
    # a wrong output row fails the float check; a wrong accumulator fails the integer check
    kind, d = _affine_item()
    d["y"][2] = d["y"][2] * 1.5
    with pytest.raises(AssertionError):
        bench.check_item((kind, d))
    kind, d = _int8_item("w8a8")
    d["acc"][0, 0] += 1
    with pytest.raises(AssertionError):
        bench.check_item((kind, d))
    kind, d = _gptq_items()[1]
    d["y"] = d["y"].clone()
    d["y"][0, 0] = -d["y"][0, 0] if d["y"][0, 0] != 0 else 1.0
    with pytest.raises(AssertionError):
        bench.check_item((kind, d))


def test_bench_copies_exceed_twice_the_l2():
    for nbytes in (2_400_000, 9_400_000, 33_000_000, 148_000_000):
        n = bench.copies_for(nbytes)
        assert n >= 2 and (n * nbytes > 2 * bench.L2_BYTES or n * nbytes > (1 << 30) - nbytes)


def test_bench_aggregate_units():
    w1 = bench.Work("a", None, 2, nbytes=3e6, flops=4e9, kernel="k")
    w2 = bench.Work("b", None, 2, nbytes=1e6, flops=2e9, kernel="k")
    hbm = bench.aggregate("x", [(w1, 2.0), (w2, 2.0)], 6540.8, "measured", "GB/s", "hbm")
    assert hbm["value"] == 1000.0                      # 4e6 bytes in 4 us
    assert hbm["roofline"]["frac"] == round(1000.0 / 6540.8, 4)
    ten = bench.aggregate("x", [(w1, 2.0), (w2, 2.0)], 1656.2, "measured", "TFLOP/s", "tensor")
    assert ten["value"] == 1500.0                      # 6e9 flop in 4 us
    assert [s["TFLOP/s"] for s in ten["shapes"]] == [2000.0, 1000.0]

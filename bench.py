"""Benchmark of the fused dequant + matmul hot path on B200.

One step = one pass of the decode GEMV sweep at M = 1 (bf16 activations,
MLX affine weights, group size 64): N x K in {2048x2048, 512x2048, 8192x2048,
2048x8192, 128256x2048} at 4 bits, plus 8192x2048 at 2 and 8 bits.  The
headline value is whole-job HBM throughput (algorithmic bytes: packed codes +
bf16 scales and biases + activations + outputs, per call) in GB/s.  The same
JSON line also carries the prefill GEMM at M = 2048 (4-bit, group size 64,
shapes 4096x4096, 1024x4096, 14336x4096, 4096x14336) in TFLOP/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {gwb,reference}]

N > 1 is launched by torchrun: every rank runs an independent replica of the
step on its own GPU (the path has no exchange step); the time is the max over
ranks and the value counts the bytes of all ranks ("scaling": "weak").
--impl reference times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import threading
import time

import numpy as np
import torch

import gwb_synth as synth

DECODE = [  # (N, K, bits)
    (2048, 2048, 4), (512, 2048, 4), (8192, 2048, 4), (2048, 8192, 4), (128256, 2048, 4),
    (8192, 2048, 2), (8192, 2048, 8),
]
PREFILL = [(4096, 4096), (1024, 4096), (14336, 4096), (4096, 14336)]
GS = 64
M_PREFILL = 2048
METRIC = "qmm GB/s (M=1) and TFLOP/s (M=2048), % of roofline, 4-bit gs=64, 1 B200"
WORKLOAD = ("decode GEMV sweep, M=1, bf16 x, MLX affine gs=64: 4-bit NxK 2048x2048, 512x2048, 8192x2048, "
            "2048x8192, 128256x2048; 2-bit and 8-bit 8192x2048")
ROOT = os.path.dirname(os.path.abspath(__file__))


def gemv_bytes(N, K, bits, M=1, gs=GS):
    """Algorithmic bytes of one qmm call: packed codes, bf16 scales + biases, x and y."""
    return N * K * bits // 8 + 2 * 2 * N * (K // gs) + 2 * M * K + 2 * M * N


STEP_BYTES = sum(gemv_bytes(N, K, b) for N, K, b in DECODE)
LMHEAD = (128256, 2048, 4)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def traffic_for(kernel_key):
    """Per-launch DRAM bytes (read + write) of a kernel from the committed ncu summary, or None."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.txt")) as f:
            for line in f:
                parts = line.split()
                if parts and not parts[0].startswith("#") and parts[0] == kernel_key:
                    return int(parts[1])
    except Exception:
        pass
    return None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running (reads only)."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index):
        self.index, self.samples, self.reasons, self.max_mhz = index, [], set(), None
        self._stop = threading.Event()
        self._t = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        except Exception:
            self._t = None
        return self

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                r = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ distributed plumbing
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world):
    """The largest of the ranks' values (a device time: the job ends with its slowest rank)."""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cpu" if dist.get_backend() == "gloo" else "cuda"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(world, bytes_per_step, steps, ms_max):
    """Whole-job throughput of `world` replicas that each moved bytes_per_step per step, timed as the
    slowest rank: every rank processes its own copy of the workload (weak scaling)."""
    return world * bytes_per_step * steps / (ms_max * 1e-3) / 1e9


# ------------------------------------------------------------------ GPU arm
def build_decode(gwb, dev, n_sets=2):
    """Quantizes every decode weight on the device (seeded N(0, 0.02)); n_sets copies rotate."""
    sets = []
    for s in range(n_sets):
        layers = []
        for i, (N, K, bits) in enumerate(DECODE):
            g = torch.Generator(device=dev)
            g.manual_seed(1000 * s + i)
            w = torch.randn((N, K), generator=g, device=dev, dtype=torch.float32) * 0.02
            wq, sc, bi = gwb.qpack_affine(w, bits, GS)
            del w
            x = synth.activations(1, K, seed=1).to(dev)
            y = torch.empty((1, N), dtype=torch.bfloat16, device=dev)
            layers.append((wq, sc, bi, x, y, bits))
        sets.append(layers)
    torch.cuda.synchronize()
    return sets


def run_gpu(args, world, rank, local):
    import group_wise_bit_b200 as gwb

    dev = torch.device("cuda", local)
    hbm_peak, bf16_peak, peak_kind = peaks()
    sets = build_decode(gwb, dev)
    lm_idx = DECODE.index(LMHEAD)

    # One CUDA graph per step: [event] lm_head GEMV [event] the six other GEMVs, with
    # programmatic launch chaining the GEMVs.  Each step has its own graph and its
    # own event-record nodes, so the lm_head launch of every timed step is timed on
    # the device; consecutive steps alternate between the two weight sets.
    n_graphs = max(args.steps, 1)
    stream = torch.cuda.Stream(device=dev)
    graphs, lm_events = [], []
    with torch.cuda.stream(stream):
        for layers in sets:
            for (wq, sc, bi, x, y, bits) in layers:           # warm the launch path before capture
                gwb.qmm_affine(x, wq, sc, bi, bits, GS, y=y)
        torch.cuda.synchronize()
        for gi in range(n_graphs):
            layers = sets[gi % len(sets)]
            ev = (torch.cuda.Event(enable_timing=True, external=True),
                  torch.cuda.Event(enable_timing=True, external=True))
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                wq, sc, bi, x, y, bits = layers[lm_idx]
                ev[0].record(stream)
                gwb.qmm_affine(x, wq, sc, bi, bits, GS, y=y)
                ev[1].record(stream)
                for i, (wq, sc, bi, x, y, bits) in enumerate(layers):
                    if i != lm_idx:
                        gwb.qmm_affine(x, wq, sc, bi, bits, GS, y=y)
            graphs.append(g)
            lm_events.append(ev)
    torch.cuda.synchronize()

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            graphs[i % n_graphs].replay()
    torch.cuda.synchronize()

    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            t0.record(stream)
            for i in range(args.steps):
                graphs[i].replay()
            t1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms = t0.elapsed_time(t1)
    ms_max = max_over_ranks(ms, world)
    ms_step = ms_max / args.steps
    value = job_gbs(world, STEP_BYTES, args.steps, ms_max)
    lm_ms = float(np.mean([a.elapsed_time(b) for a, b in lm_events[:args.steps]]))
    lm_bytes = gemv_bytes(*LMHEAD)
    achieved = lm_bytes / (lm_ms * 1e-3) / 1e9
    del graphs

    # End to end through the public API: pinned host x -> device, qmm, y -> pinned host, every layer.
    host_x = [l[3].cpu().pin_memory() for l in sets[0]]
    host_y = [torch.empty(l[4].shape, dtype=torch.bfloat16).pin_memory() for l in sets[0]]
    h2d = sum(t.numel() * 2 for t in host_x)
    d2h = sum(t.numel() * 2 for t in host_y)

    def e2e_step(i):
        layers = sets[i % len(sets)]
        for j, (wq, sc, bi, x, y, bits) in enumerate(layers):
            x.copy_(host_x[j], non_blocking=True)
            gwb.qmm_affine(x, wq, sc, bi, bits, GS, y=y)
            host_y[j].copy_(y, non_blocking=True)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(args.steps):
            e2e_step(i)
        e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_value = job_gbs(world, STEP_BYTES, args.steps, e_ms)

    prefill = run_prefill(gwb, dev, stream, bf16_peak, peak_kind) if not args.no_prefill else None
    int8 = {}
    int8["decode_mlp_fused"] = run_mlp_fused(gwb, dev, stream, hbm_peak)
    int8["w4a8_decode_fused"] = run_w4a8_decode(gwb, dev, stream, hbm_peak)
    if not args.no_prefill:
        i8peak = int8_peak_tops(dev, stream)
        int8["w4a8_m4096"] = run_int8(gwb, dev, stream, "w4a8", 14336, 4096, 4096, i8peak, hbm_peak)
        int8["w8a8_m4096"] = run_int8(gwb, dev, stream, "w8a8", 14336, 4096, 4096, i8peak, hbm_peak)
        int8["w8a8_m1"] = run_int8(gwb, dev, stream, "w8a8", 14336, 4096, 1, i8peak, hbm_peak)

    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": 1, "group_size": GS, "bytes_per_step": STEP_BYTES,
                   "l2": "inputs larger than L2: 192 MB of weights per step, two weight sets rotate (384 MB)",
                   "graphs": "each step replays its own CUDA graph of the seven GEMVs (lm_head first, bracketed by event nodes)",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"kernel": "k_gemv_pipe<4,64,1> (lm_head 128256x2048)", "bound": "hbm",
                     "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                     "frac": round(achieved / hbm_peak, 4), "peak_source": peak_kind,
                     "bytes_per_launch": lm_bytes, "avg_launch_us": round(lm_ms * 1e3, 2),
                     "traffic": traffic_for("k_gemv_pipe_lmhead")},
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "note": "weights resident in HBM; per layer: H2D of x, qmm_affine call, D2H of y"},
        "gpu_launches": len(DECODE) * args.steps,
        "clocks": clk.summary(),
    }
    if prefill:
        out["prefill_m2048"] = prefill
    out.update(int8)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(budget_s=args.cpu_seconds)
    if rank == 0:
        print(json.dumps(out), flush=True)


def int8_peak_tops(dev, stream, reps=5):
    """Dense int8 tensor throughput of this GPU, measured here: torch._int_mm on
    8192^3 (2 * 8192^3 ops per call), best of `reps` launches."""
    a = torch.randint(-64, 64, (8192, 8192), dtype=torch.int8, device=dev)
    b = torch.randint(-64, 64, (8192, 8192), dtype=torch.int8, device=dev)
    best = float("inf")
    with torch.cuda.stream(stream):
        torch._int_mm(a, b)
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            torch._int_mm(a, b)
            e1.record(stream)
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1))
    return 2.0 * 8192 ** 3 / (best * 1e-3) / 1e12


def int8_operands(gwb, dev, fmt, N, K, M, seed=91):
    """Quantized weights (fmt 'w4a8': int4 codes, 'w8a8': int8) and per-token int8 activations."""
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    w = torch.randn((N, K), generator=g, device=dev, dtype=torch.float32) * 0.02
    wq, sw = gwb.qpack_sym_i4(w) if fmt == "w4a8" else gwb.qpack_sym_i8(w)
    del w
    x = synth.activations(M, K, seed=1).to(dev)
    qx, sx = gwb.quant_per_token_i8(x)
    return wq, sw, qx, sx


def int8_gemm(gwb, fmt):
    return gwb.gemm_i8i4 if fmt == "w4a8" else gwb.gemm_i8i8


def run_int8(gwb, dev, stream, fmt, N, K, M, int8_peak, hbm_peak, reps=5):
    """int8-activation GEMM (fmt 'w4a8' or 'w8a8', int32 accumulation, bf16 out) on an N x K
    weight at M tokens, each launch timed alone with an L2 flush before it.  M = 1 is
    HBM-bound (bytes = weights + scales + activations + output); larger M is tensor-bound
    (ops = 2 M N K)."""
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.int32, device=dev)
    wq, sw, qx, sx = int8_operands(gwb, dev, fmt, N, K, M)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    gemm = int8_gemm(gwb, fmt)
    ts = []
    with torch.cuda.stream(stream):
        for r in range(reps + 2):
            flush.fill_(r)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            gemm(qx, sx, wq, sw, y=y)
            b.record(stream)
            b.synchronize()
            if r >= 2:
                ts.append(a.elapsed_time(b))
    ms = statistics.median(ts)
    if fmt == "w4a8":
        kern = "k_tc2<I8,4,256,pair,A in TMEM> (kind::i8)"
    elif M <= 8 and K % 512 == 0:
        kern = "k_gemv_pipe<8,64,%d,i8w8> (int8 x int8 weight streaming, exact int32 sums)" % (M,)
    else:
        kern = "k_tc2<W8,8,%s> (kind::i8, both operands by TMA)" % ("256,pair" if M > 128 else "128" if M > 32 else "32")
    out = {"N": N, "K": K, "M": M, "us": round(ms * 1e3, 1)}
    if M <= 8:
        wbytes = N * K // (2 if fmt == "w4a8" else 1)
        nbytes = wbytes + N * 4 + M * K + M * 4 + M * N * 2
        gbs = nbytes / (ms * 1e-3) / 1e9
        out.update({"value": round(gbs, 1), "unit": "GB/s",
                    "roofline": {"kernel": kern, "bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak,
                                 "unit": "GB/s", "frac": round(gbs / hbm_peak, 4), "bytes_per_launch": nbytes,
                                 "peak_source": "measured (MEASURED_PEAKS.json hbm_gbs)"}})
    else:
        tops = 2.0 * M * N * K / (ms * 1e-3) / 1e12
        out.update({"value": round(tops, 1), "unit": "TOP/s",
                    "roofline": {"kernel": kern, "bound": "tensor", "achieved": round(tops, 1),
                                 "peak": round(int8_peak, 1), "unit": "TOP/s", "frac": round(tops / int8_peak, 4),
                                 "peak_source": "measured in this run: torch._int_mm 8192^3 int8, best of 5",
                                 "traffic": traffic_for(f"k_tc2_{fmt}_m{M}")}})
    return out


def run_prefill(gwb, dev, stream, bf16_peak, peak_kind, reps=5):
    """M = 2048 prefill GEMMs (4-bit, gs 64), each launch timed alone with an L2 flush before it."""
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.int32, device=dev)
    total_flop, total_ms, per = 0.0, 0.0, []
    for i, (N, K) in enumerate(PREFILL):
        g = torch.Generator(device=dev)
        g.manual_seed(77 + i)
        w = torch.randn((N, K), generator=g, device=dev, dtype=torch.float32) * 0.02
        wq, sc, bi = gwb.qpack_affine(w, 4, GS)
        del w
        x = synth.activations(M_PREFILL, K, seed=1, outlier_frac=0.01).to(dev)
        y = torch.empty((M_PREFILL, N), dtype=torch.bfloat16, device=dev)
        ts = []
        with torch.cuda.stream(stream):
            for r in range(reps + 2):
                flush.fill_(r)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                gwb.qmm_affine(x, wq, sc, bi, 4, GS, y=y)
                b.record(stream)
                b.synchronize()
                if r >= 2:
                    ts.append(a.elapsed_time(b))
        ms = statistics.median(ts)
        flop = 2.0 * M_PREFILL * N * K
        total_flop += flop
        total_ms += ms
        per.append({"N": N, "K": K, "us": round(ms * 1e3, 1), "tflops": round(flop / (ms * 1e-3) / 1e12, 1)})
    tf = total_flop / (total_ms * 1e-3) / 1e12
    return {"value": round(tf, 1), "unit": "TFLOP/s", "M": M_PREFILL, "bits": 4, "group_size": GS,
            "l2": "256 MB buffer written before every timed launch",
            "roofline": {"kernel": "k_tc2<Affine,4,256,pair,A in TMEM> (persistent, stream-K)", "bound": "tensor",
                         "achieved": round(tf, 1),
                         "peak": bf16_peak, "unit": "TFLOP/s", "frac": round(tf / bf16_peak, 4),
                         "peak_source": peak_kind, "traffic": traffic_for("k_tc2_affine4_m2048")},
            "shapes": per}


def run_w4a8_decode(gwb, dev, stream, hbm_peak, N=14336, K=4096, M=1, reps=20):
    """W4A8 at decode: the fused product (activations quantized inside the kernel) against the
    two-launch path (quant_per_token_i8, then gemm_i8i4), each a CUDA graph of `reps` launches
    alternating two weight sets (> L2)."""
    sets = [int8_operands(gwb, dev, "w4a8", N, K, M, seed=s_) for s_ in range(2)]
    x = synth.activations(M, K, seed=1).to(dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    qx = torch.empty((M, K), dtype=torch.int8, device=dev)
    sx = torch.empty((M,), dtype=torch.float32, device=dev)

    def fused(i):
        wq, sw, _, _ = sets[i % 2]
        gwb.gemv_w4a8(x, wq, sw, y=y)

    def two(i):
        wq, sw, _, _ = sets[i % 2]
        gwb.quant_per_token_i8(x, qx=qx, sx=sx)
        gwb.gemm_i8i4(qx, sx, wq, sw, y=y)

    out = {}
    for name, fn in (("fused", fused), ("two_launch", two)):
        with torch.cuda.stream(stream):
            for i in range(2):
                fn(i)
            stream.synchronize()
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                for i in range(reps):
                    fn(i)
            gr.replay()
            stream.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            gr.replay()
            b.record(stream)
            b.synchronize()
        out[name] = a.elapsed_time(b) * 1e3 / reps
    nbytes = N * K // 2 + N * 4 + 2 * M * K + 2 * M * N
    gbs = nbytes / out["fused"] / 1e3
    return {"value": round(gbs, 1), "unit": "GB/s", "N": N, "K": K, "M": M,
            "us_fused": round(out["fused"], 2), "us_two_launch": round(out["two_launch"], 2),
            "roofline": {"kernel": "k_gemv_pipe<4,64,1,w4a8> (per-token int8 quantization inside)", "bound": "hbm",
                         "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s", "frac": round(gbs / hbm_peak, 4),
                         "bytes_per_launch": nbytes, "peak_source": "measured (MEASURED_PEAKS.json hbm_gbs)"}}


def run_mlp_fused(gwb, dev, stream, hbm_peak, bits=4, M=1, reps=20):
    """Decode MLP of a Llama-3-8B layer (hidden 4096, intermediate 14336, MLX affine gs 64) through
    the fused products: gemv_gate_up, then gemv_silu_gate_resid.  One CUDA graph of `reps` MLPs
    alternating two weight sets (> L2), timed by events around its replay."""
    H, I = 4096, 14336
    sets = []
    for s_ in range(2):
        ws = []
        for j, (n, k) in enumerate(((I, H), (I, H), (H, I))):
            g = torch.Generator(device=dev)
            g.manual_seed(500 + 10 * s_ + j)
            w = torch.randn((n, k), generator=g, device=dev, dtype=torch.float32) * 0.02
            ws.append(gwb.qpack_affine(w, bits, GS))
            del w
        sets.append(ws)
    x = synth.activations(M, H, seed=1).to(dev)
    gate = torch.empty((M, I), dtype=torch.bfloat16, device=dev)
    up = torch.empty((M, I), dtype=torch.bfloat16, device=dev)
    y = torch.empty((M, H), dtype=torch.bfloat16, device=dev)

    def mlp(i):
        wg, wu, wd = sets[i % 2]
        gwb.gemv_gate_up(x, wg, wu, bits, GS, y_gate=gate, y_up=up)
        gwb.gemv_silu_gate(gate, up, *wd, bits, GS, x_resid=x, y=y)

    with torch.cuda.stream(stream):
        for i in range(2):
            mlp(i)
        stream.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            for i in range(reps):
                mlp(i)
        gr.replay()
        stream.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        gr.replay()
        b.record(stream)
        b.synchronize()
    us = a.elapsed_time(b) * 1e3 / reps
    nbytes = (2 * gemv_bytes(I, H, bits, M=M) - 2 * M * H) + (gemv_bytes(H, I, bits, M=M) + 2 * M * I + 2 * M * H)
    gbs = nbytes / us / 1e3
    return {"value": round(gbs, 1), "unit": "GB/s", "M": M, "bits": bits, "group_size": GS,
            "us_per_mlp": round(us, 2), "bytes_per_mlp": nbytes, "launches_per_mlp": 2,
            "roofline": {"kernel": "k_gemv_pipe<dual> + k_gemv_pipe<silu> (Llama-3-8B MLP, hidden 4096)",
                         "bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                         "frac": round(gbs / hbm_peak, 4), "peak_source": "measured (MEASURED_PEAKS.json hbm_gbs)"}}


# ------------------------------------------------------------------ CPU oracle (baseline / reference arm)
def oracle_sample(frac, seed=0):
    """A row sample of every decode layer, quantized by the oracle (untimed preparation)."""
    import oracle
    layers = []
    for i, (N, K, bits) in enumerate(DECODE):
        n = max(8, int(N * frac))
        w = synth.weights(n, K, seed=seed + i)
        wq, sc, bi, _ = oracle.qpack_affine(w.numpy(), bits, GS)
        x = synth.bits16(synth.activations(1, K, seed=1))
        layers.append((x, wq, sc, bi, n, K, bits))
    return layers


def oracle_pass(layers):
    import oracle
    nbytes = 0
    for x, wq, sc, bi, n, K, bits in layers:
        oracle.qmm_affine(x, wq, sc, bi, n, K, bits, GS)
        nbytes += gemv_bytes(n, K, bits)
    return nbytes


def cpu_baseline(budget_s=12.0, frac=0.25):
    layers = oracle_sample(frac)
    t = time.perf_counter()
    nbytes, passes = 0, 0
    while passes < 1 or time.perf_counter() - t < budget_s:
        nbytes += oracle_pass(layers)
        passes += 1
    dt = time.perf_counter() - t
    return {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{passes} pass(es) over the first {frac:.0%} of the output rows of every decode layer "
                      f"(M=1, gs=64), single-threaded C, fp64, {dt:.1f} s"}


def run_reference(args, world, rank):
    if rank != 0:
        return
    frac = args.ref_frac
    layers = oracle_sample(frac)
    for _ in range(args.warmup):
        oracle_pass(layers)
    t = time.perf_counter()
    nbytes = 0
    for _ in range(args.steps):
        nbytes += oracle_pass(layers)
    dt = time.perf_counter() - t
    value = nbytes / dt / 1e9
    out = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": 1, "group_size": GS,
                   "sample": f"first {frac:.1%} of the output rows of every layer per step"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"{args.steps} steps, each over the first {frac:.1%} of the output rows of "
                                   f"every decode layer, single-threaded C, fp64"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def run_layer(args):
    """One layer only (for profiling): qmm_affine (or, with --fmt, the int8-activation GEMM) on an
    N x K weight at M tokens, replayed in a CUDA graph of 20 launches that alternate between two
    weight sets (> L2)."""
    import group_wise_bit_b200 as gwb
    N, K, bits, M = (list(map(int, args.layer.split(","))) + [1])[:4]
    dev = torch.device("cuda", 0)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    if args.fmt == "affine":
        sets = []
        for s in range(2):
            g = torch.Generator(device=dev)
            g.manual_seed(s)
            w = torch.randn((N, K), generator=g, device=dev, dtype=torch.float32) * 0.02
            sets.append(gwb.qpack_affine(w, bits, GS))
            del w
        x = synth.activations(M, K, seed=1).to(dev)

        def launch(i):
            wq, sc, bi = sets[i % 2]
            gwb.qmm_affine(x, wq, sc, bi, bits, GS, y=y)
    elif args.fmt in ("gate_up", "silu_resid"):
        sets = []
        for s in range(2):
            ws = []
            for j in range(2 if args.fmt == "gate_up" else 1):
                g = torch.Generator(device=dev)
                g.manual_seed(10 * s + j)
                w = torch.randn((N, K), generator=g, device=dev, dtype=torch.float32) * 0.02
                ws.append(gwb.qpack_affine(w, bits, GS))
                del w
            sets.append(ws)
        x = synth.activations(M, K, seed=1).to(dev)
        x2 = synth.activations(M, K, seed=2).to(dev)
        res = synth.activations(M, N, seed=3).to(dev)
        y2 = torch.empty((M, N), dtype=torch.bfloat16, device=dev)

        def launch(i):
            ws = sets[i % 2]
            if args.fmt == "gate_up":
                gwb.gemv_gate_up(x, ws[0], ws[1], bits, GS, y_gate=y, y_up=y2)
            else:
                gwb.gemv_silu_gate(x, x2, *ws[0], bits, GS, x_resid=res, y=y)
    else:
        sets = [int8_operands(gwb, dev, args.fmt, N, K, M, seed=s) for s in range(2)]
        gemm = int8_gemm(gwb, args.fmt)
        bits = 4 if args.fmt == "w4a8" else 8

        def launch(i):
            wq, sw, qx, sx = sets[i % 2]
            gemm(qx, sx, wq, sw, y=y)
    st = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(st):
        for i in range(2):
            launch(i)
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=st):
            for i in range(20):
                launch(i)
        for _ in range(args.warmup):
            gr.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        for _ in range(args.steps):
            gr.replay()
        b.record(st)
    torch.cuda.synchronize()
    us = a.elapsed_time(b) * 1e3 / (20 * args.steps)
    if args.fmt == "affine":
        nbytes = gemv_bytes(N, K, bits, M=M) if M <= 8 else None
    elif args.fmt == "gate_up":
        nbytes = 2 * gemv_bytes(N, K, bits, M=M) - 2 * M * K      # x is read once
    elif args.fmt == "silu_resid":
        nbytes = gemv_bytes(N, K, bits, M=M) + 2 * M * K + 2 * M * N   # up and the residual
    else:
        nbytes = (N * K * bits // 8 + N * 4 + M * K + M * 4 + M * N * 2) if M <= 8 else None
    out = {"layer": {"fmt": args.fmt, "N": N, "K": K, "bits": bits, "group_size": GS, "M": M},
           "us_per_launch": round(us, 2)}
    if nbytes:
        out["GB/s"] = round(nbytes / us / 1e3, 1)
    else:
        out["TFLOP/s" if args.fmt == "affine" else "TOP/s"] = round(2.0 * M * N * K / us / 1e6, 1)
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["gwb", "reference"], default="gwb")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--fmt", choices=["affine", "w4a8", "w8a8", "gate_up", "silu_resid"], default="affine",
                    help="--layer: weight format (affine: MLX group-wise, bits from --layer)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-frac", type=float, default=1 / 16)
    ap.add_argument("--layer", default=None,
                    help="N,K,bits[,M]: time one layer (qmm_affine at group size 64, or --fmt) instead of the sweep")
    args = ap.parse_args()
    if args.layer:
        run_layer(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        run_gpu(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

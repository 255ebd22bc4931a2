"""Benchmark of the fused dequant + matmul hot path on B200.

One step = one pass of the decode GEMV sweep at M = 1 (bf16 activations,
MLX affine weights, group size 64): N x K in {2048x2048, 512x2048, 8192x2048,
2048x8192, 128256x2048} at 4 bits, plus 8192x2048 at 2 and 8 bits.  The
headline value is whole-job HBM throughput (algorithmic bytes: packed codes +
bf16 scales and biases + activations + outputs, per call) in GB/s.  The same
JSON line carries the rest of the workloads, each with its roofline:

  * prefill GEMM, 4-bit gs 64, shapes 4096x4096, 1024x4096, 14336x4096,
    4096x14336 at M = 16 (GB/s), 128 (GB/s and TFLOP/s), 512 and 2048
    (TFLOP/s); at M = 2048 also 8-bit gs 64 and 4-bit gs 32 / gs 128;
  * GPTQ int4 (K = 4096, N = 11008, gs 128, with and without a permuted
    g_idx): dequant (GB/s), qmm at M = 1 and 32 (GB/s) and 1024 (TFLOP/s);
  * W4A8 and W8A8 on 4096x4096, 14336x4096, 4096x14336 at M = 8, 64 (GB/s)
    and 512, 4096 (TOP/s); W8A8 at M = 1; the fused W4A8 decode product;
  * the fused decode MLP of a Llama-3-8B layer (gate/up pair, silu product).

Every workload is timed as a CUDA graph of back-to-back launches that rotate
through enough copies of its weights that they exceed twice the L2 cache;
the time per launch is the graph's device time (CUDA events) divided by the
launches.  Before anything is timed, rank 0 at N = 1 runs the CPU baseline
leg: the CPU oracle on sampled outputs of every workload (the bench's own
device-drawn weights, copied to the host), which must match the GPU outputs
(bit-exact integers, the float tolerance otherwise), else the run fails.

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
import sys
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
PREFILL_M = (16, 128, 512, 2048)
INT8_SHAPES = [(4096, 4096), (14336, 4096), (4096, 14336)]
INT8_M = (8, 64, 512, 4096)
GPTQ_K, GPTQ_N, GPTQ_GS = 4096, 11008, 128
GS = 64
M_PREFILL = 2048
L2_BYTES = 126 * 2 ** 20
METRIC = "qmm GB/s (M=1) and TFLOP/s (M=2048), % of roofline, 4-bit gs=64, 1 B200"
WORKLOAD = ("decode GEMV sweep, M=1, bf16 x, MLX affine gs=64: 4-bit NxK 2048x2048, 512x2048, 8192x2048, "
            "2048x8192, 128256x2048; 2-bit and 8-bit 8192x2048")
ROOT = os.path.dirname(os.path.abspath(__file__))


def gemv_bytes(N, K, bits, M=1, gs=GS):
    """Algorithmic bytes of one qmm call: packed codes, bf16 scales + biases, x and y."""
    return N * K * bits // 8 + 2 * 2 * N * (K // gs) + 2 * M * K + 2 * M * N


def gptq_bytes(K, N, gs, M, g_idx):
    """One GPTQ qmm call: int4 codes, fp16 scales, packed zeros, g_idx (if given), fp16 x and y."""
    return K * N // 2 + 2 * N * (K // gs) + N * (K // gs) // 2 + (4 * K if g_idx else 0) + 2 * M * K + 2 * M * N


def gptq_dequant_bytes(K, N, gs, g_idx):
    """One GPTQ dequant call: the packed tensors in, the fp16 [N, K] weight out."""
    return gptq_bytes(K, N, gs, 0, g_idx) + 2 * N * K


def int8_bytes(N, K, M, wbits):
    """One int8-activation GEMM call: weight codes, fp32 weight scales, int8 x, fp32 token scales, bf16 y."""
    return N * K * wbits // 8 + 4 * N + M * K + 4 * M + 2 * M * N


STEP_BYTES = sum(gemv_bytes(N, K, b) for N, K, b in DECODE)
LMHEAD = (128256, 2048, 4)


def copies_for(nbytes, cap=1 << 30):
    """Weight copies a timing graph rotates through: their total exceeds twice the L2
    (at least 2 copies, at most `cap` bytes unless 2 copies already pass it)."""
    n = max(2, math.ceil(2 * L2_BYTES / max(nbytes, 1)) + 1)
    while n > 2 and n * nbytes > cap:
        n -= 1
    return n


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def traffic_entry(kernel_key):
    """(per-launch DRAM bytes read + written, source summary) of a kernel from the committed ncu
    summaries, or (None, None)."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.txt")) as f:
            for line in f:
                parts = line.split()
                if parts and not parts[0].startswith("#") and parts[0] == kernel_key:
                    return int(parts[1]), parts[2]
    except Exception:
        pass
    return None, None


def traffic_for(kernel_key):
    """Per-launch DRAM bytes (read + write) of a kernel from the committed ncu summary, or None."""
    return traffic_entry(kernel_key)[0]


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running (reads only)."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index, period_s=0.0002):
        self.index, self.samples, self.reasons, self.max_mhz = index, [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._first = threading.Event()
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
            self._first.wait(1.0)            # the window opens with a sample in hand
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
            self._first.set()
            time.sleep(self.period)

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


def roofline(kernel, bound, achieved, peak, unit, peak_source, traffic=None, **extra):
    out = {"kernel": kernel, "bound": bound, "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": unit,
           "frac": round(achieved / peak, 4), "peak_source": peak_source, "traffic": traffic}
    out.update(extra)
    return out


# ------------------------------------------------------------------ GPU timing helpers
def graph_us(launch, n, stream, replays=3):
    """Device time per launch of a CUDA graph of `n` back-to-back launch(i), i = 0 .. n-1
    (CUDA events around `replays` replays, after one untimed replay)."""
    with torch.cuda.stream(stream):
        for i in range(min(n, 2)):
            launch(i)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                launch(i)
        g.replay()
        stream.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(replays):
            g.replay()
        b.record(stream)
        b.synchronize()
    us = a.elapsed_time(b) * 1e3 / (n * replays)
    del g
    return us


def dev_weight(dev, N, K, seed):
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    return torch.randn((N, K), generator=g, device=dev, dtype=torch.float32) * 0.02


def clone_all(ts, n):
    """n copies of a tuple of tensors (copy 0 is the original)."""
    return [ts] + [tuple(t.clone() for t in ts) for _ in range(n - 1)]


# ------------------------------------------------------------------ workloads
class Work:
    """One timed workload: `launch(i)` runs the product on weight copy i (of n); `nbytes` and
    `flops` are its algorithmic bytes and operations per launch; each of `checks` returns the
    host copy of copy 0's output and inputs for the CPU baseline leg's comparison."""

    def __init__(self, key, launch, n, nbytes, flops, kernel, checks=()):
        self.key, self.launch, self.n, self.nbytes, self.flops = key, launch, n, nbytes, flops
        self.kernel, self.checks = kernel, list(checks)


def build_decode(gwb, dev, n_sets=2):
    """Quantizes every decode weight on the device (seeded N(0, 0.02)); n_sets copies rotate."""
    sets = []
    for s in range(n_sets):
        layers = []
        for i, (N, K, bits) in enumerate(DECODE):
            w = dev_weight(dev, N, K, 1000 * s + i)
            wq, sc, bi = gwb.qpack_affine(w, bits, GS)
            del w
            x = synth.activations(1, K, seed=1).to(dev)
            y = torch.empty((1, N), dtype=torch.bfloat16, device=dev)
            layers.append((wq, sc, bi, x, y, bits))
        sets.append(layers)
    torch.cuda.synchronize()
    return sets


def affine_work(gwb, dev, key, shapes, M, bits, gs, kernel, seed0=77):
    """qmm_affine at M tokens over several N x K shapes (one Work per shape)."""
    works = []
    for j, (N, K) in enumerate(shapes):
        w = dev_weight(dev, N, K, seed0 + j)
        wt = gwb.qpack_affine(w, bits, gs)
        del w
        wbytes = gemv_bytes(N, K, bits, M=0, gs=gs)
        cps = clone_all(wt, copies_for(wbytes))
        x = synth.activations(M, K, seed=1, outlier_frac=0.01)
        xd = x.to(dev)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)

        def launch(i, cps=cps, xd=xd, y=y, bits=bits, gs=gs):
            wq, sc, bi = cps[i % len(cps)]
            gwb.qmm_affine(xd, wq, sc, bi, bits, gs, y=y)

        def check(cps=cps, x=x, y=y, N=N, K=K, M=M, bits=bits, gs=gs):
            return ("affine", dict(x=x, w=tuple(t.cpu() for t in cps[0]), y=y.cpu(), N=N, K=K, M=M, bits=bits,
                                   gs=gs))

        works.append(Work(f"{key} {N}x{K}", launch, len(cps), gemv_bytes(N, K, bits, M=M, gs=gs), 2.0 * M * N * K,
                          kernel, [check]))
    return works


def gptq_work(gwb, dev, M, permuted, dequant=False):
    K, N, gs = GPTQ_K, GPTQ_N, GPTQ_GS
    qw, sc, qz, gi = synth.gptq_quartet(K, N, gs, seed=0, permuted=permuted)
    d = (qw.to(dev), sc.to(dev), qz.to(dev))
    gid = gi.to(dev) if permuted else None
    cps = clone_all(d, copies_for(gptq_bytes(K, N, gs, 0, permuted)))
    if dequant:
        out = torch.empty((N, K), dtype=torch.float16, device=dev)

        def launch(i):
            q, s, z = cps[i % len(cps)]
            gwb.gptq_dequant(q, s, z, gid, gs, out=out)

        def check():
            return ("gptq_dequant", dict(h=(qw, sc, qz, gi if permuted else None), y=out.cpu(), K=K, N=N, gs=gs))

        return Work(f"gptq dequant perm={int(permuted)}", launch, len(cps), gptq_dequant_bytes(K, N, gs, permuted),
                    0.0, "k_gptq_dequant", [check])
    x = synth.activations(M, K, seed=1, dtype=torch.float16)
    xd = x.to(dev)
    y = torch.empty((M, N), dtype=torch.float16, device=dev)

    def launch(i):
        q, s, z = cps[i % len(cps)]
        gwb.gptq_qmm(xd, q, s, z, gid, gs, y=y)

    def check():
        return ("gptq", dict(x=x, h=(qw, sc, qz, gi if permuted else None), y=y.cpu(), K=K, N=N, gs=gs, M=M))

    if M <= 8:
        kern = "k_gemv_gptq_pipe" if N % 32 == 0 and K % 256 == 0 else "k_gemv_gptq"
    else:
        kern = "k_gptq_dequant + k_tc2<F16>" if permuted else "k_tc2<Gptq>"
    return Work(f"gptq M={M} perm={int(permuted)}", launch, len(cps), gptq_bytes(K, N, gs, M, permuted),
                2.0 * M * N * K, kern, [check])


def tc2_tile(M):
    """The persistent GEMM's token tile for M tokens (single CTAs up to 128, CTA pairs above)."""
    return "32" if M <= 32 else "64" if M <= 64 else "128" if M <= 128 else "256,pair"


def int8_work(gwb, dev, fmt, shapes, M):
    works = []
    for j, (N, K) in enumerate(shapes):
        w = dev_weight(dev, N, K, 91 + j)
        wt = gwb.qpack_sym_i4(w) if fmt == "w4a8" else gwb.qpack_sym_i8(w)
        del w
        wbits = 4 if fmt == "w4a8" else 8
        cps = clone_all(wt, copies_for(N * K * wbits // 8))
        x = synth.activations(M, K, seed=1)
        qx, sx = gwb.quant_per_token_i8(x.to(dev))
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        gemm = gwb.gemm_i8i4 if fmt == "w4a8" else gwb.gemm_i8i8

        def launch(i, cps=cps, qx=qx, sx=sx, y=y, gemm=gemm):
            wq, sw = cps[i % len(cps)]
            gemm(qx, sx, wq, sw, y=y)

        def check(cps=cps, qx=qx, sx=sx, x=x, y=y, N=N, K=K, gemm=gemm, fmt=fmt):
            _, acc = gemm(qx, sx, cps[0][0], cps[0][1], want_y=False, want_acc=True)
            return (fmt, dict(x=x, qx=qx.cpu(), sx=sx.cpu(), w=tuple(t.cpu() for t in cps[0]), y=y.cpu(),
                              acc=acc.cpu(), N=N, K=K))

        if fmt == "w4a8":
            kern = f"k_tc2<I8,4,{tc2_tile(M)}>"
        else:
            kern = "k_gemv_pipe<8,64,M,i8w8>" if M <= 8 and K % 512 == 0 else \
                f"k_tc2<W8,8,{'32' if M <= 32 else '128' if M <= 128 else '256,pair'}>"
        works.append(Work(f"{fmt} {N}x{K} M={M}", launch, len(cps), int8_bytes(N, K, M, wbits), 2.0 * M * N * K,
                          kern, [check]))
    return works


def run_works(works, stream):
    """Times each Work's graph; returns [(work, us per launch)]."""
    return [(w, graph_us(w.launch, w.n, stream)) for w in works]


def aggregate(key, timed, peak, peak_source, unit, bound, traffic_key=None, extra=None):
    """Sum of work over sum of time across a workload's shapes, with its roofline."""
    work = (lambda w: w.nbytes) if bound == "hbm" else (lambda w: w.flops)
    scale = 1e3 if bound == "hbm" else 1e6          # bytes/us -> GB/s; ops/us -> T(FL)OP/s
    tot_us = sum(us for _, us in timed)
    val = sum(work(w) for w, _ in timed) / tot_us / scale
    kernels = sorted({w.kernel for w, _ in timed})
    out = {"value": round(val, 1), "unit": unit,
           "shapes": [{"case": w.key, "us": round(us, 2), unit: round(work(w) / us / scale, 1)} for w, us in timed],
           "roofline": roofline(" + ".join(kernels), bound, val, peak, unit, peak_source)}
    if traffic_key:
        # DRAM bytes of one launch of the captured shape (profiles/<case>), not of the aggregate
        tb, case = traffic_entry(traffic_key)
        out["roofline"]["traffic"] = tb
        out["roofline"]["traffic_case"] = case
    if extra:
        out.update(extra)
    return out


# ------------------------------------------------------------------ CPU baseline leg (oracle)
def _rows_of(M):
    """The sampled rows of a bench workload's output: first, middle, last."""
    return np.unique(np.array([0, M // 2, M - 1] if M > 2 else list(range(M)), dtype=np.int64))


def _w16(t):
    """Raw 16-bit patterns (np.uint16) of a bf16 / fp16 torch tensor, or the words of an int32 one."""
    if t.dtype in (torch.bfloat16, torch.float16):
        return synth.bits16(t)
    return t.numpy()


def check_item(item):
    """Compares one workload's GPU output (copied to the host) with the CPU oracle on sampled
    rows; raises AssertionError on a mismatch.  item = (kind, dict of host tensors and sizes)."""
    import oracle
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from tol import check_float

    kind, d = item
    if kind == "affine":
        wq, sc, bi = (_w16(t) for t in d["w"])
        wq = wq.view(np.uint32)
        r = _rows_of(d["M"])
        ref = oracle.qmm_affine(synth.bits16(d["x"]), wq, sc, bi, d["N"], d["K"], d["bits"], d["gs"], rows=r)
        s = oracle.bf16_array_to_f64(sc)
        b = oracle.bf16_array_to_f64(bi)
        wmax = float(np.max(np.maximum(np.abs(b), np.abs(b + ((1 << d["bits"]) - 1) * s))))
        check_float(d["y"].float().numpy()[r], ref, d["K"], wmax, float(d["x"].float().abs().max()),
                    f"affine {d['N']}x{d['K']} b{d['bits']} gs{d['gs']} M={d['M']}")
    elif kind == "gptq":
        qw, sc, qz, gi = d["h"]
        h = (qw.numpy(), synth.bits16(sc), qz.numpy(), None if gi is None else gi.numpy())
        r = _rows_of(d["M"])
        ref = oracle.gptq_qmm(synth.bits16(d["x"]), *h, d["K"], d["N"], d["gs"], rows=r)
        # an upper bound of max|w|: scale * 16 (|code - zero| <= 15 under the "+1" convention)
        wmax = float(sc.float().abs().max()) * 16
        check_float(d["y"].float().numpy()[r], ref, d["K"], wmax, float(d["x"].float().abs().max()),
                    f"gptq M={d['M']}")
    elif kind == "gptq_dequant":
        qw, sc, qz, gi = d["h"]
        ref = oracle.gptq_dequant_f16(qw.numpy(), synth.bits16(sc), qz.numpy(), None if gi is None else gi.numpy(),
                                      d["K"], d["N"], d["gs"])
        if not np.array_equal(synth.bits16(d["y"]), ref):
            raise AssertionError("gptq_dequant: fp16 weights differ")
    elif kind in ("w4a8", "w8a8"):
        qx, sx = d["qx"].numpy(), d["sx"].numpy()
        qx_o, sx_o = oracle.quant_per_token_i8(synth.bits16(d["x"]))
        if not (np.array_equal(qx, qx_o) and np.array_equal(sx, sx_o)):
            raise AssertionError(f"{kind}: per-token int8 activations differ")
        wq, sw = (t.numpy() for t in d["w"])
        r = _rows_of(qx.shape[0])
        if kind == "w4a8":
            acc_o, y_o, ovf = oracle.gemm_i8i4(qx, sx, wq.view(np.uint32), sw, d["N"], d["K"], rows=r)
            wmax = float(np.abs(sw).max() * 7)
        else:
            acc_o, y_o, ovf = oracle.gemm_i8i8(qx, sx, wq, sw, d["N"], d["K"], rows=r)
            wmax = float(np.abs(sw).max() * 127)
        if ovf or not np.array_equal(d["acc"].numpy().astype(np.int64)[r], acc_o):
            raise AssertionError(f"{kind} {d['N']}x{d['K']}: int32 accumulators differ")
        check_float(d["y"].float().numpy()[r], y_o, d["K"], wmax, float(d["x"].float().abs().max()),
                    f"{kind} {d['N']}x{d['K']} M={qx.shape[0]}")
    else:
        raise ValueError(f"unknown check kind {kind}")
    return True


def cpu_leg(checks, sets, budget_s, threads):
    """The CPU oracle on bounded samples: first timed over the decode sweep on the bench's own
    weights (rows 0 .. n of every layer, single thread), then compared with every workload's
    GPU output on sampled rows (bit-exact integers; the float tolerance otherwise, the same as
    the parity tests).  Returns (cpu_baseline dict, parity dict)."""
    import concurrent.futures as cf

    import oracle
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from tol import check_float

    def bf16_max_w(sc, bi, bits):
        s = oracle.bf16_array_to_f64(sc)
        b = oracle.bf16_array_to_f64(bi)
        return float(np.max(np.maximum(np.abs(b), np.abs(b + ((1 << bits) - 1) * s))))

    # ---- timed: the decode sweep on a row sample of weight set 0
    frac = 0.25
    layers = []
    for (wq, sc, bi, x, y, bits), (N, K, _) in zip(sets[0], DECODE):
        n = max(8, int(N * frac))
        layers.append((synth.bits16(x.cpu()), wq[:n].cpu().numpy().view(np.uint32), synth.bits16(sc[:n].cpu()),
                       synth.bits16(bi[:n].cpu()), n, K, bits, y.cpu()))
    t0 = time.perf_counter()
    nbytes, passes, refs = 0, 0, None
    while passes < 1 or time.perf_counter() - t0 < budget_s:
        refs = []
        for xh, wq, sc, bi, n, K, bits, _ in layers:
            refs.append(oracle.qmm_affine(xh, wq, sc, bi, n, K, bits, GS))
            nbytes += gemv_bytes(n, K, bits)
        passes += 1
    dt = time.perf_counter() - t0
    cpu = {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
           "sample": f"{passes} pass(es) over the first {frac:.0%} of the output rows of every decode layer "
                     f"(M=1, gs=64, the bench's own weights), single-threaded C, fp64, {dt:.1f} s"}

    failures, checked = [], 0
    for (xh, wq, sc, bi, n, K, bits, yg), ref, (N, _, _) in zip(layers, refs, DECODE):
        try:
            check_float(yg.float().numpy()[:, :n], ref, K, bf16_max_w(sc, bi, bits),
                        float(np.abs(oracle.bf16_array_to_f64(xh)).max()), f"decode {N}x{K} b{bits}")
            checked += 1
        except AssertionError as e:
            failures.append(str(e))

    # ---- every other workload, on sampled rows (threads: the oracle's C calls release the GIL)
    with cf.ThreadPoolExecutor(max(1, threads)) as ex:
        futs = [ex.submit(check_item, c) for c in checks]
        for f in futs:
            try:
                f.result()
                checked += 1
            except Exception as e:   # a mismatch, or a check that could not run: both fail the line
                failures.append(f"{type(e).__name__}: {e}")
    parity = {"checked": checked, "failed": len(failures), "ok": not failures,
              "how": "CPU oracle on sampled rows of every workload before timing (bit-exact integers, "
                     "max-abs 2e-2*sqrt(K)*max|w|*max|x| and rel. Frobenius 5e-3 for floats)"}
    if failures:
        parity["failures"] = failures[:10]
    return cpu, parity


# ------------------------------------------------------------------ GPU arm
def run_gpu(args, world, rank, local):
    import group_wise_bit_b200 as gwb

    dev = torch.device("cuda", local)
    hbm_peak, bf16_peak, peak_kind = peaks()
    hbm_src = f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback"
    bf16_src = f"{peak_kind} (MEASURED_PEAKS.json bf16_tflops, burst)" if peak_kind == "measured" else "fallback"
    stream = torch.cuda.Stream(device=dev)
    sets = build_decode(gwb, dev)
    lm_idx = DECODE.index(LMHEAD)
    full = not args.no_prefill

    # ---- every other workload: set up, run once (the CPU leg compares these outputs)
    groups = {}
    if full:
        pk = "k_tc2<Affine,4,256,pair,A in TMEM>"
        groups["prefill_m16"] = affine_work(gwb, dev, "prefill M=16", PREFILL, 16, 4, GS, "k_tc2<Affine,4,32>")
        groups["prefill_m128"] = affine_work(gwb, dev, "prefill M=128", PREFILL, 128, 4, GS, "k_tc2<Affine,4,128>")
        groups["prefill_m512"] = affine_work(gwb, dev, "prefill M=512", PREFILL, 512, 4, GS, pk)
        groups["prefill_m2048"] = affine_work(gwb, dev, "prefill M=2048", PREFILL, M_PREFILL, 4, GS, pk)
        groups["prefill_m2048_b8"] = affine_work(gwb, dev, "prefill M=2048 8-bit", PREFILL, M_PREFILL, 8, GS,
                                                 "k_tc2<Affine,8,256,pair,A in TMEM>")
        groups["prefill_m2048_gs32"] = affine_work(gwb, dev, "prefill M=2048 gs32", PREFILL, M_PREFILL, 4, 32, pk)
        groups["prefill_m2048_gs128"] = affine_work(gwb, dev, "prefill M=2048 gs128", PREFILL, M_PREFILL, 4, 128, pk)
        groups["gptq_dequant"] = [gptq_work(gwb, dev, 0, p, dequant=True) for p in (False, True)]
        for M in (1, 32, 1024):
            groups[f"gptq_m{M}"] = [gptq_work(gwb, dev, M, p) for p in (False, True)]
        for fmt in ("w4a8", "w8a8"):
            for M in INT8_M:
                groups[f"{fmt}_m{M}"] = int8_work(gwb, dev, fmt, INT8_SHAPES, M)
        groups["w8a8_m1"] = int8_work(gwb, dev, "w8a8", [(14336, 4096)], 1)
    with torch.cuda.stream(stream):
        for layers in sets:
            for (wq, sc, bi, x, y, bits) in layers:
                gwb.qmm_affine(x, wq, sc, bi, bits, GS, y=y)
        for ws in groups.values():
            for w in ws:
                w.launch(0)
    torch.cuda.synchronize()
    gwb.check_device_error()

    # ---- CPU baseline leg: the oracle, timed, and compared with the outputs above
    cpu, parity = None, None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        with torch.cuda.stream(stream):
            checks = [c() for ws in groups.values() for w in ws for c in w.checks]
        torch.cuda.synchronize()
        cpu, parity = cpu_leg(checks, sets, args.cpu_seconds, threads=min(16, os.cpu_count() or 1))
        if not parity["ok"]:
            print(json.dumps({"metric": METRIC, "error": "parity check before timing failed", "parity": parity}),
                  flush=True)
            sys.exit(1)

    # ---- the decode step: one CUDA graph per step of the seven GEMVs (programmatic launch
    # chains them); consecutive steps alternate between the two weight sets
    n_graphs = max(args.steps, 1)
    graphs = []
    with torch.cuda.stream(stream):
        torch.cuda.synchronize()
        for gi in range(n_graphs):
            layers = sets[gi % len(sets)]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for (wq, sc, bi, x, y, bits) in layers:
                    gwb.qmm_affine(x, wq, sc, bi, bits, GS, y=y)
            graphs.append(g)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            graphs[i % n_graphs].replay()
    torch.cuda.synchronize()

    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    # clocks are sampled from here through the last timed group (the step alone is a few ms)
    clk = ClockSampler(local).__enter__()
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
    del graphs

    # ---- the dominant kernel alone: the lm_head GEMV in a graph of back-to-back launches
    # alternating the two weight sets (296 MB, over twice the L2)
    def lm_launch(i):
        wq, sc, bi, x, y, bits = sets[i % 2][lm_idx]
        gwb.qmm_affine(x, wq, sc, bi, bits, GS, y=y)

    lm_us = graph_us(lm_launch, 20, stream, replays=5)
    lm_bytes = gemv_bytes(*LMHEAD)
    achieved = lm_bytes / (lm_us * 1e-6) / 1e9

    # ---- end to end through the public API: per step one H2D copy of the seven activation
    # vectors from pinned host memory, the seven qmm_affine calls, one D2H copy of the outputs
    Ks = [K for _, K, _ in DECODE]
    Ns = [N for N, _, _ in DECODE]
    xoff = np.concatenate([[0], np.cumsum(Ks)])
    yoff = np.concatenate([[0], np.cumsum(Ns)])
    host_x = torch.cat([l[3].cpu().reshape(-1) for l in sets[0]]).pin_memory()
    host_y = torch.empty(int(yoff[-1]), dtype=torch.bfloat16).pin_memory()
    dev_x = torch.empty_like(host_x, device=dev)
    dev_y = torch.empty(int(yoff[-1]), dtype=torch.bfloat16, device=dev)
    xs = [dev_x[xoff[j]:xoff[j + 1]].view(1, -1) for j in range(len(DECODE))]
    ys = [dev_y[yoff[j]:yoff[j + 1]].view(1, -1) for j in range(len(DECODE))]
    h2d, d2h = host_x.numel() * 2, host_y.numel() * 2

    def e2e_step(i):
        layers = sets[i % len(sets)]
        dev_x.copy_(host_x, non_blocking=True)
        for j, (wq, sc, bi, _, _, bits) in enumerate(layers):
            gwb.qmm_affine(xs[j], wq, sc, bi, bits, GS, y=ys[j])
        host_y.copy_(dev_y, non_blocking=True)

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

    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": 1, "group_size": GS, "bytes_per_step": STEP_BYTES,
                   "l2": "inputs larger than L2: 192 MB of weights per step, two weight sets rotate (384 MB)",
                   "graphs": "each step replays its own CUDA graph of the seven GEMVs",
                   "parallelism": f"replicas x{world}"},
        "roofline": roofline("k_gemv_pipe<4,64,1> (lm_head 128256x2048)", "hbm", achieved, hbm_peak, "GB/s", hbm_src,
                             traffic_for("k_gemv_pipe_lmhead"), bytes_per_launch=lm_bytes,
                             avg_launch_us=round(lm_us, 2),
                             timing="CUDA graph of 20 back-to-back lm_head launches alternating two weight sets "
                                    "(296 MB), events around 5 replays"),
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "note": "weights resident in HBM; per step: one H2D copy of the 7 activation vectors (pinned), "
                        "7 qmm_affine calls through the public API, one D2H copy of the 7 outputs"},
        "gpu_launches": len(DECODE) * args.steps,
    }
    if parity is not None:
        out["parity"] = parity

    if full:
        i8peak = int8_peak_tops(dev, stream)
        i8src = "measured in this run: torch._int_mm 8192^3 int8, best of 5"
        t = {k: run_works(ws, stream) for k, ws in groups.items()}
        for M in PREFILL_M:
            key = f"prefill_m{M}"
            if M <= 128:
                out[key] = aggregate(key, t[key], hbm_peak, hbm_src, "GB/s", "hbm",
                                     traffic_key=f"k_tc2_affine4_m{M}")
            if M >= 128:
                k2 = key if M > 128 else key + "_tflops"
                out[k2] = aggregate(key, t[key], bf16_peak, bf16_src, "TFLOP/s", "tensor",
                                    traffic_key=f"k_tc2_affine4_m{M}")
        for key, tk in (("prefill_m2048_b8", "k_tc2_affine8_m2048"), ("prefill_m2048_gs32", "k_tc2_affine4_gs32_m2048"),
                        ("prefill_m2048_gs128", "k_tc2_affine4_gs128_m2048")):
            out[key] = aggregate(key, t[key], bf16_peak, bf16_src, "TFLOP/s", "tensor", traffic_key=tk)
        out["gptq_dequant"] = aggregate("gptq_dequant", t["gptq_dequant"][:1], hbm_peak, hbm_src, "GB/s", "hbm",
                                        traffic_key="k_gptq_dequant",
                                        extra={"permuted_g_idx": aggregate("gptq_dequant", t["gptq_dequant"][1:],
                                                                           hbm_peak, hbm_src, "GB/s", "hbm",
                                                                           traffic_key="k_gptq_dequant_perm")})
        for M in (1, 32, 1024):
            key = f"gptq_m{M}"
            tm = t[key]
            if M >= 512:
                out[key] = aggregate(key, tm[:1], bf16_peak, bf16_src + " (fp16 peak taken equal to bf16)",
                                     "TFLOP/s", "tensor", traffic_key="k_tc2_gptq_m1024", extra={"permuted_g_idx": aggregate(
                                         key, tm[1:], bf16_peak, bf16_src, "TFLOP/s", "tensor",
                                         traffic_key="k_gptq_dequant_tc2_f16_m1024")})
            else:
                out[key] = aggregate(key, tm[:1], hbm_peak, hbm_src, "GB/s", "hbm",
                                     traffic_key="k_gemv_gptq_pipe_m1" if M == 1 else "k_tc2_gptq_m32",
                                     extra={"permuted_g_idx": aggregate(
                                         key, tm[1:], hbm_peak, hbm_src, "GB/s", "hbm",
                                         traffic_key="k_gemv_gptq_pipe_perm_m1" if M == 1 else "k_gptq_dequant_tc2_f16_m32")})
        for fmt in ("w4a8", "w8a8"):
            for M in INT8_M:
                key = f"{fmt}_m{M}"
                if M >= 512:
                    out[key] = aggregate(key, t[key], i8peak, i8src, "TOP/s", "tensor",
                                         traffic_key=f"k_tc2_{fmt}_m{M}")
                else:
                    out[key] = aggregate(key, t[key], hbm_peak, hbm_src, "GB/s", "hbm",
                                         traffic_key=f"k_gemv_pipe_i8w8_m{M}" if fmt == "w8a8" and M <= 8
                                         else f"k_tc2_{fmt}_m{M}")
        out["w8a8_m1"] = aggregate("w8a8_m1", t["w8a8_m1"], hbm_peak, hbm_src, "GB/s", "hbm", traffic_key="k_gemv_pipe_i8w8")
        out["int8_peak_tops"] = round(i8peak, 1)
    out["decode_mlp_fused"] = run_mlp_fused(gwb, dev, stream, hbm_peak, hbm_src)
    out["w4a8_decode_fused"] = run_w4a8_decode(gwb, dev, stream, hbm_peak, hbm_src)
    clk.__exit__(None, None, None)
    out["clocks"] = dict(clk.summary(), window="the decode step's timed region through the last timed group")
    if cpu is not None:
        out["cpu_baseline"] = cpu
    gwb.check_device_error()
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
    w = dev_weight(dev, N, K, seed)
    wq, sw = gwb.qpack_sym_i4(w) if fmt == "w4a8" else gwb.qpack_sym_i8(w)
    del w
    x = synth.activations(M, K, seed=1).to(dev)
    qx, sx = gwb.quant_per_token_i8(x)
    return wq, sw, qx, sx


def int8_gemm(gwb, fmt):
    return gwb.gemm_i8i4 if fmt == "w4a8" else gwb.gemm_i8i8


def run_w4a8_decode(gwb, dev, stream, hbm_peak, hbm_src, N=14336, K=4096, M=1):
    """W4A8 at decode: the fused product (activations quantized inside the kernel) against the
    two-launch path (quant_per_token_i8, then gemm_i8i4), each a CUDA graph of back-to-back
    launches rotating through weight copies (> 2x L2)."""
    wq, sw, _, _ = int8_operands(gwb, dev, "w4a8", N, K, M)
    cps = clone_all((wq, sw), copies_for(N * K // 2))
    x = synth.activations(M, K, seed=1).to(dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    qx = torch.empty((M, K), dtype=torch.int8, device=dev)
    sx = torch.empty((M,), dtype=torch.float32, device=dev)

    def fused(i):
        w, s = cps[i % len(cps)]
        gwb.gemv_w4a8(x, w, s, y=y)

    def two(i):
        w, s = cps[i % len(cps)]
        gwb.quant_per_token_i8(x, qx=qx, sx=sx)
        gwb.gemm_i8i4(qx, sx, w, s, y=y)

    us_f = graph_us(fused, len(cps), stream)
    us_t = graph_us(two, len(cps), stream)
    nbytes = N * K // 2 + N * 4 + 2 * M * K + 2 * M * N
    gbs = nbytes / us_f / 1e3
    return {"value": round(gbs, 1), "unit": "GB/s", "N": N, "K": K, "M": M,
            "us_fused": round(us_f, 2), "us_two_launch": round(us_t, 2),
            "roofline": roofline("k_gemv_pipe<4,64,1,w4a8> (per-token int8 quantization inside)", "hbm", gbs,
                                 hbm_peak, "GB/s", hbm_src, traffic_for("k_gemv_pipe_w4a8"), bytes_per_launch=nbytes)}


def run_mlp_fused(gwb, dev, stream, hbm_peak, hbm_src, bits=4, M=1):
    """Decode MLP of a Llama-3-8B layer (hidden 4096, intermediate 14336, MLX affine gs 64) through
    the fused products: gemv_gate_up, then gemv_silu_gate_resid.  A CUDA graph of back-to-back
    MLPs rotating through weight copies (> 2x L2)."""
    H, I = 4096, 14336
    ws = []
    for j, (n, k) in enumerate(((I, H), (I, H), (H, I))):
        w = dev_weight(dev, n, k, 500 + j)
        ws.append(gwb.qpack_affine(w, bits, GS))
        del w
    mlp_w = sum(gemv_bytes(n, k, bits, M=0) for n, k in ((I, H), (I, H), (H, I)))
    cps = [ws] + [[tuple(t.clone() for t in w3) for w3 in ws] for _ in range(copies_for(mlp_w) - 1)]
    x = synth.activations(M, H, seed=1).to(dev)
    gate = torch.empty((M, I), dtype=torch.bfloat16, device=dev)
    up = torch.empty((M, I), dtype=torch.bfloat16, device=dev)
    y = torch.empty((M, H), dtype=torch.bfloat16, device=dev)

    def mlp(i):
        wg, wu, wd = cps[i % len(cps)]
        gwb.gemv_gate_up(x, wg, wu, bits, GS, y_gate=gate, y_up=up)
        gwb.gemv_silu_gate(gate, up, *wd, bits, GS, x_resid=x, y=y)

    us = graph_us(mlp, len(cps), stream)
    nbytes = (2 * gemv_bytes(I, H, bits, M=M) - 2 * M * H) + (gemv_bytes(H, I, bits, M=M) + 2 * M * I + 2 * M * H)
    gbs = nbytes / us / 1e3
    return {"value": round(gbs, 1), "unit": "GB/s", "M": M, "bits": bits, "group_size": GS,
            "us_per_mlp": round(us, 2), "bytes_per_mlp": nbytes, "launches_per_mlp": 2,
            "roofline": roofline("k_gemv_pipe<dual> + k_gemv_pipe<silu> (Llama-3-8B MLP, hidden 4096)", "hbm", gbs,
                                 hbm_peak, "GB/s", hbm_src, traffic=mlp_traffic())}


def mlp_traffic():
    """DRAM bytes of one fused MLP at decode: the gate/up launch plus the silu launch."""
    a, b = traffic_for("k_gemv_pipe_dual"), traffic_for("k_gemv_pipe_silu")
    return None if a is None or b is None else a + b


# ------------------------------------------------------------------ CPU oracle (reference arm)
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
    """One layer only (for profiling): qmm_affine (or, with --fmt, another product) on an N x K
    weight at M tokens, replayed in a CUDA graph of 20 launches that alternate between two
    weight sets (> L2)."""
    import group_wise_bit_b200 as gwb
    N, K, bits, M = (list(map(int, args.layer.split(","))) + [1])[:4]
    dev = torch.device("cuda", 0)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    if args.fmt == "affine":
        sets = []
        for s in range(2):
            w = dev_weight(dev, N, K, s)
            sets.append(gwb.qpack_affine(w, bits, args.gs))
            del w
        x = synth.activations(M, K, seed=1).to(dev)

        def launch(i):
            wq, sc, bi = sets[i % 2]
            gwb.qmm_affine(x, wq, sc, bi, bits, args.gs, y=y)
    elif args.fmt in ("gate_up", "silu_resid"):
        sets = []
        for s in range(2):
            ws = []
            for j in range(2 if args.fmt == "gate_up" else 1):
                w = dev_weight(dev, N, K, 10 * s + j)
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
    elif args.fmt in ("gptq", "gptq_perm", "gptq_dequant", "gptq_dequant_perm"):
        perm = args.fmt in ("gptq_perm", "gptq_dequant_perm")
        sets = []
        for s in range(2):
            qw, sc, qz, gi = synth.gptq_quartet(K, N, GPTQ_GS, seed=s, permuted=perm)
            sets.append((qw.to(dev), sc.to(dev), qz.to(dev), gi.to(dev) if perm else None))
        x = synth.activations(M, K, seed=1, dtype=torch.float16).to(dev)
        y = torch.empty((M, N), dtype=torch.float16, device=dev)
        wo = torch.empty((N, K), dtype=torch.float16, device=dev) if args.fmt.startswith("gptq_dequant") else None
        bits = 4

        def launch(i):
            q, s, z, gi = sets[i % 2]
            if wo is not None:
                gwb.gptq_dequant(q, s, z, gi, GPTQ_GS, out=wo)
            else:
                gwb.gptq_qmm(x, q, s, z, gi, GPTQ_GS, y=y)
    elif args.fmt == "w4a8_fused":
        sets = [int8_operands(gwb, dev, "w4a8", N, K, M, seed=s)[:2] for s in range(2)]
        x = synth.activations(M, K, seed=1).to(dev)
        bits = 4

        def launch(i):
            wq, sw = sets[i % 2]
            gwb.gemv_w4a8(x, wq, sw, y=y)
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
    elif args.fmt.startswith("gptq_dequant"):
        nbytes = gptq_dequant_bytes(K, N, GPTQ_GS, args.fmt == "gptq_dequant_perm")
    elif args.fmt in ("gptq", "gptq_perm"):
        nbytes = gptq_bytes(K, N, GPTQ_GS, M, args.fmt == "gptq_perm") if M <= 32 else None
    elif args.fmt == "w4a8_fused":
        nbytes = N * K // 2 + 4 * N + 2 * M * K + 2 * M * N
    else:
        nbytes = int8_bytes(N, K, M, bits) if M <= 64 else None
    out = {"layer": {"fmt": args.fmt, "N": N, "K": K, "bits": bits,
                     "group_size": GPTQ_GS if args.fmt.startswith("gptq") else args.gs, "M": M},
           "us_per_launch": round(us, 2)}
    if nbytes:
        out["GB/s"] = round(nbytes / us / 1e3, 1)
    else:
        out["TFLOP/s" if args.fmt in ("affine", "gptq", "gptq_perm") else "TOP/s"] = round(2.0 * M * N * K / us / 1e6, 1)
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["gwb", "reference"], default="gwb")
    ap.add_argument("--no-prefill", action="store_true",
                    help="time the decode sweep (and the fused decode products) only")
    ap.add_argument("--fmt", choices=["affine", "w4a8", "w8a8", "gate_up", "silu_resid", "gptq", "gptq_perm",
                                      "gptq_dequant", "gptq_dequant_perm", "w4a8_fused"], default="affine",
                    help="--layer: weight format (affine: MLX group-wise, bits from --layer; gptq*: N,K = out, in "
                         "features at group size 128)")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the CPU baseline leg (and with it the parity check before timing)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-frac", type=float, default=1 / 16)
    ap.add_argument("--layer", default=None,
                    help="N,K,bits[,M]: time one layer (qmm_affine at group size 64, or --fmt) instead of the sweep")
    ap.add_argument("--gs", type=int, default=GS, help="--layer with --fmt affine: the group size")
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

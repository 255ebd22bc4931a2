"""GPU parity: the CUDA library (through the C ABI) against the CPU oracle on
the same seeded inputs.

Integer / byte work (packing, unpacking, dequantized weights, per-token int8,
W4A8 int32 accumulators) must be bit-exact; float matmul outputs must meet the
tolerance in tests/tol.py.  Small cases span several tiles and ragged tails in
N, M and K; the full-size cases use the workloads' shapes, with the oracle
evaluated on sampled output rows where all rows would take too long.
"""
import concurrent.futures as cf
import os

import numpy as np
import pytest
import torch

import gwb_synth as synth
import oracle
from tol import check_float

gwb = pytest.importorskip("group_wise_bit_b200")
pytestmark = pytest.mark.gpu

DEV = "cuda"


def _np16(t):
    return synth.bits16(t.cpu())


def _words(t):
    return t.cpu().numpy().view(np.uint32)


TOKEN_BLOCK = 128   # the smallest token tile of the tensor-core kernels (256-token tiles hold two blocks)


def _rows(M, N, K, seed=0, budget=3e8):
    """All rows when the oracle finishes quickly, else: the first and last rows, one
    seeded row inside every block of TOKEN_BLOCK tokens (so every token tile of
    every kernel, and with all N columns every output tile and every stream-K
    share, is compared), and a seeded sample of further rows (about `budget`
    multiply-adds on top)."""
    if M * N * K <= budget or M <= 2:
        return None
    rng = np.random.default_rng(seed)
    blocks = [b + int(rng.integers(0, min(TOKEN_BLOCK, M - b))) for b in range(0, M, TOKEN_BLOCK)]
    n = int(max(0, min(M - 2, budget // (N * K) - 2)))
    r = rng.choice(np.arange(1, M - 1), size=n, replace=False) if n else []
    return np.unique(np.concatenate([[0, M - 1], blocks, r]).astype(np.int64))


ORACLE_THREADS = max(1, min(32, os.cpu_count() or 1))


def _by_rows(fn, *args, rows=None, **kw):
    """fn(*args, rows=..., **kw) of the oracle, with a long row list split over
    threads (the oracle's C calls release the GIL); the results are put back
    together in row order: arrays concatenated, flags or-ed."""
    if rows is None or len(rows) < 2 * ORACLE_THREADS // 4 or ORACLE_THREADS == 1:
        return fn(*args, rows=rows, **kw)
    chunks = [c for c in np.array_split(np.asarray(rows), min(ORACLE_THREADS, len(rows))) if len(c)]
    with cf.ThreadPoolExecutor(len(chunks)) as ex:
        parts = list(ex.map(lambda c: fn(*args, rows=c, **kw), chunks))
    if isinstance(parts[0], tuple):
        return tuple(np.concatenate([p[i] for p in parts]) if isinstance(parts[0][i], np.ndarray)
                     else any(p[i] for p in parts) for i in range(len(parts[0])))
    return np.concatenate(parts)


def _affine_max_w(sc, bi, bits):
    s = oracle.bf16_array_to_f64(sc)
    b = oracle.bf16_array_to_f64(bi)
    return float(np.max(np.maximum(np.abs(b), np.abs(b + ((1 << bits) - 1) * s))))


class Affine:
    """A quantized MLX-affine linear built on both sides from one fp32 weight."""

    def __init__(self, N, K, bits, gs, seed=0):
        self.N, self.K, self.bits, self.gs = N, K, bits, gs
        w = synth.weights(N, K, seed=seed)
        self.wq_o, self.sc_o, self.bi_o, _ = oracle.qpack_affine(w.numpy(), bits, gs)
        self.wq, self.sc, self.bi = gwb.qpack_affine(w.to(DEV), bits, gs)
        torch.cuda.synchronize()
        self.max_w = _affine_max_w(self.sc_o, self.bi_o, bits)

    def check_pack(self):
        assert np.array_equal(_words(self.wq), self.wq_o), "packed words differ"
        assert np.array_equal(_np16(self.sc), self.sc_o), "scales differ"
        assert np.array_equal(_np16(self.bi), self.bi_o), "biases differ"

    def check_qmm(self, M, seed=1, outlier_frac=0.0, label=""):
        x = synth.activations(M, self.K, seed=seed, outlier_frac=outlier_frac)
        y = gwb.qmm_affine(x.to(DEV), self.wq, self.sc, self.bi, self.bits, self.gs)
        rows = _rows(M, self.N, self.K)
        y_ref = _by_rows(oracle.qmm_affine, synth.bits16(x), self.wq_o, self.sc_o, self.bi_o, self.N, self.K,
                         self.bits, self.gs, rows=rows)
        yg = y.float().cpu().numpy()
        if rows is not None:
            yg = yg[rows]
        max_x = float(x.float().abs().max())
        return check_float(yg, y_ref, self.K, self.max_w, max_x, label or f"qmm M={M}")


# --------------------------------------------------------------------------- packing
@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("gs", [32, 64, 128])
def test_qpack_and_dequant_affine_bit_exact(bits, gs):
    N, K = 300, 4 * 128
    a = Affine(N, K, bits, gs, seed=bits * 10 + gs)
    a.check_pack()
    w_deq = gwb.dequant_affine(a.wq, a.sc, a.bi, K, bits, gs)
    ref = oracle.dequant_affine_bf16(a.wq_o, a.sc_o, a.bi_o, N, K, bits, gs)
    assert np.array_equal(_np16(w_deq), ref)


def test_qpack_affine_signed_zeros_and_constant_groups():
    w = synth.weights(16, 128, seed=5)
    w[0, :64] = 0.0
    w[0, 5] = -0.0
    w[1, :32] = 0.25
    w[2, 64:] = -0.0
    w[2, 70] = 0.0
    wq_o, sc_o, bi_o, _ = oracle.qpack_affine(w.numpy(), 4, 32)
    wq, sc, bi = gwb.qpack_affine(w.to(DEV), 4, 32)
    assert np.array_equal(_words(wq), wq_o)
    assert np.array_equal(_np16(sc), sc_o)
    assert np.array_equal(_np16(bi), bi_o)


def test_qpack_sym_i4_bit_exact():
    w = synth.weights(333, 512, seed=9)
    w[7] = 0.0
    wq_o, sw_o, _ = oracle.qpack_sym_i4(w.numpy())
    wq, sw = gwb.qpack_sym_i4(w.to(DEV))
    assert np.array_equal(_words(wq), wq_o)
    assert np.array_equal(sw.cpu().numpy(), sw_o)


@pytest.mark.parametrize("M,K", [(1, 512), (7, 4096), (64, 1000), (300, 96), (5, 14336)])
def test_quant_per_token_i8_bit_exact(M, K):
    x = synth.activations(M, K, seed=M + K, outlier_frac=0.01)
    if M > 3:
        x[2] = 0
    qx_o, sx_o = oracle.quant_per_token_i8(synth.bits16(x))
    qx, sx = gwb.quant_per_token_i8(x.to(DEV))
    assert np.array_equal(sx.cpu().numpy(), sx_o)
    assert np.array_equal(qx.cpu().numpy(), qx_o)


# --------------------------------------------------------------------------- affine qmm
@pytest.mark.parametrize("bits,gs", [(4, 64), (4, 32), (4, 128), (8, 32), (8, 64), (8, 128), (2, 64), (2, 128)])
@pytest.mark.parametrize("M", [1, 3, 8])
def test_qmm_affine_gemv_small(bits, gs, M):
    a = Affine(200, 1024, bits, gs, seed=bits + gs)
    a.check_qmm(M, label=f"gemv b{bits} gs{gs} M{M}")


@pytest.mark.parametrize("bits,gs", [(4, 64), (4, 32), (8, 128), (8, 64), (2, 64), (2, 32)])
@pytest.mark.parametrize("M", [9, 16, 40, 130, 300])
def test_qmm_affine_tensor_core_small(bits, gs, M):
    # N = 300 ragged against the 128-row tile; K = 384 = 6 K-steps
    a = Affine(300, 384, bits, gs, seed=bits * gs)
    a.check_qmm(M, outlier_frac=0.01, label=f"tc b{bits} gs{gs} M{M}")


@pytest.mark.parametrize("gs", [32, 64])
@pytest.mark.parametrize("M", [9, 16, 40, 130, 300])
def test_qmm_affine_tensor_core_odd_groups(gs, M):
    # K = 192: three groups per row at gs 64 (six at gs 32), 3 K steps of 64; an odd
    # number of groups per row is staged by the per-tile kernel at every M
    a = Affine(300, 192, 4, gs, seed=gs + 1)
    a.check_qmm(M, outlier_frac=0.01, label=f"tc K=192 gs{gs} M{M}")


@pytest.mark.parametrize("M", [1, 5])
def test_qmm_affine_gemv_register_fed_fallback(M):
    # an odd number of groups per row (K / gs = 3) is served by the register-fed GEMV
    Affine(264, 192, 4, 64).check_qmm(M, label=f"register-fed GEMV M={M}")


@pytest.mark.parametrize("bits,M", [(4, 1), (4, 3), (8, 2), (2, 1)])
def test_qmm_affine_gemv_persistent_tiles(bits, M):
    # 157 tiles of 128 rows on 148 persistent CTAs: some CTAs stream two tiles
    Affine(20000, 512, bits, 64, seed=3).check_qmm(M, label=f"persistent b{bits} M={M}")


@pytest.mark.parametrize("N,K,bits,gs,M", [
    (264, 768, 4, 32, 1),      # 1.5 stages of 512 k: the last stage is zero-filled past K
    (264, 768, 4, 32, 5),
    (136, 1536, 2, 64, 2),     # 1.5 stages of 1024 k
    (200, 384, 4, 64, 1),      # K / gs = 6 (not a multiple of 8): the per-warp-ring GEMV
    (200, 384, 4, 64, 8),
    (256, 4096, 8, 64, 7),     # 16 strips: K split over a cluster, 7 tokens
    (48, 8192, 4, 128, 4),     # 3 strips: the widest K split
])
def test_qmm_affine_gemv_layout_edges(N, K, bits, gs, M):
    Affine(N, K, bits, gs, seed=N + K).check_qmm(M, label=f"gemv edge {N}x{K} b{bits} gs{gs} M{M}")


def test_qmm_affine_k_tail_and_unsupported_gemv_combo():
    # K = 96 (1.5 tensor-core K steps), and 2-bit gs32 at M=1 (no GEMV kernel: tensor-core path)
    Affine(256, 96, 4, 32).check_qmm(20, label="K tail")
    Affine(136, 256, 2, 32).check_qmm(1, label="2-bit gs32 M=1")


def test_qmm_affine_rejects_2bit_k_not_multiple_of_64_on_tc_path():
    a = Affine(64, 96, 2, 32)
    x = torch.zeros(16, 96, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(gwb.GwbError, match="UNSUPPORTED"):
        gwb.qmm_affine(x, a.wq, a.sc, a.bi, 2, 32)


def test_qmm_affine_degenerate_inputs():
    a = Affine(128, 256, 4, 64)
    x = torch.zeros(4, 256, dtype=torch.bfloat16, device=DEV)
    y = gwb.qmm_affine(x, a.wq, a.sc, a.bi, 4, 64)
    assert torch.all(y == 0)
    y = gwb.qmm_affine(torch.zeros(0, 256, dtype=torch.bfloat16, device=DEV), a.wq, a.sc, a.bi, 4, 64)
    assert y.shape == (0, 128)


# --------------------------------------------------------------------------- GPTQ
class Gptq:
    def __init__(self, K, N, gs, permuted, seed=0):
        self.K, self.N, self.gs = K, N, gs
        qw, sc, qz, gi = synth.gptq_quartet(K, N, gs, seed=seed, permuted=permuted)
        self.h = (qw.numpy(), synth.bits16(sc), qz.numpy(), gi.numpy() if permuted else None)
        self.d = (qw.to(DEV), sc.to(DEV), qz.to(DEV), gi.to(DEV) if permuted else None)

    def check_dequant(self):
        w = gwb.gptq_dequant(*self.d, self.gs)
        ref = oracle.gptq_dequant_f16(*self.h, self.K, self.N, self.gs)
        assert np.array_equal(_np16(w), ref)
        return float(w.float().abs().max())

    def check_qmm(self, M, seed=1):
        max_w = self.check_dequant()
        x = synth.activations(M, self.K, seed=seed, dtype=torch.float16)
        y = gwb.gptq_qmm(x.to(DEV), *self.d, self.gs)
        rows = _rows(M, self.N, self.K, budget=2e9)
        y_ref = _by_rows(oracle.gptq_qmm, synth.bits16(x), *self.h, self.K, self.N, self.gs, rows=rows)
        yg = y.float().cpu().numpy()
        if rows is not None:
            yg = yg[rows]
        return check_float(yg, y_ref, self.K, max_w, float(x.float().abs().max()), f"gptq M={M}")


@pytest.mark.parametrize("permuted", [False, True])
@pytest.mark.parametrize("gs", [32, 128])
def test_gptq_dequant_bit_exact(permuted, gs):
    Gptq(512, 200, gs, permuted, seed=gs).check_dequant()


@pytest.mark.parametrize("permuted", [False, True])
@pytest.mark.parametrize("M", [1, 4, 8, 32, 150])
def test_gptq_qmm_small(permuted, M):
    Gptq(384, 264, 128 if M % 2 else 64, permuted, seed=M).check_qmm(M)


@pytest.mark.parametrize("permuted", [False, True])
@pytest.mark.parametrize("K,N,gs", [(256, 32, 32), (768, 96, 64), (1280, 4800, 64), (2048, 9536, 32),
                                    (1024, 4800, 128)])
def test_gptq_gemv_streamed_layouts(permuted, K, N, gs):
    """The shared-memory streamed GEMV (N % 32 == 0, K % 256 == 0): one strip; fewer strips
    than SMs; more strips than SMs with a remainder (150 and 298 strips on 148 SMs); strips cut
    between warps at every stage boundary (5 stages a strip); 8, 4 and 2 groups a stage; M from 1
    to 8 (token padding 1, 2, 4, 8 with ragged M)."""
    g = Gptq(K, N, gs, permuted, seed=K + N)
    for M in (1, 2, 3, 5, 8):
        g.check_qmm(M, seed=M)


# --------------------------------------------------------------------------- fused decode products
def _gate_up_case(N, K, bits, gs, M, seed):
    g = Affine(N, K, bits, gs, seed=seed)
    u = Affine(N, K, bits, gs, seed=seed + 1)
    x = synth.activations(M, K, seed=seed + 2, outlier_frac=0.01)
    yg, yu = gwb.gemv_gate_up(x.to(DEV), (g.wq, g.sc, g.bi), (u.wq, u.sc, u.bi), bits, gs)
    rows = _rows(M, N, K)
    rg, ru = oracle.qmv_gate_up(synth.bits16(x), (g.wq_o, g.sc_o, g.bi_o), (u.wq_o, u.sc_o, u.bi_o), N, K, bits, gs,
                                rows=rows)
    max_x = float(x.float().abs().max())
    for y, ref, w, name in ((yg, rg, g, "gate"), (yu, ru, u, "up")):
        yy = y.float().cpu().numpy()
        if rows is not None:
            yy = yy[rows]
        check_float(yy, ref, K, w.max_w, max_x, f"gate_up {name} {N}x{K} b{bits} gs{gs} M={M}")


@pytest.mark.parametrize("bits,gs", [(8, 64), (8, 32), (4, 64), (4, 128), (2, 64)])
@pytest.mark.parametrize("M", [1, 3, 8])
def test_gemv_gate_up(bits, gs, M):
    _gate_up_case(200, 1024, bits, gs, M, seed=bits + M)      # ragged last strip of each weight


@pytest.mark.parametrize("N,K", [(64, 8192), (48, 2048), (1000, 512)])
def test_gemv_gate_up_split_layouts(N, K):
    # few strips: K split over a cluster; many short strips: strips shared by warps
    _gate_up_case(N, K, 8, 64, 2, seed=N)


def _silu_case(N, K, bits, gs, M, seed, resid=False, alias=False):
    a = Affine(N, K, bits, gs, seed=seed)
    gate = (synth.activations(M, K, seed=seed + 1) * 4).to(torch.bfloat16)
    up = synth.activations(M, K, seed=seed + 2, outlier_frac=0.01)
    res = synth.activations(M, N, seed=seed + 3) if resid else None
    dres = res.to(DEV) if resid else None
    y = gwb.gemv_silu_gate(gate.to(DEV), up.to(DEV), a.wq, a.sc, a.bi, bits, gs, x_resid=dres,
                           y=dres if alias else None)
    rows = _rows(M, N, K)
    ref = oracle.qmv_silu_gate(synth.bits16(gate), synth.bits16(up), a.wq_o, a.sc_o, a.bi_o, N, K, bits, gs,
                               resid_bf16=synth.bits16(res) if resid else None, rows=rows)
    yy = y.float().cpu().numpy()
    if rows is not None:
        yy = yy[rows]
    max_x = float(np.abs(oracle.silu_mul(synth.bits16(gate), synth.bits16(up))).max())
    return check_float(yy, ref, K, a.max_w, max_x, f"silu_gate {N}x{K} b{bits} gs{gs} M={M} resid={resid}")


@pytest.mark.parametrize("bits,gs", [(8, 64), (4, 64), (4, 128), (2, 128)])
@pytest.mark.parametrize("M", [1, 2, 5, 8])
@pytest.mark.parametrize("resid", [False, True])
def test_gemv_silu_gate(bits, gs, M, resid):
    _silu_case(136, 2048, bits, gs, M, seed=bits * 7 + M, resid=resid)


def test_gemv_silu_gate_resid_in_place():
    _silu_case(256, 1024, 8, 64, 4, seed=3, resid=True, alias=True)   # x_resid is y


def test_fused_decode_argument_errors():
    a = Affine(64, 384, 4, 64, seed=1)                 # K / gs = 6: not a multiple of 8
    x = torch.zeros(1, 384, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(gwb.GwbError, match="UNSUPPORTED"):
        gwb.gemv_silu_gate(x, x, a.wq, a.sc, a.bi, 4, 64)
    b = Affine(64, 512, 4, 64, seed=2)
    x9 = torch.zeros(9, 512, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(gwb.GwbError, match="SHAPE"):
        gwb.gemv_gate_up(x9, (b.wq, b.sc, b.bi), (b.wq, b.sc, b.bi), 4, 64)
    y0g, y0u = gwb.gemv_gate_up(x9[:0], (b.wq, b.sc, b.bi), (b.wq, b.sc, b.bi), 4, 64)
    assert y0g.shape == (0, 64) and y0u.shape == (0, 64)


# --------------------------------------------------------------------------- AWQ zero convention
class Awq:
    """The GPTQ tensors without g_idx, the stored zero used as is."""

    def __init__(self, K, N, gs, seed=0):
        self.K, self.N, self.gs = K, N, gs
        qw, sc, qz, _ = synth.gptq_quartet(K, N, gs, seed=seed)
        self.h = (qw.numpy(), synth.bits16(sc), qz.numpy())
        self.d = (qw.to(DEV), sc.to(DEV), qz.to(DEV))

    def check_dequant(self):
        w = gwb.awq_dequant(*self.d, self.gs)
        ref = oracle.awq_dequant_f16(*self.h, self.K, self.N, self.gs)
        assert np.array_equal(_np16(w), ref)
        return float(w.float().abs().max())

    def check_qmm(self, M, seed=1):
        max_w = self.check_dequant()
        x = synth.activations(M, self.K, seed=seed, dtype=torch.float16)
        y = gwb.awq_qmm(x.to(DEV), *self.d, self.gs)
        rows = _rows(M, self.N, self.K, budget=2e9)
        y_ref = _by_rows(oracle.awq_qmm, synth.bits16(x), *self.h, self.K, self.N, self.gs, rows=rows)
        yg = y.float().cpu().numpy()
        if rows is not None:
            yg = yg[rows]
        return check_float(yg, y_ref, self.K, max_w, float(x.float().abs().max()), f"awq M={M}")


@pytest.mark.parametrize("gs", [32, 128])
def test_awq_dequant_bit_exact(gs):
    Awq(512, 200, gs, seed=gs).check_dequant()


@pytest.mark.parametrize("M", [1, 4, 8, 32, 150, 300])
def test_awq_qmm_small(M):
    Awq(384, 264, 128 if M % 2 else 64, seed=M).check_qmm(M)


@pytest.mark.parametrize("K,N,gs", [(1280, 4800, 64), (512, 64, 128)])
def test_awq_gemv_streamed_layouts(K, N, gs):
    a = Awq(K, N, gs, seed=K + N)
    for M in (1, 3, 8):
        a.check_qmm(M, seed=M)


def test_awq_equals_gptq_with_stored_zero_minus_one():
    """Both entry points on the same codes: AWQ with stored zeros z in 1..15 gives the same
    fp16 weights and outputs as GPTQ with stored zeros z - 1."""
    K, N, gs = 512, 192, 64
    qw, sc, qz, _ = synth.gptq_quartet(K, N, gs, seed=9)
    nib = [((qz.to(torch.int64) >> (4 * j)) & 0xF).clamp(min=1) for j in range(8)]
    pack = lambda d: sum((v - d) << (4 * j) for j, v in enumerate(nib)).to(torch.uint32).view(torch.int32)
    qz_awq, qz_gptq = pack(0).to(DEV), pack(1).to(DEV)
    qw, sc = qw.to(DEV), sc.to(DEV)
    assert torch.equal(gwb.awq_dequant(qw, sc, qz_awq, gs), gwb.gptq_dequant(qw, sc, qz_gptq, None, gs))
    for M in (1, 200):
        x = synth.activations(M, K, seed=M, dtype=torch.float16).to(DEV)
        assert torch.equal(gwb.awq_qmm(x, qw, sc, qz_awq, gs), gwb.gptq_qmm(x, qw, sc, qz_gptq, None, gs))


# --------------------------------------------------------------------------- W4A8
class W4A8:
    def __init__(self, N, K, seed=0):
        self.N, self.K = N, K
        w = synth.weights(N, K, seed=seed)
        self.wq_o, self.sw_o, _ = oracle.qpack_sym_i4(w.numpy())
        self.wq, self.sw = gwb.qpack_sym_i4(w.to(DEV))
        assert np.array_equal(_words(self.wq), self.wq_o) and np.array_equal(self.sw.cpu().numpy(), self.sw_o)

    def check(self, M, seed=1):
        x = synth.activations(M, self.K, seed=seed)
        qx_o, sx_o = oracle.quant_per_token_i8(synth.bits16(x))
        qx, sx = gwb.quant_per_token_i8(x.to(DEV))
        assert np.array_equal(qx.cpu().numpy(), qx_o) and np.array_equal(sx.cpu().numpy(), sx_o)
        y, acc = gwb.gemm_i8i4(qx, sx, self.wq, self.sw, want_y=True, want_acc=True)
        rows = _rows(M, self.N, self.K)
        acc_o, y_o, ovf = _by_rows(oracle.gemm_i8i4, qx_o, sx_o, self.wq_o, self.sw_o, self.N, self.K, rows=rows)
        assert not ovf
        a = acc.cpu().numpy().astype(np.int64)
        yg = y.float().cpu().numpy()
        if rows is not None:
            a, yg = a[rows], yg[rows]
        assert np.array_equal(a, acc_o), "int32 accumulators differ"
        max_w = float(np.max(np.abs(self.sw_o)) * 7)
        return check_float(yg, y_o, self.K, max_w, float(x.float().abs().max()), f"w4a8 M={M}")


@pytest.mark.parametrize("M", [1, 8, 16, 64, 100, 300])
def test_w4a8_small(M):
    W4A8(200, 384, seed=M).check(M)


def test_w4a8_k_tail():
    W4A8(136, 96).check(24)   # K = 96 < one 128-wide K step


# --------------------------------------------------------------------------- W8A8
class W8A8:
    def __init__(self, N, K, seed=0):
        self.N, self.K = N, K
        w = synth.weights(N, K, seed=seed)
        self.wq_o, self.sw_o = oracle.qpack_sym_i8(w.numpy())
        self.wq, self.sw = gwb.qpack_sym_i8(w.to(DEV))
        assert np.array_equal(self.wq.cpu().numpy(), self.wq_o) and np.array_equal(self.sw.cpu().numpy(), self.sw_o)

    def check(self, M, seed=1):
        x = synth.activations(M, self.K, seed=seed)
        qx_o, sx_o = oracle.quant_per_token_i8(synth.bits16(x))
        qx, sx = gwb.quant_per_token_i8(x.to(DEV))
        assert np.array_equal(qx.cpu().numpy(), qx_o) and np.array_equal(sx.cpu().numpy(), sx_o)
        y, acc = gwb.gemm_i8i8(qx, sx, self.wq, self.sw, want_y=True, want_acc=True)
        rows = _rows(M, self.N, self.K)
        acc_o, y_o, ovf = _by_rows(oracle.gemm_i8i8, qx_o, sx_o, self.wq_o, self.sw_o, self.N, self.K, rows=rows)
        assert not ovf
        a = acc.cpu().numpy().astype(np.int64)
        yg = y.float().cpu().numpy()
        if rows is not None:
            a, yg = a[rows], yg[rows]
        assert np.array_equal(a, acc_o), "int32 accumulators differ"
        # y alone (no acc) must match the y written next to acc
        y_only, none = gwb.gemm_i8i8(qx, sx, self.wq, self.sw, want_y=True, want_acc=False)
        assert none is None and torch.equal(y_only, y)
        max_w = float(np.max(np.abs(self.sw_o)) * 127)
        return check_float(yg, y_o, self.K, max_w, float(x.float().abs().max()), f"w8a8 M={M}")


@pytest.mark.parametrize("M", [1, 8, 31, 32, 33, 100, 128, 129, 300])
def test_w8a8_small(M):
    W8A8(200, 384, seed=M).check(M)


@pytest.mark.parametrize("N,K", [(200, 1024), (1000, 8192), (4096, 14336)])
@pytest.mark.parametrize("M", [1, 2, 3, 5, 8])
def test_w8a8_decode(N, K, M):
    # M <= 8 with K % 512 == 0: the weight-streaming decode kernel with exact int32 sums (K = 14336
    # with more than 4 tokens does not fit on chip and takes the tensor-core kernel)
    W8A8(N, K, seed=M).check(M)


@pytest.mark.parametrize("N,K,M", [(136, 96, 24), (264, 144, 40), (72, 272, 200)])
def test_w8a8_k_tail(N, K, M):
    W8A8(N, K).check(M)    # K below or between 128-wide K steps


@pytest.mark.parametrize("M", [1, 300, 512])
def test_w8a8_stream_k_split_tiles(M):
    # few tiles and 16 K steps each over 148 CTAs (74 pairs): tiles are split
    W8A8(2048, 2048, seed=5).check(M)


def test_w8a8_rejects_misaligned_and_bad_k():
    buf = torch.zeros(4 * 256 + 16, dtype=torch.int8, device=DEV)
    qx = buf[1:1 + 4 * 256].view(4, 256)
    wq = torch.zeros(64, 256, dtype=torch.int8, device=DEV)
    sx = torch.ones(4, device=DEV)
    sw = torch.ones(64, device=DEV)
    with pytest.raises(gwb.GwbError, match="ALIGN"):
        gwb.gemm_i8i8(qx, sx, wq, sw)
    with pytest.raises(gwb.GwbError, match="SHAPE"):
        gwb.gemm_i8i8(torch.zeros(4, 72, dtype=torch.int8, device=DEV), sx, wq[:, :72].contiguous(), sw)


# --------------------------------------------------------------------------- W4A8, quantization fused
@pytest.mark.parametrize("N,K", [(200, 1024), (4096, 4096), (1000, 8192), (1000, 14336)])
@pytest.mark.parametrize("M", [1, 2, 3, 5, 8])
def test_gemv_w4a8_matches_two_launch_path(N, K, M):
    """The fused product equals quant_per_token_i8 + gemm_i8i4 bit for bit, and the oracle within the
    float tolerance.  At K = 14336 with more than 4 tokens the rows do not fit one CTA: K is split
    over a cluster whose CTAs exchange their per-token maxima."""
    w = W4A8(N, K, seed=N + M)
    x = synth.activations(M, K, seed=M, outlier_frac=0.01)
    xd = x.to(DEV)
    y = gwb.gemv_w4a8(xd, w.wq, w.sw)
    qx, sx = gwb.quant_per_token_i8(xd)
    y2, _ = gwb.gemm_i8i4(qx, sx, w.wq, w.sw)
    assert torch.equal(y, y2), "fused W4A8 differs from the two-launch path"
    rows = _rows(M, N, K)
    acc_o, y_o, ovf = oracle.w4a8_fused(synth.bits16(x), w.wq_o, w.sw_o, N, K, rows=rows)
    assert not ovf
    yg = y.float().cpu().numpy()
    if rows is not None:
        yg = yg[rows]
    check_float(yg, y_o, K, float(np.max(np.abs(w.sw_o)) * 7), float(x.float().abs().max()), f"w4a8 fused M={M}")


def test_gemv_w4a8_argument_errors():
    w = W4A8(64, 256)
    with pytest.raises(gwb.GwbError, match="UNSUPPORTED"):      # K % 512 != 0
        gwb.gemv_w4a8(torch.zeros(1, 256, dtype=torch.bfloat16, device=DEV), w.wq, w.sw)
    w2 = W4A8(64, 512)
    with pytest.raises(gwb.GwbError, match="SHAPE"):            # more than 8 tokens
        gwb.gemv_w4a8(torch.zeros(9, 512, dtype=torch.bfloat16, device=DEV), w2.wq, w2.sw)
    z = gwb.gemv_w4a8(torch.zeros(2, 512, dtype=torch.bfloat16, device=DEV), w2.wq, w2.sw)
    assert torch.all(z == 0)                                     # all-zero tokens: sx = 0, q = 0


@pytest.mark.parametrize("bits,M", [(4, 512), (4, 300), (8, 512)])
def test_qmm_affine_stream_k_split_tiles(bits, M):
    # 8 x 2 tiles of 256 x 256 and 32 K steps over 74 CTA pairs: every tile is
    # split between four or five pairs and finished from their partials
    Affine(2048, 2048, bits, 64, seed=11).check_qmm(M, outlier_frac=0.01, label=f"stream-K b{bits} M={M}")


def test_w4a8_stream_k_split_tiles():
    W4A8(2048, 2048).check(512)


def test_stream_k_gemm_replayed_in_a_cuda_graph_with_new_inputs():
    """A stream-K GEMM captured into a CUDA graph: every replay takes a fresh epoch on the
    device, so replays with new activations in the same buffer are exactly the eager result
    (the same split and summation order), and match the oracle."""
    N, K, M = 2048, 2048, 512
    a = Affine(N, K, 4, 64, seed=12)
    xs = [synth.activations(M, K, seed=s, outlier_frac=0.01) for s in (5, 6)]
    eager = [gwb.qmm_affine(x.to(DEV), a.wq, a.sc, a.bi, 4, 64) for x in xs]
    st = torch.cuda.Stream()
    xd = xs[0].to(DEV)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    with torch.cuda.stream(st):
        gwb.qmm_affine(xd, a.wq, a.sc, a.bi, 4, 64, y=y)      # the stream's workspace exists before capture
        st.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            gwb.qmm_affine(xd, a.wq, a.sc, a.bi, 4, 64, y=y)
        for j in (0, 1, 0, 1, 1):
            xd.copy_(xs[j].to(DEV))
            y.fill_(float("nan"))
            g.replay()
            st.synchronize()
            assert torch.equal(y, eager[j]), f"replay with input {j} differs from the eager call"
    rows = np.array([0, 255, 256, 511])
    ref = oracle.qmm_affine(synth.bits16(xs[1]), a.wq_o, a.sc_o, a.bi_o, N, K, 4, 64, rows=rows)
    check_float(y.float().cpu().numpy()[rows], ref, K, a.max_w, float(xs[1].float().abs().max()), "graph replay")
    del g
    gwb.check_device_error()


def test_gptq_act_order_captured_with_and_without_the_scratch():
    """Act-order GPTQ at M > 8 in a CUDA graph.  A stream that has no dequant scratch yet
    cannot allocate one under capture, so the captured call takes the per-tile kernel; once an
    eager call on the stream has made the scratch, a captured call dequantizes into it and
    runs the dense fp16 GEMM.  Both replays match the oracle."""
    K, N, gs, M = 512, 264, 128, 40
    g = Gptq(K, N, gs, True, seed=21)
    x = synth.activations(M, K, seed=22, dtype=torch.float16)
    ref = oracle.gptq_qmm(synth.bits16(x), *g.h, K, N, gs)
    max_w = float(np.abs(oracle.gptq_dequant_f16(*g.h, K, N, gs).view(np.float16).astype(np.float32)).max())
    xd = x.to(DEV)
    st = torch.cuda.Stream()
    y = torch.empty((M, N), dtype=torch.float16, device=DEV)
    with torch.cuda.stream(st):
        for eager_first in (False, True):
            if eager_first:
                gwb.gptq_qmm(xd, *g.d, gs, y=y)           # the stream's scratch exists from here on
                st.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=st):
                gwb.gptq_qmm(xd, *g.d, gs, y=y)
            y.fill_(float("nan"))
            graph.replay()
            st.synchronize()
            check_float(y.float().cpu().numpy(), ref, K, max_w, float(x.float().abs().max()),
                        f"act order captured, scratch={'yes' if eager_first else 'no'}")
            del graph
    gwb.check_device_error()


# --------------------------------------------------------------------------- full sizes
def test_full_single_affine_linear_512():
    a = Affine(512, 512, 4, 64)
    a.check_pack()
    a.check_qmm(1, label="512x512 M=1")


DECODE_SHAPES = [(2048, 2048, 4), (512, 2048, 4), (8192, 2048, 4), (2048, 8192, 4), (128256, 2048, 4),
                 (8192, 2048, 2), (8192, 2048, 8)]


@pytest.mark.parametrize("N,K,bits", DECODE_SHAPES)
def test_full_decode_gemv(N, K, bits):
    a = Affine(N, K, bits, 64)
    a.check_pack()
    a.check_qmm(1, label=f"decode {N}x{K} b{bits}")


PREFILL_SHAPES = [(4096, 4096), (1024, 4096), (14336, 4096), (4096, 14336)]


PREFILL_M = (16, 128, 512, 2048)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("N,K", PREFILL_SHAPES)
def test_full_prefill_gemm_gs64(N, K, bits):
    a = Affine(N, K, bits, 64)
    a.check_pack()
    for M in PREFILL_M:
        a.check_qmm(M, outlier_frac=0.01, label=f"prefill {N}x{K} b{bits} M={M}")


@pytest.mark.parametrize("bits,gs", [(8, 32), (8, 128), (4, 32), (4, 128)])
def test_full_prefill_other_group_sizes(bits, gs):
    a = Affine(4096, 4096, bits, gs)
    a.check_pack()
    for M in (16, 512):
        a.check_qmm(M, outlier_frac=0.01, label=f"prefill 4096x4096 b{bits} gs{gs} M={M}")
    b = Affine(14336, 4096, bits, gs, seed=1)
    for M in (128, 512):
        b.check_qmm(M, outlier_frac=0.01, label=f"prefill 14336x4096 b{bits} gs{gs} M={M}")


@pytest.mark.parametrize("permuted", [False, True])
def test_full_gptq(permuted):
    g = Gptq(4096, 11008, 128, permuted)
    for M in (1, 32, 1024):
        g.check_qmm(M)


def test_full_awq():
    a = Awq(4096, 11008, 128)
    for M in (1, 32, 1024):
        a.check_qmm(M)


@pytest.mark.parametrize("bits", [4, 8])
def test_full_decode_mlp_fused(bits):
    # Llama-3-8B MLP at decode: gate/up 14336 x 4096 and down 4096 x 14336 with the residual
    for M in (1, 4):
        _gate_up_case(14336, 4096, bits, 64, M, seed=40 + M)
        _silu_case(4096, 14336, bits, 64, M, seed=50 + M, resid=True)


@pytest.mark.parametrize("N,K", [(4096, 4096), (14336, 4096), (4096, 14336)])
def test_full_w8a8(N, K):
    w = W8A8(N, K)
    for M in (1, 64, 512, 4096):
        w.check(M)


@pytest.mark.parametrize("N,K", [(4096, 4096), (14336, 4096), (4096, 14336)])
def test_full_w4a8(N, K):
    w = W4A8(N, K)
    for M in (8, 64, 512, 4096):
        w.check(M)


def test_no_device_wait_gave_up():
    gwb.check_device_error()

"""GPU check of gwb_qmm_affine_noalloc, the prefill GEMM entry point that
allocates nothing.

It exists for callers that cannot allocate device memory: code running under
an allocator that already owns all of the GPU's memory (a framework's caching
pool, a serving runtime that reserves memory up front), and code that must not
call cudaMalloc / cudaFree at all, since both may synchronize the whole device.
The entry point keeps the GEMM's stream-K scratch (partial tiles and their
flags) in a fixed device array of the library instead.

The test calls it through the C ABI and compares it with gwb_qmm_affine (whose
scratch is the library-allocated workspace) on the same inputs, within the
float tolerance of the parity tests, twice in a row: the second call finds the
first call's data still in the shared array.  Both calls are also compared
with the CPU oracle on rows sampled from every 128-token block.  The shapes
split every output tile between several CTA pairs, so the scratch is really
used.  This file is named to be collected last.
"""
import numpy as np
import pytest
import torch

import gwb_synth as synth
import oracle
from tol import check_float

gwb = pytest.importorskip("group_wise_bit_b200")
pytestmark = pytest.mark.gpu

DEV = "cuda"


def _max_w(sc, bi, bits):
    b = bi.float()
    return float(torch.maximum(b.abs(), (b + ((1 << bits) - 1) * sc.float()).abs()).max())


def _oracle_rows(M):
    rng = np.random.default_rng(M)
    picks = [b + int(rng.integers(0, min(128, M - b))) for b in range(0, M, 128)]
    return np.unique(np.concatenate([[0, M - 1], picks]))


@pytest.mark.parametrize("N,K,bits,M", [(2048, 2048, 4, 512), (1024, 4096, 8, 300)])
def test_qmm_affine_noalloc_matches_qmm_affine(N, K, bits, M):
    wh = synth.weights(N, K, seed=21)
    wq, sc, bi = gwb.qpack_affine(wh.to(DEV), bits, 64)
    xh = synth.activations(M, K, seed=22, outlier_frac=0.01)
    x = xh.to(DEV)
    y_ref = gwb.qmm_affine(x, wq, sc, bi, bits, 64)
    torch.cuda.synchronize()
    ref = y_ref.float().cpu().numpy()
    max_w, max_x = _max_w(sc, bi, bits), float(x.float().abs().max())
    # the CPU oracle on the same packed weights (its packing is bit-identical to the library's)
    wq_o, sc_o, bi_o, _ = oracle.qpack_affine(wh.numpy(), bits, 64)
    rows = _oracle_rows(M)
    y_o = oracle.qmm_affine(synth.bits16(xh), wq_o, sc_o, bi_o, N, K, bits, 64, rows=rows)
    for call in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)   # the caller's output
        gwb.qmm_affine_noalloc(x, wq, sc, bi, bits, 64, y=y)
        torch.cuda.synchronize()
        yc = y.float().cpu().numpy()
        check_float(yc, ref, K, max_w, max_x, f"noalloc {N}x{K} b{bits} M={M} call {call}")
        check_float(yc[rows], y_o, K, max_w, max_x, f"noalloc vs oracle {N}x{K} b{bits} M={M} call {call}")
    gwb.check_device_error()


def test_qmm_affine_noalloc_rejects_small_m():
    w = synth.weights(256, 256, seed=23).to(DEV)
    wq, sc, bi = gwb.qpack_affine(w, 4, 64)
    x = torch.zeros(64, 256, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(gwb.GwbError, match="SHAPE"):
        gwb.qmm_affine_noalloc(x, wq, sc, bi, 4, 64)

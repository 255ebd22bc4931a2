"""GPU check of the bounded-wait failure path: a device wait that runs out
makes the kernel stop, free what it holds and return, the host reads
GWB_ERR_TIMEOUT, and the context stays usable (metrale_gpu_runtime/mlx_int8.rs,
MlxInt8Weight::load: failures come back as errors, not crashes).

No GPU is faulted: the prefill GEMM's stream-K handshake is told to wait for a
partial tile that no CTA publishes (a flag that nothing sets), with the wait
limit lowered to about 10 ms, so the head CTAs' waits give up.  The next
ordinary call on the same stream must then be correct against the oracle.
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
SHORT_WAIT = 20_000_000   # SM clock cycles: about 10 ms


def test_stream_k_wait_runs_out_and_the_context_recovers():
    N, K, M, bits, gs = 2048, 2048, 512, 4, 64    # 8 x 2 tiles of 256 x 256, 32 K steps, 74 pairs: stream-K
    w = synth.weights(N, K, seed=31)
    wq_o, sc_o, bi_o, _ = oracle.qpack_affine(w.numpy(), bits, gs)
    wq, sc, bi = gwb.qpack_affine(w.to(DEV), bits, gs)
    x = synth.activations(M, K, seed=32, outlier_frac=0.01)
    xd = x.to(DEV)
    gwb.qmm_affine(xd, wq, sc, bi, bits, gs)          # allocates the stream's workspace (outside the test's window)
    gwb.check_device_error()
    gwb.debug_set_wait_cycles(SHORT_WAIT)
    try:
        gwb.debug_inject_stream_k_stall(True)
        gwb.qmm_affine(xd, wq, sc, bi, bits, gs)      # its head CTAs wait for partials nobody publishes
        with pytest.raises(gwb.GwbError, match="TIMEOUT"):
            gwb.check_device_error()
    finally:
        gwb.debug_inject_stream_k_stall(False)
        gwb.debug_set_wait_cycles(0)
    gwb.check_device_error()                          # the flag was cleared by the read above
    y = gwb.qmm_affine(xd, wq, sc, bi, bits, gs)
    gwb.check_device_error()
    rows = np.array([0, 100, 255, 256, 300, 511], dtype=np.int64)
    y_ref = oracle.qmm_affine(synth.bits16(x), wq_o, sc_o, bi_o, N, K, bits, gs, rows=rows)
    s = oracle.bf16_array_to_f64(sc_o)
    b = oracle.bf16_array_to_f64(bi_o)
    max_w = float(np.max(np.maximum(np.abs(b), np.abs(b + 15 * s))))
    check_float(y.float().cpu().numpy()[rows], y_ref, K, max_w, float(x.float().abs().max()), "after the timeout")


def test_wait_limit_round_trip():
    gwb.debug_set_wait_cycles(SHORT_WAIT)
    gwb.debug_set_wait_cycles(0)
    gwb.check_device_error()

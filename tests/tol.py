"""Float-output tolerance of the parity tests.

For every bf16 / fp16 result y of a matmul, compared against the fp64 oracle
y_ref computed from the same packed inputs:
    max |y - y_ref|                  <= 2e-2 * sqrt(K) * max|w| * max|x|
    ||y - y_ref||_F / ||y_ref||_F    <= 5e-3
where max|w| is the largest dequantized weight magnitude and max|x| the largest
activation magnitude.  The expected error is far below both: the output is
rounded once to bf16 (relative 2^-9) and, on the tensor-core path, every
dequantized weight is rounded once to bf16 (relative 2^-9, random sign), so the
relative Frobenius error sits near 2e-3 at most.
"""
import numpy as np

MAX_ABS_COEF = 2e-2
REL_FRO = 5e-3


def check_float(y, y_ref, K, max_w, max_x, label=""):
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    assert y.shape == y_ref.shape, (label, y.shape, y_ref.shape)
    assert np.all(np.isfinite(y)), f"{label}: non-finite output"
    err = np.abs(y - y_ref)
    bound = MAX_ABS_COEF * np.sqrt(K) * max_w * max_x
    assert err.max() <= bound, f"{label}: max abs err {err.max():.3e} > {bound:.3e}"
    denom = np.linalg.norm(y_ref)
    rel = np.linalg.norm(y - y_ref) / denom if denom > 0 else np.linalg.norm(y - y_ref)
    assert rel <= REL_FRO, f"{label}: rel Frobenius err {rel:.3e} > {REL_FRO}"
    return float(err.max()), float(rel)

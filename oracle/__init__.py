"""CPU oracle for group-wise low-bit linear layers (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline / reference arm may import this package.  The library's product path
(``group_wise_bit_b200``) never imports it and shares no code with it.

The arithmetic lives in ``gwb_oracle.c`` (plain C, fp64 loops, fp32 where the
method defines fp32); this module only marshals numpy arrays into it.  The
shared object is built with gcc on first use (or by ``build()``), with
``-ffp-contract=off`` so that no fused multiply-add is formed.

bf16 and fp16 values travel as their raw 16-bit patterns in ``np.uint16``
arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gwb_oracle.c")
_LIB = os.path.join(_HERE, "_gwb_oracle.so")
_lib = None

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_INT = ctypes.c_int


def build(force: bool = False) -> str:
    """Compile gwb_oracle.c into _gwb_oracle.so (plain gcc, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        sig = {
            "orc_bf16_to_f64": (ctypes.c_double, [ctypes.c_uint16]),
            "orc_f32_to_bf16": (ctypes.c_uint16, [ctypes.c_float]),
            "orc_f16_to_f64": (ctypes.c_double, [ctypes.c_uint16]),
            "orc_f64_to_f16": (ctypes.c_uint16, [ctypes.c_double]),
            "orc_unpack_affine": (None, [_P, _I64, _I64, _INT, _P]),
            "orc_pack_affine": (None, [_P, _I64, _I64, _INT, _P]),
            "orc_qpack_affine": (None, [_P, _I64, _I64, _INT, _INT, _P, _P, _P, _P]),
            "orc_dequant_affine_f64": (None, [_P, _P, _P, _I64, _I64, _INT, _INT, _P]),
            "orc_dequant_affine_bf16": (None, [_P, _P, _P, _I64, _I64, _INT, _INT, _P]),
            "orc_qmm_affine": (None, [_P, _I64, _P, _I64, _P, _P, _P, _I64, _I64, _INT, _INT, _P]),
            "orc_gptq_dequant_f64": (None, [_P, _P, _P, _P, _I64, _I64, _INT, _P]),
            "orc_gptq_dequant_f16": (None, [_P, _P, _P, _P, _I64, _I64, _INT, _P]),
            "orc_gptq_qmm": (None, [_P, _I64, _P, _I64, _P, _P, _P, _P, _I64, _I64, _INT, _P]),
            "orc_awq_dequant_f64": (None, [_P, _P, _P, _I64, _I64, _INT, _P]),
            "orc_awq_dequant_f16": (None, [_P, _P, _P, _I64, _I64, _INT, _P]),
            "orc_awq_qmm": (None, [_P, _I64, _P, _I64, _P, _P, _P, _I64, _I64, _INT, _P]),
            "orc_quant_per_token_i8": (None, [_P, _I64, _I64, _P, _P]),
            "orc_qpack_sym_i4": (None, [_P, _I64, _I64, _P, _P, _P]),
            "orc_gemm_i8i4": (_INT, [_P, _P, _I64, _P, _I64, _P, _P, _I64, _I64, _P, _P]),
            "orc_qpack_sym_i8": (None, [_P, _I64, _I64, _P, _P]),
            "orc_silu_mul": (None, [_P, _P, _I64, _P]),
            "orc_qmv_silu_gate": (None, [_P, _P, _I64, _P, _I64, _P, _P, _P, _I64, _I64, _INT, _INT, _P, _P]),
            "orc_gemm_i8i8": (_INT, [_P, _P, _I64, _P, _I64, _P, _P, _I64, _I64, _P, _P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _c(a, dtype):
    """Contiguous array of the given dtype (no silent dtype change allowed)."""
    a = np.asarray(a)
    if a.dtype != np.dtype(dtype):
        raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
    return np.ascontiguousarray(a)


def _p(a):
    return None if a is None else a.ctypes.data_as(_P)


def _rows(rows, M):
    if rows is None:
        return None, M
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    if r.size and (r.min() < 0 or r.max() >= M):
        raise IndexError("row index out of range")
    return r, int(r.size)


# ----------------------------------------------------------------- scalars
def bf16_to_f64(h: int) -> float:
    return _load().orc_bf16_to_f64(int(h))


def f32_to_bf16(f: float) -> int:
    return _load().orc_f32_to_bf16(float(f))


def f16_to_f64(h: int) -> float:
    return _load().orc_f16_to_f64(int(h))


def f64_to_f16(v: float) -> int:
    return _load().orc_f64_to_f16(float(v))


def bf16_array_to_f64(a) -> np.ndarray:
    """Vector form of bf16_to_f64 (a bf16 is the top half of an fp32)."""
    a = np.asarray(a, dtype=np.uint16)
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ----------------------------------------------------------------- MLX affine
def unpack_affine(wq, N, K, bits):
    wq = _c(wq, np.uint32)
    codes = np.empty((N, K), np.int32)
    _load().orc_unpack_affine(_p(wq), N, K, bits, _p(codes))
    return codes


def pack_affine(codes, bits):
    codes = _c(codes, np.int32)
    N, K = codes.shape
    wq = np.empty((N, K * bits // 32), np.uint32)
    _load().orc_pack_affine(_p(codes), N, K, bits, _p(wq))
    return wq


def qpack_affine(w, bits, gs):
    """Returns (wq uint32 [N, K*bits/32], scales bf16 [N, K/gs], biases bf16, codes int32 [N, K])."""
    w = _c(w, np.float32)
    N, K = w.shape
    wq = np.empty((N, K * bits // 32), np.uint32)
    sc = np.empty((N, K // gs), np.uint16)
    bi = np.empty((N, K // gs), np.uint16)
    codes = np.empty((N, K), np.int32)
    _load().orc_qpack_affine(_p(w), N, K, bits, gs, _p(wq), _p(sc), _p(bi), _p(codes))
    return wq, sc, bi, codes


def dequant_affine_f64(wq, scales, biases, N, K, bits, gs):
    wq, scales, biases = _c(wq, np.uint32), _c(scales, np.uint16), _c(biases, np.uint16)
    out = np.empty((N, K), np.float64)
    _load().orc_dequant_affine_f64(_p(wq), _p(scales), _p(biases), N, K, bits, gs, _p(out))
    return out


def dequant_affine_bf16(wq, scales, biases, N, K, bits, gs):
    wq, scales, biases = _c(wq, np.uint32), _c(scales, np.uint16), _c(biases, np.uint16)
    out = np.empty((N, K), np.uint16)
    _load().orc_dequant_affine_bf16(_p(wq), _p(scales), _p(biases), N, K, bits, gs, _p(out))
    return out


def qmm_affine(x_bf16, wq, scales, biases, N, K, bits, gs, rows=None):
    """fp64 y[len(rows) or M, N] = x[rows] . W^T."""
    x = _c(x_bf16, np.uint16)
    M = x.shape[0]
    r, nr = _rows(rows, M)
    wq, scales, biases = _c(wq, np.uint32), _c(scales, np.uint16), _c(biases, np.uint16)
    y = np.empty((nr, N), np.float64)
    _load().orc_qmm_affine(_p(x), M, _p(r), nr, _p(wq), _p(scales), _p(biases), N, K, bits, gs, _p(y))
    return y


# ----------------------------------------------------------------- GPTQ
def gptq_dequant_f64(qweight, scales, qzeros, g_idx, K, N, gs):
    qw, sc, qz = _c(qweight, np.int32), _c(scales, np.uint16), _c(qzeros, np.int32)
    gi = None if g_idx is None else _c(g_idx, np.int32)
    out = np.empty((N, K), np.float64)
    _load().orc_gptq_dequant_f64(_p(qw), _p(sc), _p(qz), _p(gi), K, N, gs, _p(out))
    return out


def gptq_dequant_f16(qweight, scales, qzeros, g_idx, K, N, gs):
    qw, sc, qz = _c(qweight, np.int32), _c(scales, np.uint16), _c(qzeros, np.int32)
    gi = None if g_idx is None else _c(g_idx, np.int32)
    out = np.empty((N, K), np.uint16)
    _load().orc_gptq_dequant_f16(_p(qw), _p(sc), _p(qz), _p(gi), K, N, gs, _p(out))
    return out


def gptq_qmm(x_f16, qweight, scales, qzeros, g_idx, K, N, gs, rows=None):
    x = _c(x_f16, np.uint16)
    M = x.shape[0]
    r, nr = _rows(rows, M)
    qw, sc, qz = _c(qweight, np.int32), _c(scales, np.uint16), _c(qzeros, np.int32)
    gi = None if g_idx is None else _c(g_idx, np.int32)
    y = np.empty((nr, N), np.float64)
    _load().orc_gptq_qmm(_p(x), M, _p(r), nr, _p(qw), _p(sc), _p(qz), _p(gi), K, N, gs, _p(y))
    return y


# ----------------------------------------------------------------- AWQ
def awq_dequant_f64(qweight, scales, qzeros, K, N, gs):
    qw, sc, qz = _c(qweight, np.int32), _c(scales, np.uint16), _c(qzeros, np.int32)
    out = np.empty((N, K), np.float64)
    _load().orc_awq_dequant_f64(_p(qw), _p(sc), _p(qz), K, N, gs, _p(out))
    return out


def awq_dequant_f16(qweight, scales, qzeros, K, N, gs):
    qw, sc, qz = _c(qweight, np.int32), _c(scales, np.uint16), _c(qzeros, np.int32)
    out = np.empty((N, K), np.uint16)
    _load().orc_awq_dequant_f16(_p(qw), _p(sc), _p(qz), K, N, gs, _p(out))
    return out


def awq_qmm(x_f16, qweight, scales, qzeros, K, N, gs, rows=None):
    x = _c(x_f16, np.uint16)
    M = x.shape[0]
    r, nr = _rows(rows, M)
    qw, sc, qz = _c(qweight, np.int32), _c(scales, np.uint16), _c(qzeros, np.int32)
    y = np.empty((nr, N), np.float64)
    _load().orc_awq_qmm(_p(x), M, _p(r), nr, _p(qw), _p(sc), _p(qz), K, N, gs, _p(y))
    return y


# ----------------------------------------------------------------- W4A8
def quant_per_token_i8(x_bf16):
    x = _c(x_bf16, np.uint16)
    M, K = x.shape
    qx = np.empty((M, K), np.int8)
    sx = np.empty((M,), np.float32)
    _load().orc_quant_per_token_i8(_p(x), M, K, _p(qx), _p(sx))
    return qx, sx


def qpack_sym_i4(w):
    """Returns (wq uint32 [N, K/8], sw float32 [N], codes int32 [N, K])."""
    w = _c(w, np.float32)
    N, K = w.shape
    wq = np.empty((N, K // 8), np.uint32)
    sw = np.empty((N,), np.float32)
    codes = np.empty((N, K), np.int32)
    _load().orc_qpack_sym_i4(_p(w), N, K, _p(wq), _p(sw), _p(codes))
    return wq, sw, codes


def gemm_i8i4(qx, sx, wq, sw, N, K, rows=None):
    """Returns (acc int64 [R, N], y fp64 [R, N], overflow flag)."""
    qx, sx = _c(qx, np.int8), _c(sx, np.float32)
    wq, sw = _c(wq, np.uint32), _c(sw, np.float32)
    M = qx.shape[0]
    r, nr = _rows(rows, M)
    acc = np.empty((nr, N), np.int64)
    y = np.empty((nr, N), np.float64)
    ovf = _load().orc_gemm_i8i4(_p(qx), _p(sx), M, _p(r), nr, _p(wq), _p(sw), N, K, _p(acc), _p(y))
    return acc, y, bool(ovf)


def w4a8_fused(x_bf16, wq, sw, N, K, rows=None):
    """The W4A8 product with the activation quantization inside it: by definition the
    per-token quantizer followed by the int8 x int4 product.  Returns (acc, y, overflow)."""
    qx, sx = quant_per_token_i8(x_bf16)
    return gemm_i8i4(qx, sx, wq, sw, N, K, rows=rows)


# ----------------------------------------------------------------- W8A8
def qpack_sym_i8(w):
    """Returns (wq int8 [N, K], sw float32 [N])."""
    w = _c(w, np.float32)
    N, K = w.shape
    wq = np.empty((N, K), np.int8)
    sw = np.empty((N,), np.float32)
    _load().orc_qpack_sym_i8(_p(w), N, K, _p(wq), _p(sw))
    return wq, sw


def gemm_i8i8(qx, sx, wq, sw, N, K, rows=None):
    """Returns (acc int64 [R, N], y fp64 [R, N], overflow flag)."""
    qx, sx = _c(qx, np.int8), _c(sx, np.float32)
    wq, sw = _c(wq, np.int8), _c(sw, np.float32)
    M = qx.shape[0]
    r, nr = _rows(rows, M)
    acc = np.empty((nr, N), np.int64)
    y = np.empty((nr, N), np.float64)
    ovf = _load().orc_gemm_i8i8(_p(qx), _p(sx), M, _p(r), nr, _p(wq), _p(sw), N, K, _p(acc), _p(y))
    return acc, y, bool(ovf)


# ----------------------------------------------------------------- fused decode products
def silu_mul(gate_bf16, up_bf16):
    """fp64 silu(gate) * up, elementwise, for bf16 bit patterns of equal shape."""
    g, u = _c(gate_bf16, np.uint16), _c(up_bf16, np.uint16)
    h = np.empty(g.shape, np.float64)
    _load().orc_silu_mul(_p(g), _p(u), g.size, _p(h))
    return h


def qmv_silu_gate(gate_bf16, up_bf16, wq, scales, biases, N, K, bits, gs, resid_bf16=None, rows=None):
    """fp64 y[len(rows) or M, N] = resid + (silu(gate) * up) . W^T (resid optional)."""
    g, u = _c(gate_bf16, np.uint16), _c(up_bf16, np.uint16)
    M = g.shape[0]
    r, nr = _rows(rows, M)
    wq, scales, biases = _c(wq, np.uint32), _c(scales, np.uint16), _c(biases, np.uint16)
    res = None if resid_bf16 is None else _c(resid_bf16, np.uint16)
    y = np.empty((nr, N), np.float64)
    _load().orc_qmv_silu_gate(_p(g), _p(u), M, _p(r), nr, _p(wq), _p(scales), _p(biases), N, K, bits, gs,
                              _p(res), _p(y))
    return y


def qmv_gate_up(x_bf16, gate_w, up_w, N, K, bits, gs, rows=None):
    """(gate_y, up_y) = (x . W_gate^T, x . W_up^T) in fp64; gate_w, up_w = (wq, scales, biases)."""
    return (qmm_affine(x_bf16, *gate_w, N, K, bits, gs, rows=rows),
            qmm_affine(x_bf16, *up_w, N, K, bits, gs, rows=rows))

"""Python binding of the group-wise low-bit linear-layer library (libgwb.so).

Argument marshalling only: every function below checks dtypes, shapes,
devices and contiguity of torch CUDA tensors, allocates outputs that were not
given, and calls the C entry point of the same name (see include/gwb.h) on
torch's current CUDA stream.  All computation happens in the library's CUDA
kernels; there is no CPU fallback.  Errors from the library raise GwbError.

Packed uint32 words may be held in torch.int32 or torch.uint32 tensors (the
bits are what matters); bf16 / fp16 tensors are passed as such.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgwb.so")

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_INT = ctypes.c_int

# name -> argument types (all return int gwb_status)
SIGNATURES = {
    "gwb_qpack_affine": [_P, _I64, _I64, _INT, _INT, _P, _P, _P, _P],
    "gwb_dequant_affine": [_P, _P, _P, _I64, _I64, _INT, _INT, _P, _P],
    "gwb_qmm_affine": [_P, _I64, _P, _P, _P, _I64, _I64, _INT, _INT, _P, _P],
    "gwb_qmm_affine_noalloc": [_P, _I64, _P, _P, _P, _I64, _I64, _INT, _INT, _P, _P],
    "gwb_gptq_dequant": [_P, _P, _P, _P, _I64, _I64, _INT, _P, _P],
    "gwb_gptq_qmm": [_P, _I64, _P, _P, _P, _P, _I64, _I64, _INT, _P, _P],
    "gwb_gemv_gate_up": [_P, _I64, _P, _P, _P, _P, _P, _P, _I64, _I64, _INT, _INT, _P, _P, _P],
    "gwb_gemv_silu_gate": [_P, _P, _I64, _P, _P, _P, _I64, _I64, _INT, _INT, _P, _P],
    "gwb_gemv_silu_gate_resid": [_P, _P, _I64, _P, _P, _P, _I64, _I64, _INT, _INT, _P, _P, _P],
    "gwb_awq_dequant": [_P, _P, _P, _I64, _I64, _INT, _P, _P],
    "gwb_awq_qmm": [_P, _I64, _P, _P, _P, _I64, _I64, _INT, _P, _P],
    "gwb_quant_per_token_i8": [_P, _I64, _I64, _P, _P, _P],
    "gwb_qpack_sym_i4": [_P, _I64, _I64, _P, _P, _P],
    "gwb_gemm_i8i4": [_P, _P, _I64, _P, _P, _I64, _I64, _P, _P, _P],
    "gwb_gemv_w4a8": [_P, _I64, _P, _P, _I64, _I64, _P, _P],
    "gwb_qpack_sym_i8": [_P, _I64, _I64, _P, _P, _P],
    "gwb_gemm_i8i8": [_P, _P, _I64, _P, _P, _I64, _I64, _P, _P, _P],
    "gwb_check_device_error": [_P],
    "gwb_debug_set_wait_cycles": [ctypes.c_ulonglong],
    "gwb_debug_inject_stream_k_stall": [_INT],
}

STATUS = {0: "OK", 1: "INVALID_ARG", 2: "SHAPE", 3: "UNSUPPORTED", 4: "ALIGN", 5: "CUDA", 6: "TIMEOUT"}


class GwbError(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__(f"{fn}: {STATUS.get(status, status)}: {msg}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Loads libgwb.so (built in-tree by `python -m group_wise_bit_b200.build`)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m group_wise_bit_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, args in SIGNATURES.items():
            fn = getattr(l, name)
            fn.argtypes = args
            fn.restype = _INT
        l.gwb_last_error.restype = ctypes.c_char_p
        l.gwb_last_error.argtypes = []
        l.gwb_version.restype = ctypes.c_char_p
        l.gwb_version.argtypes = []
        _lib = l
    return _lib


def version() -> str:
    return lib().gwb_version().decode()


_fns = {}


def _call(name, *args):
    fn = _fns.get(name)
    if fn is None:
        fn = _fns[name] = getattr(lib(), name)
    st = fn(*args)
    if st != 0:
        raise GwbError(name, st, lib().gwb_last_error().decode())


try:   # the raw handle of the current stream, without building a Stream object per call
    _raw_stream = torch._C._cuda_getCurrentRawStream

    def _stream():
        return _raw_stream(torch.cuda.current_device())
except AttributeError:   # pragma: no cover - older torch
    def _stream():
        return torch.cuda.current_stream().cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _dev(t, name, dtypes, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype} not in {dtypes}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and t.shape != shape:
        raise ValueError(f"{name}: shape {tuple(t.shape)} != {tuple(shape)}")
    return t


_WORDS = (torch.int32, torch.uint32)


def _out(t, name, shape, dtype, device, dtypes=None):
    if t is None:
        return torch.empty(shape, dtype=dtype, device=device)
    return _dev(t, name, dtypes or (dtype,), shape)


# ------------------------------------------------------------------ MLX affine
def qpack_affine(w, bits, group_size, wq=None, scales=None, biases=None):
    """w fp32 [N, K] -> (wq int32 [N, K*bits/32], scales bf16 [N, K/gs], biases bf16 [N, K/gs])."""
    _dev(w, "w", (torch.float32,))
    N, K = w.shape
    wq = _out(wq, "wq", (N, K * bits // 32), torch.int32, w.device, _WORDS)
    scales = _out(scales, "scales", (N, K // group_size), torch.bfloat16, w.device)
    biases = _out(biases, "biases", (N, K // group_size), torch.bfloat16, w.device)
    _call("gwb_qpack_affine", _ptr(w), N, K, bits, group_size, _ptr(wq), _ptr(scales), _ptr(biases), _stream())
    return wq, scales, biases


def dequant_affine(wq, scales, biases, K, bits, group_size, out=None):
    """-> bf16 [N, K] with w = bf16(fp32(code*scale + bias))."""
    _dev(wq, "wq", _WORDS)
    N = wq.shape[0]
    _dev(wq, "wq", _WORDS, (N, K * bits // 32))
    _dev(scales, "scales", (torch.bfloat16,), (N, K // group_size))
    _dev(biases, "biases", (torch.bfloat16,), (N, K // group_size))
    out = _out(out, "out", (N, K), torch.bfloat16, wq.device)
    _call("gwb_dequant_affine", _ptr(wq), _ptr(scales), _ptr(biases), N, K, bits, group_size, _ptr(out), _stream())
    return out


def _affine_check(wq, scales, biases, bits, group_size):
    """(N, K) of a weight in the MLX affine layout, its three tensors checked."""
    _dev(wq, "wq", _WORDS)
    N, K = wq.shape[0], wq.shape[1] * 32 // bits
    _dev(scales, "scales", (torch.bfloat16,), (N, K // group_size))
    _dev(biases, "biases", (torch.bfloat16,), (N, K // group_size))
    return N, K


def qmm_affine(x, wq, scales, biases, bits, group_size, y=None):
    """y bf16 [M, N] = x bf16 [M, K] . W^T with W in the MLX affine layout."""
    _dev(x, "x", (torch.bfloat16,))
    M, K = x.shape
    N = wq.shape[0]
    _dev(wq, "wq", _WORDS, (N, K * bits // 32))
    _dev(scales, "scales", (torch.bfloat16,), (N, K // group_size))
    _dev(biases, "biases", (torch.bfloat16,), (N, K // group_size))
    y = _out(y, "y", (M, N), torch.bfloat16, x.device)
    _call("gwb_qmm_affine", _ptr(x), M, _ptr(wq), _ptr(scales), _ptr(biases), N, K, bits, group_size, _ptr(y),
          _stream())
    return y


def qmm_affine_noalloc(x, wq, scales, biases, bits, group_size, y=None):
    """As qmm_affine for M > 128, with the GEMM's scratch in the library's fixed
    device array instead of device memory it allocates (see gwb.h)."""
    _dev(x, "x", (torch.bfloat16,))
    M, K = x.shape
    N = wq.shape[0]
    _dev(wq, "wq", _WORDS, (N, K * bits // 32))
    _dev(scales, "scales", (torch.bfloat16,), (N, K // group_size))
    _dev(biases, "biases", (torch.bfloat16,), (N, K // group_size))
    y = _out(y, "y", (M, N), torch.bfloat16, x.device)
    _call("gwb_qmm_affine_noalloc", _ptr(x), M, _ptr(wq), _ptr(scales), _ptr(biases), N, K, bits, group_size,
          _ptr(y), _stream())
    return y


# ------------------------------------------------------------------ GPTQ
def _gptq_check(qweight, scales, qzeros, g_idx, group_size):
    _dev(qweight, "qweight", _WORDS)
    K8, N = qweight.shape
    K = K8 * 8
    _dev(scales, "scales", (torch.float16,), (K // group_size, N))
    _dev(qzeros, "qzeros", _WORDS, (K // group_size, N // 8))
    if g_idx is not None:
        _dev(g_idx, "g_idx", (torch.int32,), (K,))
    return K, N


def gptq_dequant(qweight, scales, qzeros, g_idx, group_size, out=None):
    """-> fp16 [N, K] (out-features major)."""
    K, N = _gptq_check(qweight, scales, qzeros, g_idx, group_size)
    out = _out(out, "out", (N, K), torch.float16, qweight.device)
    _call("gwb_gptq_dequant", _ptr(qweight), _ptr(scales), _ptr(qzeros), _ptr(g_idx), K, N, group_size, _ptr(out),
          _stream())
    return out


def gptq_qmm(x, qweight, scales, qzeros, g_idx, group_size, y=None):
    """y fp16 [M, N] = x fp16 [M, K] . W^T with W in the GPTQ layout."""
    K, N = _gptq_check(qweight, scales, qzeros, g_idx, group_size)
    _dev(x, "x", (torch.float16,))
    M = x.shape[0]
    _dev(x, "x", (torch.float16,), (M, K))
    y = _out(y, "y", (M, N), torch.float16, x.device)
    _call("gwb_gptq_qmm", _ptr(x), M, _ptr(qweight), _ptr(scales), _ptr(qzeros), _ptr(g_idx), K, N, group_size,
          _ptr(y), _stream())
    return y


# ------------------------------------------------------------------ fused decode products
def gemv_gate_up(x, gate_w, up_w, bits, group_size, y_gate=None, y_up=None):
    """(x W_gate^T, x W_up^T) in one launch; gate_w / up_w = (wq, scales, biases) of one shape."""
    wq, sc, bi = gate_w
    wq2, sc2, bi2 = up_w
    N, K = _affine_check(wq, sc, bi, bits, group_size)
    if _affine_check(wq2, sc2, bi2, bits, group_size) != (N, K):
        raise ValueError("gate and up weights differ in shape")
    _dev(x, "x", (torch.bfloat16,), (x.shape[0], K))
    M = x.shape[0]
    y_gate = _out(y_gate, "y_gate", (M, N), torch.bfloat16, x.device)
    y_up = _out(y_up, "y_up", (M, N), torch.bfloat16, x.device)
    _call("gwb_gemv_gate_up", _ptr(x), M, _ptr(wq), _ptr(sc), _ptr(bi), _ptr(wq2), _ptr(sc2), _ptr(bi2), N, K,
          bits, group_size, _ptr(y_gate), _ptr(y_up), _stream())
    return y_gate, y_up


def gemv_silu_gate(gate, up, wq, scales, biases, bits, group_size, x_resid=None, y=None):
    """y = (x_resid +) (silu(gate) * up) W^T; gate, up bf16 [M, K], x_resid bf16 [M, N]."""
    N, K = _affine_check(wq, scales, biases, bits, group_size)
    _dev(gate, "gate", (torch.bfloat16,), (gate.shape[0], K))
    M = gate.shape[0]
    _dev(up, "up", (torch.bfloat16,), (M, K))
    y = _out(y, "y", (M, N), torch.bfloat16, gate.device)
    if x_resid is None:
        _call("gwb_gemv_silu_gate", _ptr(gate), _ptr(up), M, _ptr(wq), _ptr(scales), _ptr(biases), N, K, bits,
              group_size, _ptr(y), _stream())
    else:
        _dev(x_resid, "x_resid", (torch.bfloat16,), (M, N))
        _call("gwb_gemv_silu_gate_resid", _ptr(gate), _ptr(up), M, _ptr(wq), _ptr(scales), _ptr(biases), N, K,
              bits, group_size, _ptr(x_resid), _ptr(y), _stream())
    return y


# ------------------------------------------------------------------ AWQ
def awq_dequant(qweight, scales, qzeros, group_size, out=None):
    """-> fp16 [N, K]: the GPTQ layout with the stored zero used as is (no "+1", no g_idx)."""
    K, N = _gptq_check(qweight, scales, qzeros, None, group_size)
    out = _out(out, "out", (N, K), torch.float16, qweight.device)
    _call("gwb_awq_dequant", _ptr(qweight), _ptr(scales), _ptr(qzeros), K, N, group_size, _ptr(out), _stream())
    return out


def awq_qmm(x, qweight, scales, qzeros, group_size, y=None):
    """y fp16 [M, N] = x fp16 [M, K] . W^T with W as awq_dequant defines it."""
    K, N = _gptq_check(qweight, scales, qzeros, None, group_size)
    _dev(x, "x", (torch.float16,), (x.shape[0], K))
    M = x.shape[0]
    y = _out(y, "y", (M, N), torch.float16, x.device)
    _call("gwb_awq_qmm", _ptr(x), M, _ptr(qweight), _ptr(scales), _ptr(qzeros), K, N, group_size, _ptr(y),
          _stream())
    return y


# ------------------------------------------------------------------ W4A8
def quant_per_token_i8(x, qx=None, sx=None):
    """x bf16 [M, K] -> (qx int8 [M, K], sx fp32 [M])."""
    _dev(x, "x", (torch.bfloat16,))
    M, K = x.shape
    qx = _out(qx, "qx", (M, K), torch.int8, x.device)
    sx = _out(sx, "sx", (M,), torch.float32, x.device)
    _call("gwb_quant_per_token_i8", _ptr(x), M, K, _ptr(qx), _ptr(sx), _stream())
    return qx, sx


def qpack_sym_i4(w, wq=None, sw=None):
    """w fp32 [N, K] -> (wq int32 [N, K/8] of two's-complement nibbles, sw fp32 [N])."""
    _dev(w, "w", (torch.float32,))
    N, K = w.shape
    wq = _out(wq, "wq", (N, K // 8), torch.int32, w.device, _WORDS)
    sw = _out(sw, "sw", (N,), torch.float32, w.device)
    _call("gwb_qpack_sym_i4", _ptr(w), N, K, _ptr(wq), _ptr(sw), _stream())
    return wq, sw


def gemm_i8i4(qx, sx, wq, sw, want_y=True, want_acc=False, y=None, acc=None):
    """-> (y bf16 [M, N] or None, acc int32 [M, N] or None)."""
    _dev(qx, "qx", (torch.int8,))
    M, K = qx.shape
    N = wq.shape[0]
    _dev(sx, "sx", (torch.float32,), (M,))
    _dev(wq, "wq", _WORDS, (N, K // 8))
    _dev(sw, "sw", (torch.float32,), (N,))
    if want_y or y is not None:
        y = _out(y, "y", (M, N), torch.bfloat16, qx.device)
    if want_acc or acc is not None:
        acc = _out(acc, "acc", (M, N), torch.int32, qx.device)
    _call("gwb_gemm_i8i4", _ptr(qx), _ptr(sx), M, _ptr(wq), _ptr(sw), N, K, _ptr(y), _ptr(acc), _stream())
    return y, acc


def gemv_w4a8(x, wq, sw, y=None):
    """y bf16 [M, N] = W4A8 product of x bf16 [M, K] (quantized per token inside the kernel, M <= 8)
    and the int4 weights (wq, sw) of qpack_sym_i4; bit-identical to quant_per_token_i8 + gemm_i8i4."""
    _dev(x, "x", (torch.bfloat16,))
    M, K = x.shape
    N = wq.shape[0]
    _dev(wq, "wq", _WORDS, (N, K // 8))
    _dev(sw, "sw", (torch.float32,), (N,))
    y = _out(y, "y", (M, N), torch.bfloat16, x.device)
    _call("gwb_gemv_w4a8", _ptr(x), M, _ptr(wq), _ptr(sw), N, K, _ptr(y), _stream())
    return y


# ------------------------------------------------------------------ W8A8
def qpack_sym_i8(w, wq=None, sw=None):
    """w fp32 [N, K] -> (wq int8 [N, K], sw fp32 [N])."""
    _dev(w, "w", (torch.float32,))
    N, K = w.shape
    wq = _out(wq, "wq", (N, K), torch.int8, w.device)
    sw = _out(sw, "sw", (N,), torch.float32, w.device)
    _call("gwb_qpack_sym_i8", _ptr(w), N, K, _ptr(wq), _ptr(sw), _stream())
    return wq, sw


def gemm_i8i8(qx, sx, wq, sw, want_y=True, want_acc=False, y=None, acc=None):
    """-> (y bf16 [M, N] or None, acc int32 [M, N] or None)."""
    _dev(qx, "qx", (torch.int8,))
    M, K = qx.shape
    N = wq.shape[0]
    _dev(sx, "sx", (torch.float32,), (M,))
    _dev(wq, "wq", (torch.int8,), (N, K))
    _dev(sw, "sw", (torch.float32,), (N,))
    if want_y or y is not None:
        y = _out(y, "y", (M, N), torch.bfloat16, qx.device)
    if want_acc or acc is not None:
        acc = _out(acc, "acc", (M, N), torch.int32, qx.device)
    _call("gwb_gemm_i8i8", _ptr(qx), _ptr(sx), M, _ptr(wq), _ptr(sw), N, K, _ptr(y), _ptr(acc), _stream())
    return y, acc


def check_device_error():
    """Synchronizes the current stream; raises GwbError(TIMEOUT) if a bounded device wait gave up."""
    _call("gwb_check_device_error", _stream())


def debug_set_wait_cycles(cycles):
    """Failure-path testing: SM clock cycles after which device waits give up on the
    current device (0 restores the default, about 2 s)."""
    _call("gwb_debug_set_wait_cycles", int(cycles))


def debug_inject_stream_k_stall(armed=True):
    """Failure-path testing: the next stream-K launch of the persistent GEMM waits for
    partial tiles that nothing publishes, so its bounded waits run out (see gwb.h);
    armed=False disarms it."""
    _call("gwb_debug_inject_stream_k_stall", 1 if armed else 0)

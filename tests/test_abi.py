"""CPU-side checks of the C ABI: the library builds and loads, exports every
entry point include/gwb.h declares, and rejects bad arguments on the host
before touching the GPU.  Also checks that the Python binding refuses CPU
tensors (there is no CPU fallback)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import group_wise_bit_b200 as gwb
from group_wise_bit_b200 import build as gbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h")]


def declared_symbols():
    names = set()
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(gwb_\w+)\s*\(", text))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    gbuild.build()
    return gwb.lib()


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    for s in ["gwb_qpack_affine", "gwb_dequant_affine", "gwb_qmm_affine", "gwb_gptq_dequant", "gwb_gptq_qmm",
              "gwb_quant_per_token_i8", "gwb_qpack_sym_i4", "gwb_gemm_i8i4", "gwb_last_error"]:
        assert s in syms


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.check_output(["nm", "-D", "--defined-only", gwb.LIB_PATH], text=True)
    exported = set(re.findall(r"\bT (gwb_\w+)", out))
    missing = [s for s in declared_symbols() if s not in exported]
    assert not missing, missing
    for s in declared_symbols():
        assert hasattr(lib, s)
    assert "sm_100a" in gwb.version()


NULL = None
BAD = ctypes.c_void_p(0x1001)  # misaligned; never dereferenced (validation fails first)
OK16 = ctypes.c_void_p(0x1000)


def _st(fn, *args):
    return getattr(gwb.lib(), fn)(*args)


def test_validation_codes(lib):
    # bits / group size / divisibility / negative sizes
    assert _st("gwb_qmm_affine", OK16, 1, OK16, OK16, OK16, 64, 128, 3, 64, OK16, NULL) == 3
    assert _st("gwb_qmm_affine", OK16, 1, OK16, OK16, OK16, 64, 128, 4, 48, OK16, NULL) == 3
    assert "group_size=48" in gwb.lib().gwb_last_error().decode()
    assert _st("gwb_qmm_affine", OK16, 1, OK16, OK16, OK16, 64, 96, 4, 64, OK16, NULL) == 2
    assert "multiple of group_size" in gwb.lib().gwb_last_error().decode()
    assert _st("gwb_qmm_affine", OK16, -1, OK16, OK16, OK16, 64, 128, 4, 64, OK16, NULL) == 1
    assert "negative M" in gwb.lib().gwb_last_error().decode()
    # NULL and misaligned pointers
    assert _st("gwb_qmm_affine", OK16, 1, OK16, OK16, OK16, 64, 128, 4, 64, NULL, NULL) == 1
    assert _st("gwb_qmm_affine", OK16, 1, OK16, OK16, OK16, 64, 128, 4, 64, BAD, NULL) == 4
    assert _st("gwb_qmm_affine", BAD, 1, OK16, OK16, OK16, 64, 128, 4, 64, OK16, NULL) == 4   # x
    assert _st("gwb_qpack_affine", BAD, 8, 64, 4, 64, OK16, OK16, OK16, NULL) == 4
    # empty problems are no-ops that succeed without launching anything
    assert _st("gwb_qmm_affine", NULL, 0, NULL, NULL, NULL, 64, 128, 4, 64, NULL, NULL) == 0
    assert _st("gwb_qpack_affine", NULL, 0, 128, 4, 64, NULL, NULL, NULL, NULL) == 0
    # GPTQ: N % 8
    assert _st("gwb_gptq_dequant", OK16, OK16, OK16, NULL, 256, 12, 128, OK16, NULL) == 2
    assert _st("gwb_gptq_qmm", OK16, 1, OK16, OK16, OK16, NULL, 256, 16, 48, OK16, NULL) == 3
    # W4A8
    assert _st("gwb_gemm_i8i4", OK16, OK16, 4, OK16, OK16, 64, 128, NULL, NULL, NULL) == 1
    assert _st("gwb_gemm_i8i4", OK16, OK16, 4, OK16, OK16, 64, 100, OK16, NULL, NULL) == 2
    assert _st("gwb_gemm_i8i4", OK16, OK16, 4, OK16, OK16, 64, 262144, OK16, NULL, NULL) == 2
    assert _st("gwb_qpack_sym_i4", OK16, 4, 40, OK16, OK16, NULL) == 2
    assert _st("gwb_quant_per_token_i8", OK16, -2, 8, OK16, OK16, NULL) == 1
    assert gwb.lib().gwb_last_error().decode() != ""


def test_validation_codes_of_the_next_step_entry_points(lib):
    """Every case here fails (or is empty) before anything is launched."""
    W = (OK16, OK16, OK16)
    # fused decode products: at most 8 tokens, the affine layout rules, aligned x, outputs present
    assert _st("gwb_gemv_gate_up", OK16, 9, *W, *W, 64, 512, 4, 64, OK16, OK16, NULL) == 2
    assert _st("gwb_gemv_gate_up", OK16, 1, *W, *W, 64, 512, 3, 64, OK16, OK16, NULL) == 3
    assert _st("gwb_gemv_gate_up", OK16, 1, *W, *W, 64, 96, 4, 64, OK16, OK16, NULL) == 2
    assert _st("gwb_gemv_gate_up", OK16, 1, *W, *W, 64, 512, 4, 64, NULL, OK16, NULL) == 1
    assert _st("gwb_gemv_gate_up", BAD, 1, *W, *W, 64, 512, 4, 64, OK16, OK16, NULL) == 4
    assert _st("gwb_gemv_gate_up", NULL, 0, *W, *W, 64, 512, 4, 64, NULL, NULL, NULL) == 0
    assert _st("gwb_gemv_silu_gate", OK16, OK16, 9, *W, 64, 512, 4, 64, OK16, NULL) == 2
    assert _st("gwb_gemv_silu_gate", OK16, BAD, 1, *W, 64, 512, 4, 64, OK16, NULL) == 4
    # K / group_size = 6 is not a multiple of 8: refused by the planner before any launch
    assert _st("gwb_gemv_silu_gate", OK16, OK16, 1, *W, 64, 384, 4, 64, OK16, NULL) == 3
    assert _st("gwb_gemv_silu_gate_resid", OK16, OK16, 1, *W, 64, 512, 4, 64, NULL, OK16, NULL) == 1
    # fused W4A8 at decode
    assert _st("gwb_gemv_w4a8", OK16, 9, OK16, OK16, 64, 512, OK16, NULL) == 2
    assert _st("gwb_gemv_w4a8", OK16, 1, OK16, OK16, 64, 100, OK16, NULL) == 3
    assert _st("gwb_gemv_w4a8", OK16, 1, OK16, OK16, 64, 32768, OK16, NULL) == 3
    assert _st("gwb_gemv_w4a8", BAD, 1, OK16, OK16, 64, 512, OK16, NULL) == 4
    assert _st("gwb_gemv_w4a8", NULL, 0, NULL, NULL, 64, 512, NULL, NULL) == 0
    # W8A8
    assert _st("gwb_qpack_sym_i8", OK16, 4, 40, OK16, OK16, NULL) == 2
    assert _st("gwb_gemm_i8i8", OK16, OK16, 4, OK16, OK16, 64, 72, OK16, NULL, NULL) == 2
    assert _st("gwb_gemm_i8i8", OK16, OK16, 4, OK16, OK16, 64, 262144, OK16, NULL, NULL) == 2
    assert _st("gwb_gemm_i8i8", OK16, OK16, 4, OK16, OK16, 64, 128, NULL, NULL, NULL) == 1
    assert _st("gwb_gemm_i8i8", BAD, OK16, 4, OK16, OK16, 64, 128, OK16, NULL, NULL) == 4
    # the allocation-free prefill GEMM: M > 128 only, aligned operands, even K/gs
    assert _st("gwb_qmm_affine_noalloc", OK16, 64, OK16, OK16, OK16, 64, 128, 4, 64, OK16, NULL) == 2
    assert _st("gwb_qmm_affine_noalloc", BAD, 256, OK16, OK16, OK16, 64, 128, 4, 64, OK16, NULL) == 4
    assert "x is not 16-byte aligned" in gwb.lib().gwb_last_error().decode()
    assert _st("gwb_qmm_affine_noalloc", OK16, 256, OK16, BAD, OK16, 64, 128, 4, 64, OK16, NULL) == 4
    assert _st("gwb_qmm_affine_noalloc", OK16, 256, OK16, OK16, OK16, 64, 192, 4, 64, OK16, NULL) == 3
    assert "even number of groups" in gwb.lib().gwb_last_error().decode()
    # AWQ: the GPTQ shape rules
    assert _st("gwb_awq_dequant", OK16, OK16, OK16, 256, 12, 128, OK16, NULL) == 2
    assert _st("gwb_awq_qmm", OK16, 1, OK16, OK16, OK16, 256, 16, 48, OK16, NULL) == 3


def test_binding_refuses_cpu_tensors(lib):
    x = torch.zeros(1, 64, dtype=torch.bfloat16)
    wq = torch.zeros(8, 8, dtype=torch.int32)
    s = torch.zeros(8, 1, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        gwb.qmm_affine(x, wq, s, s, 4, 64)
    with pytest.raises(ValueError, match="CUDA"):
        gwb.gemv_gate_up(x, (wq, s, s), (wq, s, s), 4, 64)
    with pytest.raises(ValueError, match="CUDA"):
        gwb.gemv_silu_gate(x, x, wq, s, s, 4, 64)
    with pytest.raises(ValueError, match="CUDA"):
        gwb.gemv_w4a8(x, wq, torch.zeros(8))
    with pytest.raises(ValueError, match="CUDA"):
        gwb.gemm_i8i8(torch.zeros(1, 64, dtype=torch.int8), torch.zeros(1), torch.zeros(8, 64, dtype=torch.int8),
                      torch.zeros(8))


def test_oracle_builds_independently():
    import oracle
    path = oracle.build()
    assert os.path.exists(path)
    # the oracle's sources include nothing from the library and vice versa
    src = open(os.path.join(ROOT, "oracle", "gwb_oracle.c")).read()
    assert "gwb.h" not in src and "group_wise_bit_b200" not in src
    for f in os.listdir(os.path.join(ROOT, "group_wise_bit_b200", "csrc")):
        assert "oracle" not in open(os.path.join(ROOT, "group_wise_bit_b200", "csrc", f)).read().lower()

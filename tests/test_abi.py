"""C-ABI checks that need no GPU: the library loads, exports every symbol include/fp8q.h
declares, and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest
import torch

from fp8_fine_grained_fp8q_b200 import build, ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8q.h")

# Codes from the header.
OK, ERR_ARG, ERR_SHAPE, ERR_ALIGN, ERR_CUDA, ERR_UNSUPPORTED = 0, 1, 2, 3, 4, 5
FAKE = 1 << 40            # an aligned address that is never dereferenced (checks fail first)
MISALIGNED = FAKE + 8


@pytest.fixture(scope="module")
def L():
    build.build()
    return ops.lib()


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"FP8Q_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(declared_symbols())
    assert {"fp8q_act_1x128", "fp8q_act_128x1_transposed", "fp8q_weight_128x128",
            "fp8_gemm_blockscaled", "fp8_grouped_gemm_blockscaled", "fp8q_device_status",
            "fp8q_status_string", "fp8_gemm_blockscaled_ue8m0", "fp8q_act_1x128_fmt"} <= names


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), f"{name} declared in fp8q.h but not exported"
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


def test_status_strings(L):
    for code in range(0, 8):
        assert isinstance(ops.status_string(code), str) and ops.status_string(code)
    assert L.fp8q_abi_version() == 1


P = ctypes.c_void_p


def test_act_1x128_host_checks(L):
    s = None
    assert L.fp8q_act_1x128(P(FAKE), -1, 128, P(FAKE), P(FAKE), s) == ERR_ARG
    assert L.fp8q_act_1x128(P(FAKE), 4, 100, P(FAKE), P(FAKE), s) == ERR_SHAPE
    assert L.fp8q_act_1x128(P(FAKE), 0, 128, P(FAKE), P(FAKE), s) == OK      # empty: no launch
    assert L.fp8q_act_1x128(None, 4, 128, P(FAKE), P(FAKE), s) == ERR_ARG
    assert L.fp8q_act_1x128(P(MISALIGNED), 4, 128, P(FAKE), P(FAKE), s) == ERR_ALIGN
    assert L.fp8q_act_1x128(P(FAKE), 4, 128, P(FAKE), P(FAKE + 4), s) == ERR_ALIGN


def test_act_128x1_host_checks(L):
    s = None
    assert L.fp8q_act_128x1_transposed(P(FAKE), 100, 64, P(FAKE), P(FAKE), s) == ERR_SHAPE
    assert L.fp8q_act_128x1_transposed(P(FAKE), 128, 65, P(FAKE), P(FAKE), s) == ERR_SHAPE
    assert L.fp8q_act_128x1_transposed(P(FAKE), 0, 64, P(FAKE), P(FAKE), s) == OK
    assert L.fp8q_act_128x1_transposed(P(FAKE), 128, 64, None, P(FAKE), s) == ERR_ARG
    assert L.fp8q_act_128x1_transposed(P(FAKE), 128, 64, P(MISALIGNED), P(FAKE), s) == ERR_ALIGN


def test_act_dual_host_checks(L):
    s = None
    d = L.fp8q_act_dual
    assert d(P(FAKE), 128, 64, P(FAKE), P(FAKE), P(FAKE), P(FAKE), s) == ERR_SHAPE   # C % 128
    assert d(P(FAKE), 100, 128, P(FAKE), P(FAKE), P(FAKE), P(FAKE), s) == ERR_SHAPE
    assert d(P(FAKE), -128, 128, P(FAKE), P(FAKE), P(FAKE), P(FAKE), s) == ERR_ARG
    assert d(P(FAKE), 0, 128, P(FAKE), P(FAKE), P(FAKE), P(FAKE), s) == OK
    assert d(P(FAKE), 128, 128, P(FAKE), P(FAKE), None, P(FAKE), s) == ERR_ARG
    assert d(P(FAKE), 128, 128, P(FAKE), P(FAKE), P(FAKE), P(MISALIGNED), s) == ERR_ALIGN
    assert d(P(FAKE), 128 * 65536, 128, P(FAKE), P(FAKE), P(FAKE), P(FAKE), s) == ERR_UNSUPPORTED


def test_quant_forward_host_checks(L):
    f = L.fp8q_quant_forward
    a = [P(FAKE)] * 5
    b = [P(FAKE)] * 3
    assert f(P(FAKE), 128, 100, *a[1:], P(FAKE), 128, *b, None, None) == ERR_SHAPE
    assert f(P(FAKE), 128, 128, *a[1:], P(FAKE), 100, *b, None, None) == ERR_SHAPE
    assert f(P(FAKE), -128, 128, *a[1:], P(FAKE), 128, *b, None, None) == ERR_ARG
    assert f(P(FAKE), 128, 128, *a[1:], None, 128, *b, None, None) == ERR_ARG
    assert f(P(FAKE), 128, 128, *a[1:], P(FAKE), 128, P(FAKE), P(FAKE), P(MISALIGNED), None) == ERR_ALIGN
    assert f(P(FAKE), 0, 128, *a[1:], P(FAKE), 0, *b, None, None) == OK


def test_weight_host_checks(L):
    s = None
    assert L.fp8q_weight_128x128(P(FAKE), 100, 128, P(FAKE), P(FAKE), None, s) == ERR_SHAPE
    assert L.fp8q_weight_128x128(P(FAKE), 128, 130, P(FAKE), P(FAKE), None, s) == ERR_SHAPE
    assert L.fp8q_weight_128x128(P(FAKE), 0, 128, P(FAKE), P(FAKE), None, s) == OK
    assert L.fp8q_weight_128x128(P(FAKE), 128, 128, P(FAKE), P(FAKE), P(MISALIGNED), s) == ERR_ALIGN


def test_gemm_host_checks(L):
    s = None
    g = L.fp8_gemm_blockscaled
    args = (P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE))
    assert g(7, *args, 128, 128, 128, None, 0, s) == ERR_ARG            # bad mode
    assert g(4, *args, 128, 128, 128, None, 0, s) == ERR_ARG
    assert g(3, *args, 128, 128, 0, None, 0, s) == OK                    # D += nothing: no launch
    assert g(0, *args, -1, 128, 128, None, 0, s) == ERR_ARG
    assert g(0, *args, 128, 100, 128, None, 0, s) == ERR_SHAPE
    assert g(1, *args, 128, 128, 96, None, 0, s) == ERR_SHAPE
    assert g(2, *args, 0, 128, 128, None, 0, s) == OK                    # empty: no launch
    assert g(0, P(FAKE), P(FAKE), None, P(FAKE), P(FAKE), 128, 128, 128, None, 0, s) == ERR_ARG
    assert g(0, P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(MISALIGNED), 128, 128, 128, None, 0, s) == ERR_ALIGN
    assert g(0, *args, 1 << 31, 128, 128, None, 0, s) == ERR_UNSUPPORTED
    # Stream-K workspace: one 128 x 256 FP32 slot per CTA plus flags; none for a single K group.
    assert L.fp8q_gemm_workspace_size(0, 4096, 2048, 7168) >= 148 * 128 * 256 * 4
    assert L.fp8q_gemm_workspace_size(0, 4096, 2048, 128) == 0


def test_ue8m0_entries_host_checks(L):
    s = None
    g = L.fp8_gemm_blockscaled_ue8m0
    args = (P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE))
    assert g(5, *args, 128, 128, 128, None, 0, s) == ERR_ARG             # bad mode
    assert g(3, *args, 128, 128, 0, None, 0, s) == OK                    # D += nothing
    assert g(0, *args, 128, 100, 128, None, 0, s) == ERR_SHAPE
    assert g(2, *args, 0, 128, 128, None, 0, s) == OK                    # empty
    assert g(0, P(FAKE), None, P(FAKE), P(FAKE), P(FAKE), 128, 128, 128, None, 0, s) == ERR_ARG
    assert g(0, P(FAKE), P(FAKE), P(FAKE), P(MISALIGNED), P(FAKE), 128, 128, 128, None, 0, s) == ERR_ALIGN
    # The scale-format quantisers: an unknown format is an argument error; sizes as before.
    assert L.fp8q_act_1x128_fmt(P(FAKE), 4, 128, P(FAKE), P(FAKE), 2, s) == ERR_ARG
    assert L.fp8q_act_1x128_fmt(P(FAKE), 4, 100, P(FAKE), P(FAKE), 1, s) == ERR_SHAPE
    assert L.fp8q_act_1x128_fmt(P(FAKE), 0, 128, P(FAKE), P(FAKE), 1, s) == OK
    assert L.fp8q_act_128x1_transposed_fmt(P(FAKE), 128, 64, P(FAKE), P(FAKE), -1, s) == ERR_ARG
    assert L.fp8q_act_128x1_transposed_fmt(P(FAKE), 100, 64, P(FAKE), P(FAKE), 1, s) == ERR_SHAPE
    assert L.fp8q_act_dual_fmt(P(FAKE), 128, 128, P(FAKE), P(FAKE), P(FAKE), P(FAKE), 7, s) == ERR_ARG
    assert L.fp8q_act_dual_fmt(P(FAKE), 128, 64, P(FAKE), P(FAKE), P(FAKE), P(FAKE), 1, s) == ERR_SHAPE
    assert L.fp8q_quant_forward_fmt(P(FAKE), 128, 128, P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), 128,
                                    P(FAKE), P(FAKE), None, 9, s) == ERR_ARG
    assert L.fp8q_weight_128x128_fmt(P(FAKE), 128, 128, P(FAKE), P(FAKE), None, 3, s) == ERR_ARG
    assert L.fp8q_weight_128x128_fmt(P(FAKE), 128, 130, P(FAKE), P(FAKE), None, 1, s) == ERR_SHAPE
    with pytest.raises(ValueError):
        ops._fmt("e4m3")


def test_gemm_quant_host_checks(L):
    s = None
    g = L.fp8_gemm_blockscaled_quant
    ab = (P(FAKE), P(FAKE), P(FAKE), P(FAKE))
    ws = (None, 0, s)
    assert g(2, *ab, P(FAKE), P(FAKE), P(FAKE), 128, 256, 128, *ws) == ERR_ARG          # Wgrad: no
    assert g(0, *ab, P(FAKE), None, P(FAKE), 128, 256, 128, *ws) == ERR_ARG              # Dq missing
    assert g(0, *ab, P(FAKE), P(FAKE), P(FAKE), 128, 100, 128, *ws) == ERR_SHAPE
    assert g(0, *ab, P(FAKE), P(FAKE), P(FAKE), 128, 256, 0, *ws) == ERR_UNSUPPORTED     # K = 0
    assert g(0, *ab, P(FAKE), P(FAKE), P(MISALIGNED), 128, 256, 128, *ws) == ERR_ALIGN
    assert g(1, *ab, P(FAKE), P(FAKE), P(FAKE), 0, 256, 128, *ws) == OK                  # no rows


def test_grouped_host_checks(L):
    s = None
    g = L.fp8_grouped_gemm_blockscaled
    a = (P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE))
    assert g(*a, 0, 128, 128, 128, P(FAKE), s) == ERR_ARG               # E < 1
    assert g(*a, 2000, 128, 128, 128, P(FAKE), s) == ERR_UNSUPPORTED    # E > 1024
    assert g(*a, 4, 128, 100, 128, P(FAKE), s) == ERR_SHAPE
    assert g(*a, 4, 0, 128, 128, P(FAKE), s) == OK
    assert g(P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE + 2), 4, 128, 128, 128, P(FAKE), s) == ERR_ALIGN
    assert g(P(FAKE), P(FAKE), P(FAKE), P(FAKE), None, 4, 128, 128, 128, P(FAKE), s) == ERR_ARG


def test_grouped_dgrad_host_checks(L):
    s = None
    g = L.fp8_grouped_gemm_blockscaled_dgrad
    a = (P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE))
    assert g(*a, 0, 128, 128, 128, P(FAKE), s) == ERR_ARG
    assert g(*a, 2000, 128, 128, 128, P(FAKE), s) == ERR_UNSUPPORTED
    assert g(*a, 4, 128, 128, 100, P(FAKE), s) == ERR_SHAPE
    assert g(*a, 4, 0, 128, 128, P(FAKE), s) == OK
    assert g(P(FAKE), P(FAKE), P(FAKE), P(FAKE), None, 4, 128, 128, 128, P(FAKE), s) == ERR_ARG
    assert g(P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE + 2), 4, 128, 128, 128, P(FAKE), s) == ERR_ALIGN


def test_ragged_and_grouped_wgrad_host_checks(L):
    s = None
    q = L.fp8q_act_128x1_transposed_ragged
    assert q(P(FAKE), P(FAKE), 0, 128, 64, P(FAKE), P(FAKE), 256, s) == ERR_ARG          # E < 1
    assert q(P(FAKE), P(FAKE), 2000, 128, 64, P(FAKE), P(FAKE), 256, s) == ERR_UNSUPPORTED
    assert q(P(FAKE), P(FAKE), 4, 128, 65, P(FAKE), P(FAKE), 256, s) == ERR_SHAPE
    assert q(P(FAKE), P(FAKE), 4, 128, 64, P(FAKE), P(FAKE), 200, s) == ERR_SHAPE       # Kcap % 128
    assert q(P(FAKE), P(FAKE), 4, 0, 64, P(FAKE), P(FAKE), 256, s) == OK
    assert q(P(FAKE), P(FAKE + 2), 4, 128, 64, P(FAKE), P(FAKE), 256, s) == ERR_ALIGN
    g = L.fp8_grouped_gemm_blockscaled_wgrad
    a = (P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE))
    assert g(*a, 0, 128, 128, 128, 256, P(FAKE), s) == ERR_ARG
    assert g(*a, 4, 128, 100, 128, 256, P(FAKE), s) == ERR_SHAPE
    assert g(*a, 4, 128, 128, 128, 100, P(FAKE), s) == ERR_SHAPE
    assert g(*a, 4, 128, 0, 128, 256, P(FAKE), s) == OK
    assert g(*a, 4, 128, 128, 128, 256, None, s) == ERR_ARG


def test_selftest_and_status_arg_checks(L):
    assert L.fp8q_selftest_wait_timeout(0, None) == ERR_ARG
    assert L.fp8q_selftest_wait_timeout(3_000_000_000, None) == ERR_ARG
    assert L.fp8q_device_status(None, None) == ERR_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path")
def test_valid_call_without_gpu_reports_cuda_error(L):
    # With no CUDA device, a well-formed call fails cleanly instead of crashing.
    assert L.fp8q_act_1x128(P(FAKE), 4, 128, P(FAKE), P(FAKE), None) == ERR_CUDA
    v = ctypes.c_int(-1)
    assert L.fp8q_device_status(None, ctypes.byref(v)) == ERR_CUDA


def test_binding_rejects_cpu_tensors():
    with pytest.raises(ValueError):
        ops.act_1x128(torch.zeros(4, 128, dtype=torch.bfloat16))

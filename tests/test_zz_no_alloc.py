"""The allocation-free GEMM entry point, fp8_gemm_blockscaled_noalloc, called through the C ABI.

It exists for callers that may not allocate device memory themselves (a plugin inside a host
framework that owns the memory pool, or a latency-critical path that cannot pay for cudaMalloc's
device-wide synchronisation): it keeps its stream-K scratch in a fixed device array inside the
library instead of a caller workspace.  This file is collected last on purpose, so that a run
that stops at its first failure has run every other test first; it also passes on its own in a
fresh process.

Checked, in Fprop, Dgrad and Wgrad, on two calls in a row (the second one finds the first one's
scratch contents): each output is within the GEMM tolerance of the oracle's exact result, and
bit-identical to the output of the existing entry point, fp8_gemm_blockscaled with its own
workspace (same kernel, same stream-K schedule, so the same FP32 sums in the same order; a
stale partial or flag left in the shared scratch would show up as a difference).  Stream-K is
forced so that every tile is split across CTAs and the scratch is really used.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from fp8_fine_grained_fp8q_b200 import ops, synth
from tests._util import check_gemm, f32_dev, host, u8_dev

pytestmark = pytest.mark.gpu


def _entry():
    fn = ops.lib().fp8_gemm_blockscaled_noalloc
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_int, P, P, P, P, P, I64, I64, I64, P]
    return fn


def _operands(mode):
    if mode == ops.FPROP:
        X = synth.activations_channel_outliers(512, 1024, seed=901)
        W = synth.weights(512, 1024, seed=902)
        a, sa = oracle.quant_1x128(X)
        b, sb, _ = oracle.quant_128x128(W)
    elif mode == ops.DGRAD:
        dY = synth.output_grad(384, 512, seed=905)
        W = synth.weights(512, 768, seed=906)          # forward weight [out = 512, in = 768]
        a, sa = oracle.quant_1x128(dY)
        b, sb, _ = oracle.quant_128x128(W)
    else:
        dY = synth.output_grad(1024, 512, seed=903)
        X = synth.activations_channel_outliers(1024, 512, seed=904)
        a, sa = oracle.quant_128x1_t(dY)
        b, sb = oracle.quant_128x1_t(X)
    return a, sa, b, sb


@pytest.mark.parametrize("mode", [ops.FPROP, ops.DGRAD, ops.WGRAD])
def test_noalloc_matches_oracle_and_workspace_entry_point_on_two_calls_in_a_row(mode, monkeypatch):
    monkeypatch.setenv("FP8Q_GEMM_SCHED", "sk")       # split tiles across CTAs: use the scratch
    a, sa, b, sb = _operands(mode)
    ref, S = oracle.gemm(mode, a, sa, b, sb)
    A, SA, B, SB = u8_dev(a), f32_dev(sa), u8_dev(b), f32_dev(sb)
    M, K = a.shape
    N = b.shape[1] if mode == ops.DGRAD else b.shape[0]
    bf16_out = mode != ops.WGRAD
    dtype = torch.bfloat16 if bf16_out else torch.float32
    with_ws = ops.gemm_blockscaled(mode, A, SA, B, SB)
    assert ops.device_status() == ops.DEV_OK
    check_gemm(host(with_ws), ref, S, "workspace entry point", bf16_out=bf16_out)

    fn = _entry()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        out = torch.full((M, N), float("nan"), dtype=dtype, device="cuda")
        rc = fn(mode, A.data_ptr(), SA.data_ptr(), B.data_ptr(), SB.data_ptr(), out.data_ptr(),
                M, N, K, stream)
        assert rc == 0, ops.status_string(rc)
        assert ops.device_status() == ops.DEV_OK
        check_gemm(host(out), ref, S, f"no-alloc call {call + 1}", bf16_out=bf16_out)
        assert torch.equal(out.view(torch.int16) if bf16_out else out.view(torch.int32),
                           with_ws.view(torch.int16) if bf16_out else with_ws.view(torch.int32)), \
            f"no-alloc call {call + 1} differs from the workspace entry point"

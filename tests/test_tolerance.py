"""The GEMM tolerance accepts correct results and rejects plausible mistakes (CPU only).

Correct: the exact result rounded to bf16 (what an ideal Fprop kernel returns), on the
activation workload with outlier channels, where one product often dominates the sum.
Mistakes, planted in the oracle's inputs on the CPU: one 128-K group's scales dropped, the
weight used untransposed-for-transposed, one weight block's scale off by a factor of 2 (an exponent
slip).  A 1 % scale error in one block is NOT detectable at this tolerance, by design.
"""
import numpy as np
import torch

import oracle
from fp8_fine_grained_fp8q_b200 import synth
from tests._util import check_gemm


def _bf16_round(x):
    return torch.from_numpy(x).to(torch.bfloat16).double().numpy()


def _case():
    X = synth.activations_channel_outliers(256, 512, seed=101)
    W = synth.weights(256, 512, seed=102)
    xq, xs = oracle.quant_1x128(X)
    wq, ws, _ = oracle.quant_128x128(W)
    ref, S = oracle.gemm(oracle.FPROP, xq, xs, wq, ws)
    return xq, xs, wq, ws, ref, S


def _fails(got, ref, S):
    try:
        check_gemm(got, ref, S, "planted")
    except AssertionError:
        return True
    return False


def test_rounded_exact_result_passes():
    *_, ref, S = _case()
    check_gemm(_bf16_round(ref), ref, S, "bf16(ref)")


def test_dropped_group_scale_fails():
    xq, xs, wq, ws, ref, S = _case()
    xs2 = xs.copy()
    xs2[1, :] = 0.0                                   # K group 1 contributes nothing
    bad, _ = oracle.gemm(oracle.FPROP, xq, xs2, wq, ws)
    assert _fails(_bf16_round(bad), ref, S)


def test_wrong_operand_orientation_fails():
    xq, xs, wq, ws, ref, S = _case()
    wq_t = np.ascontiguousarray(wq.reshape(256, 512)[:, :256].T)   # transposed block of W
    wq2 = wq.copy()
    wq2[:, :256] = wq_t
    bad, _ = oracle.gemm(oracle.FPROP, xq, xs, wq2, ws)
    assert _fails(_bf16_round(bad), ref, S)


def test_scale_exponent_slip_fails():
    xq, xs, wq, ws, ref, S = _case()
    ws2 = ws.copy()
    ws2[0, 0] *= np.float32(2.0)
    bad, _ = oracle.gemm(oracle.FPROP, xq, xs, wq, ws2)
    assert _fails(_bf16_round(bad), ref, S)


def test_bf16_rounding_term_comes_from_the_oracle_only():
    """The bf16 term is half a bf16 ulp of |ref| + B (B the accumulator bound): the worst
    accumulator value rounded to bf16 passes, and anything a hair past the bound fails, whatever
    the GPU's own magnitude."""
    from tests._util import tolerance, ulp_bf16
    ref = np.array([1.99, -3.999, 0.75, 1.0e-3])
    S = np.abs(ref) * 1.5
    B = 2e-3 * S + 1e-2 * ulp_bf16(ref)
    bound = tolerance(ref, S, bf16_out=True)
    assert np.allclose(bound, B + 0.5 * ulp_bf16(np.abs(ref) + B), rtol=0, atol=0)
    worst_acc = ref + np.sign(ref) * B
    check_gemm(_bf16_round(worst_acc), ref, S, "bf16 of the worst accumulator")
    over = ref + np.sign(ref) * bound * (1 + 1e-9)
    assert _fails(over, ref, S)
    assert tolerance(ref, S, bf16_out=False).tolist() == B.tolist()

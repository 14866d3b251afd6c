"""GPU quantisers vs the CPU oracle: codes and scales must be bit-exact.

Shapes: the tiny Fprop workload, the full-size activations of the linear layer (X [4096, 7168],
dY [4096, 2048]), the MLA and FFN weights ([2048|1536|512, 7168]), ragged row counts, and
groups holding special values (zeros, signed zeros, bf16 subnormals, values near the bf16
maximum, groups whose amax is under the 2^-100 floor, constant groups).  Outputs are poisoned
before each call so unwritten elements show up.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_fine_grained_fp8q_b200 import ops, synth
from tests._util import bf16_dev, host, linear_layer_inputs

pytestmark = pytest.mark.gpu


def _poison_q(shape):
    return torch.full(shape, 0xA5, dtype=torch.uint8, device="cuda")


def _poison_s(shape):
    return torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")


def run_1x128(bits):
    x = bf16_dev(bits)
    M, K = bits.shape
    q, s = ops.act_1x128(x, _poison_q((M, K)), _poison_s((K // 128, M)))
    torch.cuda.synchronize()
    return host(q), host(s)


def assert_same(gq, gs, oq, os_, what):
    assert gq.shape == oq.shape and gs.shape == os_.shape, what
    bad = np.flatnonzero(gq.reshape(-1) != oq.reshape(-1))
    assert bad.size == 0, f"{what}: {bad.size} codes differ, first at flat {bad[:5]}: " \
                          f"gpu {gq.reshape(-1)[bad[:5]]} oracle {oq.reshape(-1)[bad[:5]]}"
    assert np.array_equal(gs.view(np.uint32), os_.view(np.uint32)), f"{what}: scales differ"


def special_values(rows, cols, seed):
    """bf16 bit patterns with one kind of special group per 128-column block."""
    g = np.random.Generator(np.random.PCG64(seed))
    x = g.standard_normal((rows, cols)).astype(np.float32)
    kinds = cols // 128
    for b in range(kinds):
        blk = x[:, b * 128:(b + 1) * 128]
        k = b % 8
        if k == 0:
            blk[:] = 0.0
        elif k == 1:
            blk[:] = -0.0
        elif k == 2:
            blk[:] = g.choice([1e-39, -2e-39, 5e-40, 0.0], size=blk.shape)   # bf16 subnormals
        elif k == 3:
            blk *= np.float32(1e37)                                           # large magnitudes
        elif k == 4:
            blk *= np.float32(1e-33)                                          # amax under 2^-100
        elif k == 5:
            blk[:] = np.float32(3.0)                                          # constant group
        elif k == 6:
            blk[:, ::2] = 0.0
            blk *= np.float32(1e-20)
    return synth.f32_to_bf16_bits(x)


@pytest.mark.parametrize("M,K", [(1, 128), (3, 256), (256, 512), (300, 1024), (4096, 2048)])
def test_act_1x128_small_and_ragged(M, K):
    bits = synth.activations_entry_outliers(M, K, seed=M * 7 + K)
    gq, gs = run_1x128(bits)
    oq, os_ = oracle.quant_1x128(bits)
    assert_same(gq, gs, oq, os_, f"1x128 {M}x{K}")


def test_act_1x128_special_values():
    bits = special_values(64, 1024, seed=3)
    gq, gs = run_1x128(bits)
    oq, os_ = oracle.quant_1x128(bits)
    assert_same(gq, gs, oq, os_, "1x128 special")


def test_act_1x128_full_size_activations():
    bits = linear_layer_inputs()["X"]               # [4096, 7168], channel outliers
    gq, gs = run_1x128(bits)
    oq, os_ = oracle.quant_1x128(bits)
    assert_same(gq, gs, oq, os_, "1x128 X[4096,7168]")


def test_act_1x128_full_size_output_grad():
    bits = linear_layer_inputs()["dY"]              # [4096, 2048], Student-t entries
    gq, gs = run_1x128(bits)
    oq, os_ = oracle.quant_1x128(bits)
    assert_same(gq, gs, oq, os_, "1x128 dY[4096,2048]")


def run_128x1(bits):
    x = bf16_dev(bits)
    T, C = bits.shape
    qt, s = ops.act_128x1_transposed(x, _poison_q((C, T)), _poison_s((T // 128, C)))
    torch.cuda.synchronize()
    return host(qt), host(s)


@pytest.mark.parametrize("T,C", [(128, 64), (256, 192), (384, 1024)])
def test_act_128x1_small(T, C):
    bits = synth.output_grad(T, C, seed=T + C)
    gq, gs = run_128x1(bits)
    oq, os_ = oracle.quant_128x1_t(bits)
    assert_same(gq, gs, oq, os_, f"128x1 {T}x{C}")


def test_act_128x1_special_values():
    bits = special_values(1024, 256, seed=4).T.copy()    # groups along tokens get the specials
    gq, gs = run_128x1(bits)
    oq, os_ = oracle.quant_128x1_t(bits)
    assert_same(gq, gs, oq, os_, "128x1 special")


@pytest.mark.parametrize("which", ["X", "dY"])
def test_act_128x1_full_size(which):
    bits = linear_layer_inputs()[which]
    gq, gs = run_128x1(bits)
    oq, os_ = oracle.quant_128x1_t(bits)
    assert_same(gq, gs, oq, os_, f"128x1 {which}{bits.shape}")


def run_dual(bits):
    x = bf16_dev(bits)
    T, C = bits.shape
    q, s, qt, st = ops.act_dual(x, _poison_q((T, C)), _poison_s((C // 128, T)),
                                _poison_q((C, T)), _poison_s((T // 128, C)))
    torch.cuda.synchronize()
    return host(q), host(s), host(qt), host(st)


def check_dual(bits, what):
    gq, gs, gqt, gst = run_dual(bits)
    oq, os_ = oracle.quant_1x128(bits)
    oqt, ost = oracle.quant_128x1_t(bits)
    assert_same(gq, gs, oq, os_, f"dual 1x128 {what}")
    assert_same(gqt, gst, oqt, ost, f"dual 128x1 {what}")


@pytest.mark.parametrize("T,C", [(128, 128), (256, 384), (384, 1024)])
def test_act_dual_small(T, C):
    check_dual(synth.activations_channel_outliers(T, C, seed=T * 3 + C), f"{T}x{C}")


def test_act_dual_special_values():
    rows = special_values(256, 1024, seed=5)                 # specials in row groups
    cols = special_values(1024, 256, seed=6).T.copy()        # specials in column groups
    check_dual(np.concatenate([rows, cols], axis=0), "special")


@pytest.mark.parametrize("which", ["X", "dY"])
def test_act_dual_full_size(which):
    bits = linear_layer_inputs()[which]
    check_dual(bits, f"{which}{bits.shape}")


def check_forward(xbits, wbits, transposed, what):
    x, w = bf16_dev(xbits), bf16_dev(wbits)
    T, C = xbits.shape
    N = wbits.shape[0]
    (xq, xs, xqt, xst), (wq, ws, wqt) = ops.quant_forward(
        x, w, _poison_q((T, C)), _poison_s((C // 128, T)), _poison_q((C, T)), _poison_s((T // 128, C)),
        _poison_q((N, C)), _poison_s((N // 128, C // 128)), _poison_q((C, N)) if transposed else None)
    torch.cuda.synchronize()
    oq, os_ = oracle.quant_1x128(xbits)
    oqt, ost = oracle.quant_128x1_t(xbits)
    owq, ows, owqt = oracle.quant_128x128(wbits, want_transposed=transposed)
    assert_same(host(xq), host(xs), oq, os_, f"forward x 1x128 {what}")
    assert_same(host(xqt), host(xst), oqt, ost, f"forward x 128x1 {what}")
    assert_same(host(wq), host(ws), owq, ows, f"forward w {what}")
    if transposed:
        assert np.array_equal(host(wqt), owqt), f"forward w transposed codes {what}"


@pytest.mark.parametrize("T,C,N,transposed", [(128, 128, 128, True), (256, 384, 640, False), (384, 1024, 256, True)])
def test_quant_forward_small(T, C, N, transposed):
    check_forward(synth.activations_channel_outliers(T, C, seed=T + C + N),
                  synth.weights(N, C, seed=T + 2 * N), transposed, f"{T}x{C}, N={N}")


def test_quant_forward_special_values():
    check_forward(special_values(256, 1024, seed=11), special_values(512, 1024, seed=13), True, "special")


def test_quant_forward_full_size():
    d = linear_layer_inputs()
    check_forward(d["X"], d["W"], False, "linear layer")


def run_weight(bits, transposed):
    w = bf16_dev(bits)
    N, K = bits.shape
    qt = _poison_q((K, N)) if transposed else None
    q, s, qt = ops.weight_128x128(w, _poison_q((N, K)), _poison_s((N // 128, K // 128)), qt=qt)
    torch.cuda.synchronize()
    return host(q), host(s), (host(qt) if qt is not None else None)


@pytest.mark.parametrize("N,K", [(128, 128), (512, 512), (256, 1024)])
def test_weight_small_with_transpose(N, K):
    bits = synth.weights(N, K, seed=N + K)
    gq, gs, gqt = run_weight(bits, True)
    oq, os_, oqt = oracle.quant_128x128(bits, want_transposed=True)
    assert_same(gq, gs, oq, os_, f"128x128 {N}x{K}")
    assert np.array_equal(gqt, oqt)


def test_weight_special_values():
    bits = special_values(256, 1024, seed=5)
    gq, gs, _ = run_weight(bits, False)
    oq, os_, _ = oracle.quant_128x128(bits)
    assert_same(gq, gs, oq, os_, "128x128 special")


@pytest.mark.parametrize("N", [2048, 1536, 512])
def test_weight_full_size(N):
    bits = synth.weights(N, 7168, seed=synth.SEED_BASE + N)
    gq, gs, _ = run_weight(bits, False)
    oq, os_, _ = oracle.quant_128x128(bits)
    assert_same(gq, gs, oq, os_, f"128x128 W[{N},7168]")

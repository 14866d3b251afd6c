"""Pins for the oracle's group quantisers.

Groups: 1x128 per token for activations, 128x128 blocks for weights ("DeepSeek-V3 Technical
Report" summary page, Key ideas, FP8 bullet and the Questions answer on FP8 training), and
128x1 along tokens for the Wgrad operands, because the scaling groups lie along the GEMM's
inner dimension (DeepSeek-V3 report repost, paragraph 4) and Wgrad's inner dimension is the
token dimension.  Scaling is max-abs to 448 (this library's reading of the pages' "per-group
scaling factors").

Pins (none of them re-runs the oracle's own formula):
* worked examples with closed-form codes and scales;
* the max-abs invariant: in every group the largest magnitude encodes to +-448 (0x7E / 0xFE);
* the dequantisation error bound of round-to-nearest E4M3;
* one-hot inputs, which pin which group (and, for 128x1, which transposed position) each
  element lands in;
* a library cross-check: amax by numpy reshapes and codes by PyTorch's float8_e4m3fn cast.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_fine_grained_fp8q_b200 import synth

F448 = np.float32(448.0)
FLOOR = np.float32(2.0 ** -100)


def bits(x):
    return synth.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def f32(h):
    return synth.bf16_bits_to_f32(h)


# ------------------------------------------------------------------------------------------ #
# Worked examples
# ------------------------------------------------------------------------------------------ #

def test_worked_example_amax_one():
    row = np.zeros((1, 128), dtype=np.float32)
    row[0, :3] = [1.0, 0.5, -0.25]
    q, s = oracle.quant_1x128(bits(row))
    assert s[0, 0] == np.float32(1.0) / F448          # s = fl(1/448), inverse exactly 448
    assert q[0, 0] == 0x7E                            # 1 * 448 = 448
    assert q[0, 1] == 0x76                            # 224 = 1.75 * 2^7
    assert q[0, 2] == 0xEE                            # -112 = -1.75 * 2^6
    assert np.all(q[0, 3:] == 0)


@pytest.mark.parametrize("j", [-7, -3, 0, 2, 5])
def test_worked_example_power_of_two_scale(j):
    """amax = 448 * 2^j gives s = 2^j exactly and E4M3-representable multiples map exactly."""
    g = np.random.Generator(np.random.PCG64(7 + j))
    ints = g.integers(-16, 17, size=(2, 256)).astype(np.float32)
    ints[:, 0] = 448.0
    ints[:, 128] = -448.0
    x = ints * np.float32(2.0 ** j)
    q, s = oracle.quant_1x128(bits(x))
    assert np.all(s == np.float32(2.0 ** j))
    deq = oracle.e4m3_decode(q) * np.repeat(s.T, 128, axis=1)
    assert np.array_equal(deq, x.astype(np.float64))


def test_zero_and_signed_zero_tiles():
    x = np.zeros((2, 256), dtype=np.float32)
    x[1, 128:] = -0.0
    q, s = oracle.quant_1x128(bits(x))
    assert np.all(s == FLOOR / F448)
    assert np.all(q[0] == 0x00) and np.all(q[1, :128] == 0x00) and np.all(q[1, 128:] == 0x80)


# ------------------------------------------------------------------------------------------ #
# Invariants on the tiny workload and on random 128x1 / 128x128 inputs
# ------------------------------------------------------------------------------------------ #

def _check_groups(xg, qg, sg):
    """xg: float32 values [G, 128*r], qg: codes, sg: [G] scales of each group."""
    amax = np.abs(xg).max(axis=1)
    # The scale is amax / 448 (binary32 division), computed here from numpy's max.
    assert np.array_equal(sg, np.maximum(amax, FLOOR) / F448)
    # Max-abs invariant: the element of largest magnitude encodes to +-448.
    arg = np.abs(xg).argmax(axis=1)
    top = qg[np.arange(qg.shape[0]), arg]
    assert np.all((top & 0x7F) == 0x7E)
    dec = oracle.e4m3_decode(qg)
    assert np.all(np.abs(dec) <= 448.0)
    # Sign agreement (codes of nonzero inputs keep the input's sign).
    nz = xg != 0
    assert np.all((qg[nz] >> 7) == (xg[nz] < 0))
    # Dequantisation error of nearest rounding: 2^-4 relative in the normal E4M3 range,
    # 2^-10 * s absolute in the subnormal range (slack for the binary32 scale products).
    inv = F448 / np.maximum(amax, FLOOR)
    y = np.abs(xg * inv[:, None])
    err = np.abs(xg.astype(np.float64) - dec * sg[:, None].astype(np.float64))
    slack = 1.0 + 2.0 ** -18
    bound = np.where(y >= 2.0 ** -6, 2.0 ** -4 * np.abs(xg) * slack,
                     2.0 ** -10 * sg[:, None].astype(np.float64) * slack)
    assert np.all(err <= bound)


def test_invariants_1x128_tiny_workload():
    x = synth.tiny_fprop()["X"]
    q, s = oracle.quant_1x128(x)
    M, K = x.shape
    xf = f32(x).reshape(M, K // 128, 128).reshape(-1, 128)
    _check_groups(xf, q.reshape(-1, 128), s.T.reshape(-1))


def test_invariants_128x1_transposed():
    x = synth.output_grad(384, 256, seed=11)
    qt, s = oracle.quant_128x1_t(x)
    T, C = x.shape
    assert qt.shape == (C, T) and s.shape == (T // 128, C)
    # Groups of 128 tokens for each channel: in the transposed output they are contiguous.
    xg = f32(x).T.reshape(C, T // 128, 128).reshape(-1, 128)
    _check_groups(xg, qt.reshape(-1, 128), s.T.reshape(-1))


def test_invariants_128x128():
    w = synth.weights(256, 384, seed=12)
    q, s, qt = oracle.quant_128x128(w, want_transposed=True)
    N, K = w.shape
    assert s.shape == (N // 128, K // 128)
    wf = f32(w)
    blocks = wf.reshape(N // 128, 128, K // 128, 128).transpose(0, 2, 1, 3).reshape(-1, 128 * 128)
    qb = q.reshape(N // 128, 128, K // 128, 128).transpose(0, 2, 1, 3).reshape(-1, 128 * 128)
    _check_groups(blocks, qb, s.reshape(-1))
    assert np.array_equal(qt, q.T)


# ------------------------------------------------------------------------------------------ #
# One-hot inputs pin the group indexing
# ------------------------------------------------------------------------------------------ #

def test_one_hot_1x128():
    M, K = 5, 384
    for (r, c, v) in [(0, 0, 3.0), (3, 200, -0.125), (4, 383, 1000.0)]:
        x = np.zeros((M, K), dtype=np.float32)
        x[r, c] = v
        q, s = oracle.quant_1x128(bits(x))
        exp_q = np.zeros((M, K), dtype=np.uint8)
        exp_q[r, c] = 0x7E | (0x80 if v < 0 else 0)
        assert np.array_equal(q, exp_q)
        exp_s = np.full((K // 128, M), FLOOR / F448, dtype=np.float32)
        exp_s[c // 128, r] = np.float32(abs(v)) / F448
        assert np.array_equal(s, exp_s)


def test_one_hot_128x1_transposed():
    T, C = 256, 3
    for (t, c, v) in [(0, 0, 2.0), (130, 2, -7.0), (255, 1, 0.5)]:
        x = np.zeros((T, C), dtype=np.float32)
        x[t, c] = v
        qt, s = oracle.quant_128x1_t(bits(x))
        exp_q = np.zeros((C, T), dtype=np.uint8)
        exp_q[c, t] = 0x7E | (0x80 if v < 0 else 0)
        assert np.array_equal(qt, exp_q)
        exp_s = np.full((T // 128, C), FLOOR / F448, dtype=np.float32)
        exp_s[t // 128, c] = np.float32(abs(v)) / F448
        assert np.array_equal(s, exp_s)


def test_one_hot_128x128():
    N, K = 256, 384
    for (n, k, v) in [(0, 0, 1.0), (200, 129, -3.0), (255, 383, 0.25)]:
        x = np.zeros((N, K), dtype=np.float32)
        x[n, k] = v
        q, s, qt = oracle.quant_128x128(bits(x), want_transposed=True)
        exp_q = np.zeros((N, K), dtype=np.uint8)
        exp_q[n, k] = 0x7E | (0x80 if v < 0 else 0)
        assert np.array_equal(q, exp_q) and np.array_equal(qt, exp_q.T)
        exp_s = np.full((N // 128, K // 128), FLOOR / F448, dtype=np.float32)
        exp_s[n // 128, k // 128] = np.float32(abs(v)) / F448
        assert np.array_equal(s, exp_s)


# ------------------------------------------------------------------------------------------ #
# Library cross-check: numpy reshapes for the groups, PyTorch's cast for the codes
# ------------------------------------------------------------------------------------------ #

def _torch_quant_groups(xg):
    amax = np.abs(xg).max(axis=1)
    inv = F448 / np.maximum(amax, FLOOR)
    y = (xg * inv[:, None]).astype(np.float32)    # one binary32 multiply per element
    # |y| <= 448 * (1 + 2^-23) < 464, where PyTorch's cast agrees with saturation.
    codes = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return codes


def test_cross_check_1x128_torch():
    x = synth.activations_channel_outliers(256, 1024, seed=21)
    q, _ = oracle.quant_1x128(x)
    xg = f32(x).reshape(-1, 128)
    assert np.array_equal(q.reshape(-1, 128), _torch_quant_groups(xg))


def test_cross_check_128x1_torch():
    x = synth.output_grad(256, 384, seed=22)
    qt, _ = oracle.quant_128x1_t(x)
    xg = f32(x).T.reshape(-1, 128)
    assert np.array_equal(qt.reshape(-1, 128), _torch_quant_groups(xg))


def test_cross_check_128x128_torch():
    w = synth.weights(256, 256, seed=23)
    q, _, _ = oracle.quant_128x128(w)
    wf = f32(w)
    blocks = wf.reshape(2, 128, 2, 128).transpose(0, 2, 1, 3).reshape(-1, 128 * 128)
    qb = q.reshape(2, 128, 2, 128).transpose(0, 2, 1, 3).reshape(-1, 128 * 128)
    assert np.array_equal(qb, _torch_quant_groups(blocks))

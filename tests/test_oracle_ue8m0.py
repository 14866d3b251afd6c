"""Pins for the oracle's power-of-two (UE8M0) scale mode of the group quantisers.

The mode is not on the pages: it is the scale format the block-scaled tensor-core MMA accepts,
built as a separate mode beside the pages' max-abs scale.  Its definition (this library's
reading): a = max(amax, 2^-100); s = the smallest power of two not below the binary32 quotient
a / 448; codes are E4M3 of x / s, which is exact because s is a power of two.

Pins (none re-runs the oracle's frexp-based formula):
* worked examples whose scales and codes are worked out by hand;
* every scale is a power of two with s/2 < fl32(a/448) <= s, the bound checked with numpy;
* the codes are the round-to-nearest-even E4M3 values of x / s, found by brute force over the
  whole E4M3 grid;
* where a / 448 is already a power of two, the mode agrees with the pages' max-abs mode bit for
  bit;
* the 128x1 transposed and 128x128 forms against the 1x128 form on rearranged inputs, and one-hot
  inputs for their group indexing.
"""
import numpy as np
import pytest

import oracle
from fp8_fine_grained_fp8q_b200 import synth

F448 = np.float32(448.0)
FLOOR = np.float32(2.0 ** -100)


def bits(x):
    return synth.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def f32(h):
    return synth.bf16_bits_to_f32(h)


def _grid():
    """All finite non-negative E4M3 values (codes 0x00 .. 0x7E) by their definition: bias 7,
    3 mantissa bits, subnormals m * 2^-9."""
    vals = []
    for c in range(0x7F):
        e, m = c >> 3, c & 7
        vals.append(m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))
    return np.array(vals)


GRID = _grid()


def _rne_codes(v):
    """Round-to-nearest-even E4M3 codes of exact values |v| <= 448, by brute force."""
    a = np.abs(v)[..., None]
    d = np.abs(GRID - a)
    best = d.min(axis=-1, keepdims=True)
    cand = d == best
    # Ties: the code with an even mantissa (its last bit is 0).
    even = (np.arange(GRID.size) & 1) == 0
    pick = np.where(cand.sum(axis=-1, keepdims=True) > 1, cand & even, cand)
    code = pick.argmax(axis=-1).astype(np.uint8)
    neg = (v < 0) | ((v == 0) & np.signbit(v))
    return code | np.where(neg, 0x80, 0).astype(np.uint8)


# ------------------------------------------------------------------------------------------ #
# Worked examples
# ------------------------------------------------------------------------------------------ #

def test_worked_examples_1x128():
    rows = np.zeros((6, 128), dtype=np.float32)
    rows[0, :2] = [448.0, -448.0]      # a/448 = 1          -> s = 1, codes +-448
    rows[1, :2] = [450.0, 225.0]       # a/448 = 1.0045     -> s = 2: 225, 112.5 -> 224, 112
    rows[2, :2] = [1.0, -0.5]          # a/448 = 2^-8.8     -> s = 2^-8: 256, -128
    rows[3, :2] = [3.0, 1.0]           # a/448 = 0.0067     -> s = 2^-7: 384, 128
    rows[4, 0] = 448.0 * 2.0 ** -20    # a/448 = 2^-20      -> s = 2^-20, code 448
    # row 5 all zero: a = 2^-100, a/448 = 2^-108.8 -> s = 2^-108, zero codes
    q, s = oracle.quant_1x128(bits(rows), scale_fmt="ue8m0")
    want_s = np.float32([1.0, 2.0, 2.0 ** -8, 2.0 ** -7, 2.0 ** -20, 2.0 ** -108])
    assert np.array_equal(s[0], want_s)
    # E4M3 codes: 448 = 0x7E, 224 = 1.75*2^7 = 0x76, 112 = 1.75*2^6 = 0x6E, 256 = 2^8 = 0x78,
    # 128 = 2^7 = 0x70, 384 = 1.5*2^8 = 0x7C.
    assert list(q[0, :2]) == [0x7E, 0xFE]
    assert list(q[1, :2]) == [0x76, 0x6E]
    assert list(q[2, :2]) == [0x78, 0xF0]
    assert list(q[3, :2]) == [0x7C, 0x70]
    assert q[4, 0] == 0x7E
    assert not q[5].any() and not q[0, 2:].any()


def test_round_half_even_at_a_power_of_two_scale():
    # s = 1 (amax 448): 17 lies halfway between 16 (0x58) and 18 (0x59): ties go to the even
    # mantissa, 16.  19 is halfway between 18 and 20 (0x5A): 20.
    row = np.zeros((1, 128), dtype=np.float32)
    row[0, :3] = [448.0, 17.0, 19.0]
    q, s = oracle.quant_1x128(bits(row), scale_fmt="ue8m0")
    assert s[0, 0] == 1.0
    assert list(q[0, :3]) == [0x7E, 0x58, 0x5A]


# ------------------------------------------------------------------------------------------ #
# Invariants and brute force
# ------------------------------------------------------------------------------------------ #

def _check_groups(xg, qg, sg):
    """xg float32 [G, n] group values, qg their codes, sg [G] scales."""
    sg = sg.astype(np.float32)
    mant = sg.view(np.uint32) & 0x7FFFFF
    assert not mant.any(), "scales must be powers of two"
    r = np.maximum(np.abs(xg).max(axis=1), FLOOR) / F448       # binary32 quotient
    assert np.all(r <= sg) and np.all(r > sg / 2)
    v = xg.astype(np.float64) / sg[:, None].astype(np.float64)   # exact: s is a power of two
    assert np.all(np.abs(v) <= 448.0)
    assert np.array_equal(qg, _rne_codes(v))


def test_brute_force_1x128():
    x = synth.activations_entry_outliers(64, 512, seed=401)
    q, s = oracle.quant_1x128(x, scale_fmt="ue8m0")
    M, K = x.shape
    _check_groups(f32(x).reshape(-1, 128), q.reshape(-1, 128), s.T.reshape(-1))


def test_brute_force_128x1_transposed():
    x = synth.output_grad(256, 96, seed=402)
    qt, s = oracle.quant_128x1_t(x, scale_fmt="ue8m0")
    T, C = x.shape
    xg = f32(x).T.reshape(C, T // 128, 128).reshape(-1, 128)
    _check_groups(xg, qt.reshape(-1, 128), s.T.reshape(-1))


def test_brute_force_128x128():
    w = synth.weights(256, 256, seed=403)
    q, s, qt = oracle.quant_128x128(w, want_transposed=True, scale_fmt="ue8m0")
    N, K = w.shape
    blocks = f32(w).reshape(N // 128, 128, K // 128, 128).transpose(0, 2, 1, 3).reshape(-1, 128 * 128)
    qb = q.reshape(N // 128, 128, K // 128, 128).transpose(0, 2, 1, 3).reshape(-1, 128 * 128)
    _check_groups(blocks, qb, s.reshape(-1))
    assert np.array_equal(qt, q.T)


def test_power_of_two_ratio_agrees_with_max_abs_mode():
    # Every group's max-abs is 448 * 2^j exactly, so a / 448 = 2^j in both modes, 448 / a = 2^-j
    # exactly, and the two modes must give the same scales and codes.
    g = np.random.Generator(np.random.PCG64(404))
    x = (g.standard_normal((8, 512)) * 40).astype(np.float32)
    x = f32(bits(np.clip(x, -440, 440)))            # bf16 values below 448 in magnitude
    for r in range(8):
        for t in range(4):
            j = int(g.integers(-12, 6))
            x[r, 128 * t:128 * (t + 1)] *= np.float32(2.0 ** j)
            x[r, 128 * t + int(g.integers(0, 128))] = np.float32(448.0 * 2.0 ** j) * (1 if r % 2 else -1)
    xb = bits(x)
    assert np.array_equal(f32(xb), x), "inputs chosen to be bf16-exact"
    q0, s0 = oracle.quant_1x128(xb)
    q1, s1 = oracle.quant_1x128(xb, scale_fmt="ue8m0")
    assert np.array_equal(s0, s1) and np.array_equal(q0, q1)


def test_forms_agree_on_rearranged_inputs():
    # 128x1 on x[T, C] is 1x128 on x^T; a 128x128 block whose rows are all equal to one
    # 128-wide row has that row's 1x128 scale.
    x = synth.activations_channel_outliers(256, 128, seed=405)
    qt, st = oracle.quant_128x1_t(x, scale_fmt="ue8m0")
    q1, s1 = oracle.quant_1x128(np.ascontiguousarray(x.T), scale_fmt="ue8m0")
    assert np.array_equal(qt, q1) and np.array_equal(st, s1)
    row = x[:1]
    w = np.repeat(row, 128, axis=0)
    qw, sw, _ = oracle.quant_128x128(w, scale_fmt="ue8m0")
    qr, sr = oracle.quant_1x128(row, scale_fmt="ue8m0")
    assert sw[0, 0] == sr[0, 0] and np.array_equal(qw, np.repeat(qr, 128, axis=0))


@pytest.mark.parametrize("where", [(0, 0), (130, 5), (255, 127)])
def test_one_hot_128x1_transposed(where):
    t, c = where
    x = np.zeros((256, 128), dtype=np.float32)
    x[t, c] = -5.0                          # s = 2^-6 (5/448 = 0.0112): -320 = -1.25 * 2^8
    qt, s = oracle.quant_128x1_t(bits(x), scale_fmt="ue8m0")
    assert np.argwhere(qt != 0).tolist() == [[c, t]]
    assert qt[c, t] == 0xFA
    assert s[t // 128, c] == np.float32(2.0 ** -6)
    assert np.all(s[np.arange(2) != t // 128] == np.float32(2.0 ** -108))


def test_ragged_mode_passes_through():
    off = np.array([0, 3, 3, 200])
    x = synth.output_grad(200, 64, seed=406)
    qt, s = oracle.quant_128x1_t_ragged(x, off, scale_fmt="ue8m0")
    assert not (s.view(np.uint32) & 0x7FFFFF).any()
    P = oracle.ragged_group_prefix(off)
    blk = np.zeros((128, 64), dtype=np.uint16)
    blk[:3] = x[:3]
    q0, s0 = oracle.quant_128x1_t(blk, scale_fmt="ue8m0")
    assert np.array_equal(qt[:, :128], q0) and np.array_equal(s[P[0]], s0[0])


def test_bad_format_is_rejected():
    with pytest.raises(ValueError):
        oracle.quant_1x128(bits(np.zeros((1, 128))), scale_fmt="e4m3")

"""Pins of the oracle's ragged 128x1 quantiser (the grouped-Wgrad operand form) against facts
that do not come from its own code path: the plain 128x1 quantiser when every expert's token
count is a multiple of 128, a one-token expert whose codes and scales have a closed form, the
max-abs invariant of every (expert, group, channel), group scales recomputed from the unpadded
rows with numpy, and the position of a single non-zero input."""
import numpy as np

import oracle
from fp8_fine_grained_fp8q_b200 import synth


def _offsets(counts):
    off = np.zeros(len(counts) + 1, dtype=np.int64)
    off[1:] = np.cumsum(counts)
    return off


def _f32(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


def test_whole_groups_equal_the_plain_quantiser():
    counts = [128, 0, 256, 384]
    off = _offsets(counts)
    x = synth.output_grad(int(off[-1]), 192, seed=301)
    qt, s = oracle.quant_128x1_t_ragged(x, off)
    pq, ps = oracle.quant_128x1_t(x)
    assert np.array_equal(qt, pq) and np.array_equal(s.view(np.uint32), ps.view(np.uint32))


def test_one_token_expert_closed_form():
    # A single token: every channel's group is that one value, so its code is +-448 (0x7E with
    # the sign bit) and its scale |v| / 448; the other 127 positions are zero codes.
    vals = np.array([1.0, -3.5, 0.0, 2.0 ** -20, -448.0, 1e30], dtype=np.float32)
    C = 128
    row = np.zeros((1, C), dtype=np.float32)
    row[0, :vals.size] = vals
    bits = synth.f32_to_bf16_bits(row)
    qt, s = oracle.quant_128x1_t_ragged(bits, np.array([0, 1]))
    assert qt.shape == (C, 128) and s.shape == (1, C)
    v = _f32(bits[0])
    for c in range(C):
        a = abs(float(v[c]))
        want_code = 0 if a == 0 else (0x7E | (0x80 if v[c] < 0 else 0))
        assert qt[c, 0] == want_code
        assert not qt[c, 1:].any()
        assert s[0, c] == np.float32(max(a, 2.0 ** -100)) / np.float32(448.0)


def test_max_abs_invariant_and_group_scales_from_unpadded_rows():
    counts = [1, 0, 127, 129, 300, 5]
    off = _offsets(counts)
    C = 128
    x = synth.activations_channel_outliers(int(off[-1]), C, seed=302)
    qt, s = oracle.quant_128x1_t_ragged(x, off)
    P = oracle.ragged_group_prefix(off)
    xf = _f32(x)
    for e, n in enumerate(counts):
        for j in range(int(P[e + 1] - P[e])):
            r0 = int(off[e]) + 128 * j
            r1 = min(r0 + 128, int(off[e + 1]))
            amax = np.abs(xf[r0:r1]).max(axis=0)
            want = np.maximum(amax, np.float32(2.0 ** -100)) / np.float32(448.0)
            g = int(P[e]) + j
            assert np.array_equal(s[g], want.astype(np.float32))
            cols = qt[:, 128 * g:128 * g + (r1 - r0)]
            assert ((cols & 0x7F).max(axis=1) == np.where(amax > 0, 0x7E, 0)).all()
            assert not qt[:, 128 * g + (r1 - r0):128 * (g + 1)].any()


def test_single_nonzero_lands_at_its_padded_position():
    counts = [3, 0, 200, 1]
    off = _offsets(counts)
    C = 64
    P = oracle.ragged_group_prefix(off)
    for e, r, c in [(0, 2, 5), (2, 130, 63), (3, 0, 0)]:
        x = np.zeros((int(off[-1]), C), dtype=np.float32)
        x[int(off[e]) + r, c] = -2.0
        qt, _ = oracle.quant_128x1_t_ragged(synth.f32_to_bf16_bits(x), off)
        nz = np.argwhere(qt != 0)
        assert nz.tolist() == [[c, 128 * int(P[e]) + r]]
        assert qt[c, 128 * int(P[e]) + r] == 0xFE          # -448

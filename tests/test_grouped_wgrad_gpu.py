"""GPU grouped Wgrad for MoE experts vs the oracle: the ragged 128x1 transposed quantiser (codes
and scales bit-exact against the oracle's, the untouched tail left alone) and the K-grouped
block-scaled GEMM dW_e = dY_e^T X_e (every expert within the GEMM tolerance, experts without
tokens exactly zero), plus the device-side offset checks."""
import numpy as np
import pytest
import torch

import oracle
from fp8_fine_grained_fp8q_b200 import ops, synth
from tests._util import bf16_dev, check_gemm, host

pytestmark = pytest.mark.gpu


def _offsets(counts):
    off = np.zeros(len(counts) + 1, dtype=np.int32)
    off[1:] = np.cumsum(counts)
    return off


def _ragged(bits, off, Kcap=None):
    E = off.size - 1
    Mtot, C = bits.shape
    Kcap = ops.ragged_capacity(Mtot, E) if Kcap is None else Kcap
    qt = torch.full((C, Kcap), 0xA5, dtype=torch.uint8, device="cuda")
    s = torch.full((Kcap // 128, C), float("nan"), dtype=torch.float32, device="cuda")
    ops.act_128x1_transposed_ragged(bf16_dev(bits), torch.from_numpy(off).cuda(), Kcap, qt, s)
    status = ops.device_status()
    return qt, s, status


@pytest.mark.parametrize("counts", [[1, 0, 127, 129, 300, 5], [128, 256], [0, 0, 7], [200]])
def test_ragged_quantiser_matches_the_oracle(counts):
    off = _offsets(counts)
    C = 192
    bits = synth.output_grad(int(off[-1]), C, seed=sum(counts) + len(counts))
    qt, s, status = _ragged(bits, off)
    assert status == ops.DEV_OK
    oq, os_ = oracle.quant_128x1_t_ragged(bits, off)
    G = os_.shape[0]
    gq, gs = host(qt), host(s)
    assert np.array_equal(gq[:, :128 * G], oq), "codes differ from the oracle"
    assert np.array_equal(gs[:G].view(np.uint32), os_.view(np.uint32)), "scales differ from the oracle"
    assert (gq[:, 128 * G:] == 0xA5).all() and np.isnan(gs[G:]).all(), "the unused tail was written"


def test_ragged_quantiser_bad_offsets_and_small_capacity():
    off = _offsets([100, 50])
    bits = synth.output_grad(150, 64, seed=9)
    bad = off.copy()
    bad[2] = 160                                          # does not end at Mtot
    qt, s, status = _ragged(bits, bad)
    assert status == ops.DEV_BAD_OFFSETS and (host(qt) == 0xA5).all()
    qt, s, status = _ragged(bits, off, Kcap=128)          # two experts need two groups
    assert status == ops.DEV_BAD_OFFSETS and (host(qt) == 0xA5).all()


def _wgrad_problem(counts, M, N, seed):
    off = _offsets(counts)
    Mtot = int(off[-1])
    dY = synth.output_grad(max(Mtot, 1), M, seed=seed)[:Mtot]
    X = synth.activations_channel_outliers(max(Mtot, 1), N, seed=seed + 1)[:Mtot]
    return off, dY, X


@pytest.mark.parametrize("bn", [128, 256])
@pytest.mark.parametrize("counts", [[1, 0, 127, 129, 300, 5], [256], [0, 40]])
def test_grouped_wgrad_every_expert(counts, bn, monkeypatch):
    monkeypatch.setenv("FP8Q_GEMM_BN", str(bn))
    M, N = 256, 512
    off, dY, X = _wgrad_problem(counts, M, N, seed=7 * len(counts) + sum(counts))
    offs = torch.from_numpy(off).cuda()
    Mtot = int(off[-1])
    dyt, sdy = ops.act_128x1_transposed_ragged(bf16_dev(dY), offs)
    xt, sx = ops.act_128x1_transposed_ragged(bf16_dev(X), offs)
    out = torch.full((len(counts), M, N), float("nan"), dtype=torch.float32, device="cuda")
    ops.grouped_gemm_blockscaled_wgrad(dyt, sdy, xt, sx, offs, Mtot, out=out)
    assert ops.device_status() == ops.DEV_OK
    got = host(out).astype(np.float64)
    oq_y, os_y = oracle.quant_128x1_t_ragged(dY, off)
    oq_x, os_x = oracle.quant_128x1_t_ragged(X, off)
    P = oracle.ragged_group_prefix(off)
    for e, n in enumerate(counts):
        if n == 0:
            assert not got[e].any(), f"expert {e} has no tokens: dW must be zero"
            continue
        k0, k1 = 128 * int(P[e]), 128 * int(P[e + 1])
        ref, S = oracle.gemm(ops.WGRAD, np.ascontiguousarray(oq_y[:, k0:k1]), os_y[P[e]:P[e + 1]],
                             np.ascontiguousarray(oq_x[:, k0:k1]), os_x[P[e]:P[e + 1]])
        check_gemm(got[e], ref, S, f"grouped wgrad expert {e} ({n} tokens)", bf16_out=False)


def test_grouped_wgrad_bad_offsets_write_nothing():
    counts = [128, 128]
    off, dY, X = _wgrad_problem(counts, 128, 128, seed=3)
    offs = torch.from_numpy(off).cuda()
    dyt, sdy = ops.act_128x1_transposed_ragged(bf16_dev(dY), offs)
    xt, sx = ops.act_128x1_transposed_ragged(bf16_dev(X), offs)
    assert ops.device_status() == ops.DEV_OK
    bad = off.copy()
    bad[1] = 300                                          # decreasing
    out = torch.full((2, 128, 128), 5.0, dtype=torch.float32, device="cuda")
    ops.grouped_gemm_blockscaled_wgrad(dyt, sdy, xt, sx, torch.from_numpy(bad).cuda(), 256, out=out)
    assert ops.device_status() == ops.DEV_BAD_OFFSETS
    assert bool((out == 5.0).all())

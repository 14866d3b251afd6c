"""Full-size parity of the experts' backward GEMMs: grouped Dgrad and grouped Wgrad at the MoE shape
of the benchmark (8192 tokens x top-8 routing over 256 experts, expert width 2048, hidden 7168;
"DeepSeek-V3 Technical Report" summary page, Key ideas: 256 routed experts, 8 active).

Sampled experts (the largest, the smallest non-empty, and random ones) are checked entry by entry
against the oracle's plain GEMM of that expert: every column of sampled rows for Dgrad, sampled
(row, column) pairs of each sampled expert's dW for Wgrad.  Experts without tokens must get an
all-zero dW, every routed row of dX must be written, and the GPU's ragged 128x1 codes and scales
of the sampled experts must equal the oracle's bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_fine_grained_fp8q_b200 import ops, synth
from tests._util import bf16_dev, check_gemm, f32_dev, host, u8_dev

pytestmark = pytest.mark.gpu

E, N_OUT, K_IN, TOKENS = 256, 2048, 7168, 8192


def _routing():
    expert_of, counts = synth.moe_routing(tokens=TOKENS, experts=E)
    token_idx, off = synth.moe_grouped_rows(expert_of, E)
    assert (counts == 0).sum() >= 1 and counts.sum() == TOKENS * 8
    return counts, token_idx, off


def _sampled_experts(counts, g):
    nonempty = np.flatnonzero(counts > 0)
    pick = {int(np.argmax(counts)), int(nonempty[np.argmin(counts[nonempty])])}
    pick |= set(int(e) for e in g.choice(nonempty, size=5, replace=False))
    return sorted(pick)


def test_full_size_grouped_dgrad():
    counts, _, off = _routing()
    Mtot = int(off[-1])
    dY = synth.output_grad(Mtot, N_OUT, seed=synth.SEED_BASE + 41)
    gq, gs = oracle.quant_1x128(dY)
    # Expert weights [out = 2048, in = 7168]: 8 distinct quantised matrices reused across the
    # experts, each expert's block scales multiplied by its own seeded factor.
    pool = [oracle.quant_128x128(synth.expert_weights(p, N_OUT, K_IN)) for p in range(8)]
    g = np.random.Generator(np.random.PCG64(78))
    factor = g.uniform(0.5, 2.0, size=E).astype(np.float32)
    ws = np.stack([pool[e % 8][1] * factor[e] for e in range(E)]).astype(np.float32)
    pool_dev = torch.stack([u8_dev(pool[p][0]) for p in range(8)])
    wq_dev = pool_dev[torch.arange(E) % 8].contiguous()                  # [E, 2048, 7168]
    del pool_dev
    out = torch.full((Mtot, K_IN), float("nan"), dtype=torch.bfloat16, device="cuda")
    ops.grouped_gemm_blockscaled_dgrad(u8_dev(gq), f32_dev(gs), wq_dev, f32_dev(ws), torch.from_numpy(off).cuda(),
                                       out=out)
    assert ops.device_status() == ops.DEV_OK
    assert bool(torch.isfinite(out).all()), "every routed row of dX must be written"
    for e in _sampled_experts(counts, g):
        r0, r1 = int(off[e]), int(off[e + 1])
        rows = np.unique(np.concatenate([[r0, r1 - 1], g.integers(r0, r1, size=4)]))
        got = host(out[torch.from_numpy(rows).cuda()])
        ms = np.repeat(rows - r0, K_IN)
        ns = np.tile(np.arange(K_IN), rows.size)
        ref, S = oracle.gemm_entries(ops.DGRAD, gq[r0:r1], np.ascontiguousarray(gs[:, r0:r1]), pool[e % 8][0],
                                     ws[e], ms, ns)
        check_gemm(got.reshape(-1), ref, S, f"grouped dgrad expert {e} ({r1 - r0} rows)")


def test_full_size_grouped_wgrad():
    counts, token_idx, off = _routing()
    Mtot = int(off[-1])
    X = synth.activations_channel_outliers(TOKENS, K_IN, seed=synth.SEED_BASE + 4)[token_idx]   # expert order
    dY = synth.output_grad(Mtot, N_OUT, seed=synth.SEED_BASE + 42)
    offs = torch.from_numpy(off).cuda()
    dyt, sdy = ops.act_128x1_transposed_ragged(bf16_dev(dY), offs)
    xt, sx = ops.act_128x1_transposed_ragged(bf16_dev(X), offs)
    dw = torch.full((E, N_OUT, K_IN), float("nan"), dtype=torch.float32, device="cuda")   # 15 GB
    ops.grouped_gemm_blockscaled_wgrad(dyt, sdy, xt, sx, offs, Mtot, out=dw)
    assert ops.device_status() == ops.DEV_OK
    for e in np.flatnonzero(counts == 0):
        assert int(torch.count_nonzero(dw[int(e)])) == 0, f"expert {e} has no tokens: dW must be zero"
    P = oracle.ragged_group_prefix(off)
    g = np.random.Generator(np.random.PCG64(79))
    for e in _sampled_experts(counts, g):
        r0, r1 = int(off[e]), int(off[e + 1])
        e_off = np.array([0, r1 - r0], dtype=np.int32)
        oq_y, os_y = oracle.quant_128x1_t_ragged(dY[r0:r1], e_off)
        oq_x, os_x = oracle.quant_128x1_t_ragged(X[r0:r1], e_off)
        k0, k1 = 128 * int(P[e]), 128 * int(P[e + 1])
        # The GPU's ragged operands of this expert, bit for bit.
        assert np.array_equal(host(dyt[:, k0:k1]), oq_y) and np.array_equal(host(xt[:, k0:k1]), oq_x)
        assert np.array_equal(host(sdy[P[e]:P[e + 1]]).view(np.uint32), os_y.view(np.uint32))
        assert np.array_equal(host(sx[P[e]:P[e + 1]]).view(np.uint32), os_x.view(np.uint32))
        ms = np.concatenate([np.repeat([0, N_OUT - 1], 64), g.integers(0, N_OUT, 2048)])
        ns = np.concatenate([np.tile(g.integers(0, K_IN, 64), 2), g.integers(0, K_IN, 2048)])
        got = dw[e][torch.from_numpy(ms).cuda(), torch.from_numpy(ns).cuda()].cpu().numpy().astype(np.float64)
        ref, S = oracle.gemm_entries(ops.WGRAD, oq_y, os_y, oq_x, os_x, ms, ns)
        check_gemm(got, ref, S, f"grouped wgrad expert {e} ({r1 - r0} tokens)", bf16_out=False)
    assert bool(torch.isfinite(dw).all()), "every expert's dW must be written"

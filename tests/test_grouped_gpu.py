"""GPU grouped (MoE expert) block-scaled FP8 Fprop and Dgrad vs the oracle, and the device-side
checks.

Row groups come from the seeded Zipf-skewed top-8 routing (some experts empty).  Small cases
compare every output; the full-size case (8192 tokens x top-8 over 256 experts, N = 2048,
K = 7168) checks every row was written and samples experts (the largest, the smallest
non-empty, and random ones) entry by entry against the oracle's plain Fprop per expert.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_fine_grained_fp8q_b200 import ops, synth
from tests._util import check_gemm, f32_dev, host, u8_dev

pytestmark = pytest.mark.gpu


def run_grouped(aq, as_, bq, bs, off, bn=None, monkeypatch=None):
    if bn is not None:
        monkeypatch.setenv("FP8Q_GEMM_BN", str(bn))
    Mtot = aq.shape[0]
    N = bq.shape[1]
    out = torch.full((Mtot, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    ops.grouped_gemm_blockscaled(u8_dev(aq), f32_dev(as_), u8_dev(bq), f32_dev(bs),
                                 torch.from_numpy(off.astype(np.int32)).cuda(), out=out)
    status = ops.device_status()
    return host(out), status


def small_problem(counts, N, K, seed):
    counts = np.asarray(counts)
    E = counts.size
    off = np.zeros(E + 1, dtype=np.int32)
    off[1:] = np.cumsum(counts)
    Mtot = int(off[-1])
    A = synth.activations_channel_outliers(max(Mtot, 1), K, seed=seed)[:Mtot]
    aq, as_ = oracle.quant_1x128(A)
    bq = np.empty((E, N, K), dtype=np.uint8)
    bs = np.empty((E, N // 128, K // 128), dtype=np.float32)
    for e in range(E):
        bq[e], bs[e], _ = oracle.quant_128x128(synth.weights(N, K, seed=seed * 31 + e))
    return aq, as_, bq, bs, off


@pytest.mark.parametrize("bn", [128, 256])
@pytest.mark.parametrize("counts", [[0, 1, 130, 0, 255, 64], [128], [0, 0, 300], [5, 0]])
def test_grouped_small_all_entries(counts, bn, monkeypatch):
    N, K = 256, 384
    aq, as_, bq, bs, off = small_problem(counts, N, K, seed=len(counts) + sum(counts))
    got, status = run_grouped(aq, as_, bq, bs, off, bn, monkeypatch)
    assert status == ops.DEV_OK
    Mtot = aq.shape[0]
    ms, ns = np.meshgrid(np.arange(Mtot), np.arange(N), indexing="ij")
    ref, S = oracle.grouped_entries(aq, as_, bq, bs, off, ms.reshape(-1), ns.reshape(-1))
    check_gemm(got, ref.reshape(Mtot, N), S.reshape(Mtot, N), f"grouped {counts}")


def dgrad_problem(counts, Nin, Kout, seed):
    """dY rows grouped by expert and the experts' forward weights W_e [Kout, Nin] (128x128)."""
    counts = np.asarray(counts)
    E = counts.size
    off = np.zeros(E + 1, dtype=np.int32)
    off[1:] = np.cumsum(counts)
    Mtot = int(off[-1])
    dY = synth.output_grad(max(Mtot, 1), Kout, seed=seed)[:Mtot]
    gq, gs = oracle.quant_1x128(dY)
    wq = np.empty((E, Kout, Nin), dtype=np.uint8)
    ws = np.empty((E, Kout // 128, Nin // 128), dtype=np.float32)
    for e in range(E):
        wq[e], ws[e], _ = oracle.quant_128x128(synth.weights(Kout, Nin, seed=seed * 37 + e))
    return gq, gs, wq, ws, off


@pytest.mark.parametrize("bn", [128, 256])
@pytest.mark.parametrize("counts", [[0, 1, 130, 0, 255, 64], [128], [5, 0, 300]])
def test_grouped_dgrad_small_all_entries(counts, bn, monkeypatch):
    Nin, Kout = 512, 256
    monkeypatch.setenv("FP8Q_GEMM_BN", str(bn))
    gq, gs, wq, ws, off = dgrad_problem(counts, Nin, Kout, seed=len(counts) * 7 + sum(counts))
    out = torch.full((gq.shape[0], Nin), float("nan"), dtype=torch.bfloat16, device="cuda")
    ops.grouped_gemm_blockscaled_dgrad(u8_dev(gq), f32_dev(gs), u8_dev(wq), f32_dev(ws),
                                       torch.from_numpy(off).cuda(), out=out)
    assert ops.device_status() == ops.DEV_OK
    got = host(out)
    for e in range(len(counts)):
        r0, r1 = int(off[e]), int(off[e + 1])
        if r1 == r0:
            continue
        ref, S = oracle.gemm(ops.DGRAD, gq[r0:r1], np.ascontiguousarray(gs[:, r0:r1]), wq[e], ws[e])
        check_gemm(got[r0:r1], ref, S, f"grouped dgrad expert {e} ({r1 - r0} rows)")


def test_grouped_dgrad_bad_offsets_are_reported():
    gq, gs, wq, ws, off = dgrad_problem([128, 128], 256, 128, seed=5)
    bad = off.copy()
    bad[1], bad[2] = 200, 300          # the last offset (300) is not Mtot (256)
    out = torch.full((gq.shape[0], 256), 7.0, dtype=torch.bfloat16, device="cuda")
    ops.grouped_gemm_blockscaled_dgrad(u8_dev(gq), f32_dev(gs), u8_dev(wq), f32_dev(ws),
                                       torch.from_numpy(bad).cuda(), out=out)
    assert ops.device_status() == ops.DEV_BAD_OFFSETS
    assert bool((out == 7.0).all()), "nothing may be written for malformed offsets"


@pytest.mark.parametrize("dgrad", [False, True])
def test_grouped_at_the_expert_limit(dgrad):
    # 1024 experts (the most the kernels accept), most of them empty or tiny: every row of the
    # non-empty experts is checked, and each expert's tile list is only its own rows.
    E, N, K = 1024, 256, 256
    g = np.random.Generator(np.random.PCG64(1024))
    counts = np.where(g.random(E) < 0.8, 0, g.integers(1, 200, size=E))
    counts[[0, E - 1]] = [3, 129]
    off = np.zeros(E + 1, dtype=np.int32)
    off[1:] = np.cumsum(counts)
    Mtot = int(off[-1])
    pool_w = [oracle.quant_128x128(synth.weights(N, K, seed=900 + p)) for p in range(4)]
    bq = np.stack([pool_w[e % 4][0] for e in range(E)])
    bs = np.stack([pool_w[e % 4][1] * np.float32(1 + (e % 7) / 8) for e in range(E)]).astype(np.float32)
    A = synth.activations_channel_outliers(Mtot, K, seed=1025)
    aq, as_ = oracle.quant_1x128(A)
    out = torch.full((Mtot, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    offs = torch.from_numpy(off).cuda()
    if dgrad:
        ops.grouped_gemm_blockscaled_dgrad(u8_dev(aq), f32_dev(as_), u8_dev(bq), f32_dev(bs), offs, out=out)
    else:
        ops.grouped_gemm_blockscaled(u8_dev(aq), f32_dev(as_), u8_dev(bq), f32_dev(bs), offs, out=out)
    assert ops.device_status() == ops.DEV_OK
    got = host(out)
    mode = ops.DGRAD if dgrad else ops.FPROP
    for e in np.flatnonzero(counts):
        r0, r1 = int(off[e]), int(off[e + 1])
        ref, S = oracle.gemm(mode, aq[r0:r1], np.ascontiguousarray(as_[:, r0:r1]), bq[e], bs[e])
        check_gemm(got[r0:r1], ref, S, f"expert {e} of {E} ({r1 - r0} rows, {'dgrad' if dgrad else 'fprop'})")


@pytest.mark.parametrize("bad", ["nonzero_start", "decreasing", "wrong_total"])
def test_grouped_bad_offsets_are_reported_and_nothing_written(bad):
    N, K = 128, 256
    aq, as_, bq, bs, off = small_problem([100, 60, 40], N, K, seed=9)
    off = off.copy()
    if bad == "nonzero_start":
        off[0] = 4
    elif bad == "decreasing":
        off[1], off[2] = off[2], off[1]
    else:
        off[-1] -= 1
    got, status = run_grouped(aq, as_, bq, bs, off)
    assert status == ops.DEV_BAD_OFFSETS
    assert np.all(np.isnan(got)), "a rejected call must not write the output"
    # The status word is cleared by the read, and a good call afterwards succeeds.
    aq, as_, bq, bs, off = small_problem([100, 60, 40], N, K, seed=9)
    got, status = run_grouped(aq, as_, bq, bs, off)
    assert status == ops.DEV_OK and np.all(np.isfinite(got))


def test_timeout_path_latches_status_and_context_survives():
    ops.selftest_wait_timeout(10_000_000)            # 10 ms wait on a barrier nobody completes
    assert ops.device_status() == ops.DEV_TIMEOUT
    assert ops.device_status() == ops.DEV_OK         # cleared by the read
    x = torch.ones((4, 128), dtype=torch.bfloat16, device="cuda")
    q, s = ops.act_1x128(x)
    torch.cuda.synchronize()
    assert int(q[0, 0]) == 0x7E and ops.device_status() == ops.DEV_OK


def test_full_size_moe_grouped():
    E, N, K, tokens = 256, 2048, 7168, 8192
    expert_of, counts = synth.moe_routing(tokens=tokens, experts=E)
    token_idx, off = synth.moe_grouped_rows(expert_of, E)
    assert (counts == 0).sum() >= 1 and counts.sum() == tokens * 8
    # Activations: quantise the 8192 distinct token rows once (1x128 groups are per row), then
    # gather codes and scales into expert order.
    X = synth.activations_channel_outliers(tokens, K, seed=synth.SEED_BASE + 4)
    xq, xs = oracle.quant_1x128(X)
    aq = xq[token_idx]
    as_ = np.ascontiguousarray(xs[:, token_idx])
    # Expert weights: 8 distinct quantised matrices, reused across experts, with each expert's
    # block scales multiplied by its own seeded factor so every expert's weight differs.
    pool = [oracle.quant_128x128(synth.expert_weights(p, N, K)) for p in range(8)]
    g = np.random.Generator(np.random.PCG64(77))
    factor = g.uniform(0.5, 2.0, size=E).astype(np.float32)
    bs = np.stack([pool[e % 8][1] * factor[e] for e in range(E)]).astype(np.float32)
    pool_dev = torch.stack([u8_dev(pool[p][0]) for p in range(8)])
    bq_dev = pool_dev[torch.arange(E) % 8].contiguous()          # [E, N, K] on the device
    del pool_dev
    out = torch.full((aq.shape[0], N), float("nan"), dtype=torch.bfloat16, device="cuda")
    ops.grouped_gemm_blockscaled(u8_dev(aq), f32_dev(as_), bq_dev, f32_dev(bs),
                                 torch.from_numpy(off).cuda(), out=out)
    assert ops.device_status() == ops.DEV_OK
    assert bool(torch.isfinite(out).all()), "every routed row must be written"
    got = host(out)
    nonempty = np.flatnonzero(counts > 0)
    pick = {int(np.argmax(counts)), int(nonempty[np.argmin(counts[nonempty])])}
    pick |= set(int(e) for e in g.choice(nonempty, size=6, replace=False))
    for e in sorted(pick):
        r0, r1 = int(off[e]), int(off[e + 1])
        rows = np.unique(np.concatenate([[r0, r1 - 1], g.integers(r0, r1, size=6)]))
        ms = np.repeat(rows - r0, N)
        ns = np.tile(np.arange(N), rows.size)
        ref, S = oracle.gemm_entries(ops.FPROP, aq[r0:r1], np.ascontiguousarray(as_[:, r0:r1]),
                                     pool[e % 8][0], bs[e], ms, ns)
        check_gemm(got[rows].reshape(-1), ref, S, f"expert {e} ({r1 - r0} rows)")

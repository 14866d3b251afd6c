"""GPU power-of-two (UE8M0) scale variant vs the oracle.

* Quantisers with scale_fmt="ue8m0" (1x128, 128x1 transposed, both forms in one pass, the fused
  forward operands, 128x128 with its transposed codes): codes and scales bit for bit.
* The block-scaled-MMA GEMM (fp8_gemm_blockscaled_ue8m0, tcgen05 kind::mxf8f6f4): exact dyadic
  cases bit for bit; realistic operands over ragged shapes, both tile widths and both schedules
  within the GEMM tolerance; Wgrad accumulation; full-size shapes sampled, run twice (bitwise
  identical); a scale that is not a power of two latches DEV_BAD_SCALES.
The GEMM operands are always quantised by the oracle on the host, never by the GPU.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_fine_grained_fp8q_b200 import ops, synth
from tests._util import bf16_dev, check_gemm, f32_dev, host, linear_layer_inputs, u8_dev

pytestmark = pytest.mark.gpu

FPROP, DGRAD, WGRAD, WGRAD_ACC = ops.FPROP, ops.DGRAD, ops.WGRAD, ops.WGRAD_ACC
UE = "ue8m0"
CONFIGS = {"n128-dp": ("128", "dp"), "n256-dp": ("256", "dp"),
           "n128-sk": ("128", "sk"), "n256-sk": ("256", "sk")}


def set_config(monkeypatch, cfg):
    bn, sched = CONFIGS[cfg]
    monkeypatch.setenv("FP8Q_GEMM_BN", bn)
    monkeypatch.setenv("FP8Q_GEMM_SCHED", sched)


def same_f32(a, b):
    return np.array_equal(np.asarray(a, np.float32).view(np.uint32), np.asarray(b, np.float32).view(np.uint32))


# ------------------------------------------------------------------------------------------ #
# Quantisers
# ------------------------------------------------------------------------------------------ #

@pytest.mark.parametrize("M,K", [(256, 512), (130, 384), (1, 128), (1000, 1024)])
def test_act_1x128(M, K):
    x = synth.activations_entry_outliers(M, K, seed=M + K + 500)
    q, s = ops.act_1x128(bf16_dev(x), scale_fmt=UE)
    oq, os_ = oracle.quant_1x128(x, scale_fmt=UE)
    assert np.array_equal(host(q), oq) and same_f32(host(s), os_)


@pytest.mark.parametrize("T,C", [(256, 192), (128, 64), (640, 512)])
def test_act_128x1_transposed(T, C):
    x = synth.output_grad(T, C, seed=T + C + 501)
    qt, s = ops.act_128x1_transposed(bf16_dev(x), scale_fmt=UE)
    oq, os_ = oracle.quant_128x1_t(x, scale_fmt=UE)
    assert np.array_equal(host(qt), oq) and same_f32(host(s), os_)


@pytest.mark.parametrize("T,C", [(256, 384), (512, 1024)])
def test_act_dual(T, C):
    x = synth.activations_channel_outliers(T, C, seed=T + C + 502)
    q, s, qt, st = ops.act_dual(bf16_dev(x), scale_fmt=UE)
    oq, os_ = oracle.quant_1x128(x, scale_fmt=UE)
    oqt, ost = oracle.quant_128x1_t(x, scale_fmt=UE)
    assert np.array_equal(host(q), oq) and same_f32(host(s), os_)
    assert np.array_equal(host(qt), oqt) and same_f32(host(st), ost)


def test_quant_forward_and_weight():
    x = synth.activations_channel_outliers(384, 512, seed=503)
    w = synth.weights(256, 512, seed=504)
    (xq, xs, xqt, xst), (wq, ws, wqt) = ops.quant_forward(bf16_dev(x), bf16_dev(w), transposed_w=True,
                                                          scale_fmt=UE)
    oq, os_ = oracle.quant_1x128(x, scale_fmt=UE)
    oqt, ost = oracle.quant_128x1_t(x, scale_fmt=UE)
    owq, ows, owqt = oracle.quant_128x128(w, want_transposed=True, scale_fmt=UE)
    assert np.array_equal(host(xq), oq) and same_f32(host(xs), os_)
    assert np.array_equal(host(xqt), oqt) and same_f32(host(xst), ost)
    assert np.array_equal(host(wq), owq) and same_f32(host(ws), ows) and np.array_equal(host(wqt), owqt)
    q2, s2, qt2 = ops.weight_128x128(bf16_dev(w), transposed=True, scale_fmt=UE)
    assert torch.equal(q2, wq) and torch.equal(s2, ws) and torch.equal(qt2, wqt)


def test_zero_input_takes_the_floor_scale():
    x = np.zeros((128, 256), dtype=np.uint16)
    q, s = ops.act_1x128(bf16_dev(x), scale_fmt=UE)
    assert not host(q).any() and np.all(host(s) == np.float32(2.0 ** -108))


def test_unknown_format_is_rejected():
    with pytest.raises(ValueError):
        ops.act_1x128(bf16_dev(np.zeros((1, 128), np.uint16)), scale_fmt="e5m2")


# ------------------------------------------------------------------------------------------ #
# GEMM
# ------------------------------------------------------------------------------------------ #

def run(mode, A, sA, B, sB, cfg=None, monkeypatch=None, out=None):
    if cfg is not None:
        set_config(monkeypatch, cfg)
    M = A.shape[0]
    N = B.shape[1] if mode == DGRAD else B.shape[0]
    if out is None:
        dtype = torch.float32 if mode in (WGRAD, WGRAD_ACC) else torch.bfloat16
        out = torch.full((M, N), float("nan"), dtype=dtype, device="cuda")
    ops.gemm_blockscaled_ue8m0(mode, u8_dev(A), f32_dev(sA), u8_dev(B), f32_dev(sB), out=out)
    assert ops.device_status() == ops.DEV_OK
    return host(out)


def _ternary(g, shape, density=0.25):
    v = g.integers(-1, 2, size=shape).astype(np.float32)
    return v * (g.random(shape) < density)


@pytest.mark.parametrize("cfg", list(CONFIGS))
@pytest.mark.parametrize("M,N,K", [(200, 512, 384), (1, 256, 128), (384, 256, 1024)])
def test_exact_fprop(M, N, K, cfg, monkeypatch):
    # Every group's max-abs is 448 * 2^j: the power-of-two scales are 2^j, the products exact,
    # and the sums small integers times powers of two, representable in bf16.
    g = np.random.Generator(np.random.PCG64(M + N + K + 510))
    X, W = _ternary(g, (M, K)), _ternary(g, (N, K))
    X[:, 1::128] = 0.0
    W[:, 0::128] = 0.0
    X[:, 0::128] = 448.0 * np.where(g.random((M, K // 128)) < 0.5, -1, 1)
    for nb in range(N // 128):
        W[nb * 128, 1::128] = 448.0
    X *= np.exp2(g.integers(-4, 5, size=M))[:, None].astype(np.float32)
    W *= np.exp2(np.repeat(g.integers(-4, 5, size=N // 128), 128))[:, None].astype(np.float32)
    exact = X.astype(np.float64) @ W.astype(np.float64).T
    xq, xs = oracle.quant_1x128(synth.f32_to_bf16_bits(X), scale_fmt=UE)
    wq, ws, _ = oracle.quant_128x128(synth.f32_to_bf16_bits(W), scale_fmt=UE)
    assert np.array_equal(oracle.gemm(FPROP, xq, xs, wq, ws)[0], exact)
    assert np.array_equal(run(FPROP, xq, xs, wq, ws, cfg, monkeypatch), exact)


@pytest.mark.parametrize("cfg", list(CONFIGS))
def test_exact_wgrad_and_accumulate(cfg, monkeypatch):
    T, Cout, Cin = 512, 384, 512
    g = np.random.Generator(np.random.PCG64(511))
    dY = g.integers(-8, 9, size=(T, Cout)).astype(np.float32)
    X = g.integers(-8, 9, size=(T, Cin)).astype(np.float32)
    dY[1::128, :] = 0.0
    X[0::128, :] = 0.0
    dY[0::128, :] = 448.0
    X[1::128, :] = -448.0
    dY *= np.exp2(g.integers(-4, 5, size=Cout))[None, :].astype(np.float32)
    X *= np.exp2(g.integers(-4, 5, size=Cin))[None, :].astype(np.float32)
    P = dY.astype(np.float64).T @ X.astype(np.float64)
    assert np.array_equal(P.astype(np.float32).astype(np.float64), P)
    gq, gs = oracle.quant_128x1_t(synth.f32_to_bf16_bits(dY), scale_fmt=UE)
    xq, xs = oracle.quant_128x1_t(synth.f32_to_bf16_bits(X), scale_fmt=UE)
    assert np.array_equal(run(WGRAD, gq, gs, xq, xs, cfg, monkeypatch), P)
    D = torch.from_numpy(P.astype(np.float32)).cuda()
    assert np.array_equal(run(WGRAD_ACC, gq, gs, xq, xs, out=D), 2.0 * P)


@pytest.mark.parametrize("cfg", list(CONFIGS))
@pytest.mark.parametrize("M,N,K", [(200, 256, 384), (517, 512, 1024), (1, 256, 256)])
def test_fprop(M, N, K, cfg, monkeypatch):
    X = synth.activations_channel_outliers(M, K, seed=M + K + 520)
    W = synth.weights(N, K, seed=N + K + 521)
    xq, xs = oracle.quant_1x128(X, scale_fmt=UE)
    wq, ws, _ = oracle.quant_128x128(W, scale_fmt=UE)
    ref, S = oracle.gemm(FPROP, xq, xs, wq, ws)
    check_gemm(run(FPROP, xq, xs, wq, ws, cfg, monkeypatch), ref, S, f"ue8m0 fprop {M}x{N}x{K}")


@pytest.mark.parametrize("cfg", list(CONFIGS))
@pytest.mark.parametrize("M,N,K", [(256, 512, 256), (333, 768, 640)])
def test_dgrad(M, N, K, cfg, monkeypatch):
    dY = synth.output_grad(M, K, seed=M + K + 522)
    W = synth.weights(K, N, seed=N + K + 523)
    gq, gs = oracle.quant_1x128(dY, scale_fmt=UE)
    wq, ws, _ = oracle.quant_128x128(W, scale_fmt=UE)
    ref, S = oracle.gemm(DGRAD, gq, gs, wq, ws)
    check_gemm(run(DGRAD, gq, gs, wq, ws, cfg, monkeypatch), ref, S, f"ue8m0 dgrad {M}x{N}x{K}")


@pytest.mark.parametrize("cfg", list(CONFIGS))
@pytest.mark.parametrize("T,Cout,Cin", [(512, 256, 512), (384, 384, 768)])
def test_wgrad(T, Cout, Cin, cfg, monkeypatch):
    dY = synth.output_grad(T, Cout, seed=T + Cout + 524)
    X = synth.activations_channel_outliers(T, Cin, seed=T + Cin + 525)
    gq, gs = oracle.quant_128x1_t(dY, scale_fmt=UE)
    xq, xs = oracle.quant_128x1_t(X, scale_fmt=UE)
    ref, S = oracle.gemm(WGRAD, gq, gs, xq, xs)
    check_gemm(run(WGRAD, gq, gs, xq, xs, cfg, monkeypatch), ref, S, f"ue8m0 wgrad {T}x{Cout}x{Cin}",
               bf16_out=False)
    D0 = np.random.Generator(np.random.PCG64(526)).standard_normal((Cout, Cin)).astype(np.float32) * 1e-3
    got = run(WGRAD_ACC, gq, gs, xq, xs, out=torch.from_numpy(D0).cuda())
    check_gemm(got, D0.astype(np.float64) + ref, S, "ue8m0 wgrad accumulate", bf16_out=False)


def test_non_power_of_two_scales_latch_bad_scales():
    X = synth.activations_channel_outliers(256, 256, seed=527)
    W = synth.weights(256, 256, seed=528)
    xq, xs = oracle.quant_1x128(X)                 # max-abs scales: not powers of two
    wq, ws, _ = oracle.quant_128x128(W, scale_fmt=UE)
    out = torch.empty((256, 256), dtype=torch.bfloat16, device="cuda")
    ops.gemm_blockscaled_ue8m0(FPROP, u8_dev(xq), f32_dev(xs), u8_dev(wq), f32_dev(ws), out=out)
    assert ops.device_status() == ops.DEV_BAD_SCALES
    assert ops.device_status() == ops.DEV_OK       # read and cleared


# ------------------------------------------------------------------------------------------ #
# Full-size shapes
# ------------------------------------------------------------------------------------------ #

_q = {}


def quantised_layer():
    if not _q:
        d = linear_layer_inputs()
        _q["X"] = oracle.quant_1x128(d["X"], scale_fmt=UE)
        _q["dY"] = oracle.quant_1x128(d["dY"], scale_fmt=UE)
        _q["W"] = oracle.quant_128x128(d["W"], scale_fmt=UE)[:2]
        _q["Xt"] = oracle.quant_128x1_t(d["X"], scale_fmt=UE)
        _q["dYt"] = oracle.quant_128x1_t(d["dY"], scale_fmt=UE)
    return _q


_ref = {}


def full_check(mode, A, sA, B, sB, got, what):
    """Every entry of a full-size result against the oracle (its exact D and S are computed once
    per mode and shared by the configurations)."""
    if mode not in _ref:
        _ref[mode] = oracle.gemm(mode, A, sA, B, sB)
    ref, S = _ref[mode]
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), f"{what}: unwritten or non-finite outputs"
    return check_gemm(got, ref, S, what, bf16_out=(mode != WGRAD))


@pytest.mark.parametrize("cfg", ["n256-sk", "n256-dp", "n128-sk"])
@pytest.mark.parametrize("mode", [FPROP, DGRAD, WGRAD])
def test_full_size_deterministic_and_within_tolerance(mode, cfg, monkeypatch):
    q = quantised_layer()
    (a, sa), (b, sb) = {FPROP: (q["X"], q["W"]), DGRAD: (q["dY"], q["W"]), WGRAD: (q["dYt"], q["Xt"])}[mode]
    A, SA, B, SB = u8_dev(a), f32_dev(sa), u8_dev(b), f32_dev(sb)
    set_config(monkeypatch, cfg)
    first = ops.gemm_blockscaled_ue8m0(mode, A, SA, B, SB).clone()
    second = ops.gemm_blockscaled_ue8m0(mode, A, SA, B, SB)
    assert ops.device_status() == ops.DEV_OK
    assert torch.equal(first, second)
    full_check(mode, a, sa, b, sb, host(first), f"ue8m0 mode {mode} {cfg}")

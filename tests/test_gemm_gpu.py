"""GPU block-scaled FP8 GEMM vs the CPU oracle (Fprop, Dgrad, Wgrad).

* Exact cases: dyadic operands whose groups have power-of-two scales and whose products
  cancel nowhere but sum to small integers times powers of two; the exact result is
  representable in the output type, so any correct kernel returns it bit for bit.
* Tolerance cases: realistic operands (oracle-quantised synthetic activations, weights and
  gradients) over several tiles with ragged row counts, both tile widths, full outputs.
* Full-size cases, the shapes the benchmark times: sampled rows, columns and entries.
The quantised operands are always produced by the oracle on the host, never by the GPU.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_fine_grained_fp8q_b200 import ops, synth
from tests._util import check_gemm, f32_dev, host, linear_layer_inputs, u8_dev

pytestmark = pytest.mark.gpu

FPROP, DGRAD, WGRAD, WGRAD_ACC = ops.FPROP, ops.DGRAD, ops.WGRAD, ops.WGRAD_ACC


# Kernel configurations: tile width x schedule (data-parallel whole tiles, or stream-K over
# (tile, 128-K group) units with partials combined through the workspace).
CONFIGS = {"n128-dp": ("128", "dp"), "n256-dp": ("256", "dp"),
           "n128-sk": ("128", "sk"), "n256-sk": ("256", "sk")}


def set_config(monkeypatch, cfg):
    bn, sched = CONFIGS[cfg]
    monkeypatch.setenv("FP8Q_GEMM_BN", bn)
    monkeypatch.setenv("FP8Q_GEMM_SCHED", sched)


def run_gemm(mode, A, sA, B, sB, bn=None, monkeypatch=None):
    if bn is not None:
        set_config(monkeypatch, bn)
    M = A.shape[0]
    N = B.shape[1] if mode == DGRAD else B.shape[0]
    dtype = torch.float32 if mode == WGRAD else torch.bfloat16
    out = torch.full((M, N), float("nan"), dtype=dtype, device="cuda")
    ops.gemm_blockscaled(mode, u8_dev(A), f32_dev(sA), u8_dev(B), f32_dev(sB), out=out)
    assert ops.device_status() == ops.DEV_OK
    return host(out)


# ------------------------------------------------------------------------------------------ #
# Exact dyadic cases
# ------------------------------------------------------------------------------------------ #

def _ternary(g, shape, density=0.25):
    v = g.integers(-1, 2, size=shape).astype(np.float32)
    return v * (g.random(shape) < density)


def _bits(x):
    return synth.f32_to_bf16_bits(x)


def exact_fprop(M, N, K, seed):
    g = np.random.Generator(np.random.PCG64(seed))
    jx = g.integers(-4, 5, size=M)
    jw = g.integers(-4, 5, size=N // 128)
    X = _ternary(g, (M, K))
    W = _ternary(g, (N, K))
    X[:, 1::128] = 0.0
    W[:, 0::128] = 0.0
    X[:, 0::128] = 448.0 * np.where(g.random((M, K // 128)) < 0.5, -1, 1)
    for nb in range(N // 128):
        W[nb * 128, 1::128] = 448.0
    X *= np.exp2(jx)[:, None].astype(np.float32)
    W *= np.exp2(np.repeat(jw, 128))[:, None].astype(np.float32)
    exact = X.astype(np.float64) @ W.astype(np.float64).T
    return X, W, exact


@pytest.mark.parametrize("bn", list(CONFIGS))
@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (200, 512, 384), (1, 256, 128), (384, 256, 1024)])
def test_exact_fprop(M, N, K, bn, monkeypatch):
    X, W, exact = exact_fprop(M, N, K, seed=M + N + K)
    # Representable in bf16: integers of magnitude <= 256 times a power of two.
    ints = exact / np.exp2(np.floor(np.log2(np.maximum(np.abs(exact), 1e-300))) - 7)
    assert np.all((exact == 0) | (np.abs(ints - np.round(ints)) == 0))
    xq, xs = oracle.quant_1x128(_bits(X))
    wq, ws, _ = oracle.quant_128x128(_bits(W))
    ref, _ = oracle.gemm(FPROP, xq, xs, wq, ws)
    assert np.array_equal(ref, exact)
    got = run_gemm(FPROP, xq, xs, wq, ws, bn, monkeypatch)
    assert np.array_equal(got, exact)


@pytest.mark.parametrize("bn", list(CONFIGS))
@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (260, 512, 384)])
def test_exact_dgrad(M, N, K, bn, monkeypatch):
    # dX[M,N] = dY[M,K] W[K,N]; W is the forward weight [out=K, in=N].
    g = np.random.Generator(np.random.PCG64(M * N + K))
    jy = g.integers(-4, 5, size=M)
    jw = g.integers(-4, 5, size=N // 128)
    dY = _ternary(g, (M, K))
    W = _ternary(g, (K, N))
    dY[:, 1::128] = 0.0
    W[0::128, :] = 0.0
    dY[:, 0::128] = 448.0
    for nb in range(N // 128):
        W[1::128, nb * 128] = -448.0
    dY *= np.exp2(jy)[:, None].astype(np.float32)
    W *= np.exp2(np.repeat(jw, 128))[None, :].astype(np.float32)
    exact = dY.astype(np.float64) @ W.astype(np.float64)
    gq, gs = oracle.quant_1x128(_bits(dY))
    wq, ws, _ = oracle.quant_128x128(_bits(W))
    got = run_gemm(DGRAD, gq, gs, wq, ws, bn, monkeypatch)
    assert np.array_equal(got, exact)


@pytest.mark.parametrize("bn", list(CONFIGS))
@pytest.mark.parametrize("T,Cout,Cin", [(128, 128, 256), (512, 384, 512)])
def test_exact_wgrad(T, Cout, Cin, bn, monkeypatch):
    # dW[Cout,Cin] = dY[T,Cout]^T X[T,Cin]; FP32 output, so larger sums stay exact.
    g = np.random.Generator(np.random.PCG64(T + Cout * Cin))
    jy = g.integers(-4, 5, size=Cout)
    jx = g.integers(-4, 5, size=Cin)
    dY = g.integers(-8, 9, size=(T, Cout)).astype(np.float32)
    X = g.integers(-8, 9, size=(T, Cin)).astype(np.float32)
    dY[1::128, :] = 0.0
    X[0::128, :] = 0.0
    dY[0::128, :] = 448.0
    X[1::128, :] = -448.0
    dY *= np.exp2(jy)[None, :].astype(np.float32)
    X *= np.exp2(jx)[None, :].astype(np.float32)
    exact = dY.astype(np.float64).T @ X.astype(np.float64)
    gq, gs = oracle.quant_128x1_t(_bits(dY))
    xq, xs = oracle.quant_128x1_t(_bits(X))
    got = run_gemm(WGRAD, gq, gs, xq, xs, bn, monkeypatch)
    assert np.array_equal(got, exact)


def run_wgrad_acc(A, sA, B, sB, D0, times, bn=None, monkeypatch=None):
    """D0 (fp32 [M, N]) plus `times` accumulating Wgrad calls."""
    if bn is not None:
        set_config(monkeypatch, bn)
    D = torch.from_numpy(np.ascontiguousarray(D0, dtype=np.float32)).cuda()
    for _ in range(times):
        ops.gemm_blockscaled(WGRAD_ACC, u8_dev(A), f32_dev(sA), u8_dev(B), f32_dev(sB), out=D)
    torch.cuda.synchronize()
    assert ops.device_status() == ops.DEV_OK
    return host(D).astype(np.float64)


@pytest.mark.parametrize("bn", list(CONFIGS))
def test_exact_wgrad_accumulate(bn, monkeypatch):
    # Operands whose product P = dY^T X is exact in FP32 (as in test_exact_wgrad, where the plain
    # mode must return P bit for bit).  Accumulating into D0 = P must give 2P, into D0 = -P zero:
    # both sums are exact, so both are bit-exact checks of "D += P".
    T, Cout, Cin = 512, 384, 512
    g = np.random.Generator(np.random.PCG64(T + Cout * Cin))
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
    gq, gs = oracle.quant_128x1_t(_bits(dY))
    xq, xs = oracle.quant_128x1_t(_bits(X))
    assert np.array_equal(run_wgrad_acc(gq, gs, xq, xs, P, 1, bn, monkeypatch), 2.0 * P)
    assert np.array_equal(run_wgrad_acc(gq, gs, xq, xs, -P, 1, bn, monkeypatch), np.zeros_like(P))


@pytest.mark.parametrize("bn", list(CONFIGS))
def test_wgrad_accumulate_within_tolerance(bn, monkeypatch):
    T, Cout, Cin = 384, 384, 768
    dY = synth.output_grad(T, Cout, seed=71)
    X = synth.activations_channel_outliers(T, Cin, seed=72)
    gq, gs = oracle.quant_128x1_t(dY)
    xq, xs = oracle.quant_128x1_t(X)
    ref, S = oracle.gemm(WGRAD, gq, gs, xq, xs)
    D0 = np.random.Generator(np.random.PCG64(73)).standard_normal((Cout, Cin)).astype(np.float32) * 1e-3
    got = run_wgrad_acc(gq, gs, xq, xs, D0, 1, bn, monkeypatch)
    check_gemm(got, D0.astype(np.float64) + ref, S, f"wgrad accumulate {T}x{Cout}x{Cin}", bf16_out=False)


def test_wgrad_accumulate_rejects_missing_out():
    with pytest.raises(ValueError):
        ops.gemm_blockscaled(WGRAD_ACC, *(torch.zeros(1, device="cuda"),) * 4)


def check_gemm_quant(mode, A, sA, B, sB, what, monkeypatch=None, bn=None):
    """D within the GEMM tolerance, and (q, s) bit-exact against the oracle's 1x128 quantiser
    applied to the bf16 D this call returned; the same call without storing D gives the same
    codes and scales."""
    if bn is not None:
        set_config(monkeypatch, bn)
    args = (u8_dev(A), f32_dev(sA), u8_dev(B), f32_dev(sB))
    D, q, s = ops.gemm_blockscaled_quant(mode, *args)
    torch.cuda.synchronize()
    assert ops.device_status() == ops.DEV_OK
    d_bits = D.view(torch.int16).cpu().numpy().view(np.uint16)
    ref, S = oracle.gemm(mode, A, sA, B, sB)
    check_gemm(host(D).astype(np.float64), ref, S, what)
    oq, os_ = oracle.quant_1x128(d_bits)
    assert np.array_equal(host(q), oq), f"{what}: codes differ from the 1x128 quantiser of D"
    assert np.array_equal(host(s).view(np.uint32), os_.view(np.uint32)), f"{what}: scales differ"
    if B.shape[1 if mode == DGRAD else 0] % 256 == 0 and bn in (None, "n256-dp", "n256-sk"):
        _, q2, s2 = ops.gemm_blockscaled_quant(mode, *args, store_out=False)
        torch.cuda.synchronize()
        assert torch.equal(q2, q) and torch.equal(s2, s), f"{what}: store_out=False changed the codes"


@pytest.mark.parametrize("bn", list(CONFIGS))
@pytest.mark.parametrize("M,N,K", [(256, 512, 512), (300, 768, 1024)])
def test_fprop_fused_output_quant(M, N, K, bn, monkeypatch):
    X = synth.activations_entry_outliers(M, K, seed=M + 5)
    W = synth.weights(N, K, seed=N + 6)
    xq, xs = oracle.quant_1x128(X)
    wq, ws, _ = oracle.quant_128x128(W)
    check_gemm_quant(FPROP, xq, xs, wq, ws, f"fprop+quant {M}x{N}x{K}", monkeypatch, bn)


@pytest.mark.parametrize("bn", list(CONFIGS))
def test_dgrad_fused_output_quant(bn, monkeypatch):
    M, N, K = 384, 640, 512                      # N = 640: 256-wide tiles do not fit (fallback path)
    dY = synth.output_grad(M, K, seed=81)
    W = synth.weights(K, N, seed=82)
    gq, gs = oracle.quant_1x128(dY)
    wq, ws, _ = oracle.quant_128x128(W)
    check_gemm_quant(DGRAD, gq, gs, wq, ws, f"dgrad+quant {M}x{N}x{K}", monkeypatch, bn)


def test_full_fprop_fused_output_quant():
    q = quantised_layer()
    (xq, xs), (wq, ws) = q["X"], q["W"]
    args = (u8_dev(xq), f32_dev(xs), u8_dev(wq), f32_dev(ws))
    D, qd, sd = ops.gemm_blockscaled_quant(FPROP, *args)
    plain = ops.gemm_blockscaled(FPROP, *args)
    torch.cuda.synchronize()
    assert torch.equal(D, plain), "the fused epilogue changed the bf16 output"
    oq, os_ = oracle.quant_1x128(D.view(torch.int16).cpu().numpy().view(np.uint16))
    assert np.array_equal(host(qd), oq) and np.array_equal(host(sd).view(np.uint32), os_.view(np.uint32))


# ------------------------------------------------------------------------------------------ #
# Tolerance cases, full outputs
# ------------------------------------------------------------------------------------------ #

def test_tiny_fprop_workload():
    d = synth.tiny_fprop()
    xq, xs = oracle.quant_1x128(d["X"])
    wq, ws, _ = oracle.quant_128x128(d["W"])
    ref, S = oracle.gemm(FPROP, xq, xs, wq, ws)
    got = run_gemm(FPROP, xq, xs, wq, ws)
    check_gemm(got, ref, S, "tiny fprop 256x512x512")


@pytest.mark.parametrize("bn", list(CONFIGS))
@pytest.mark.parametrize("M,N,K", [(200, 256, 384), (517, 512, 1024), (1, 256, 256)])
def test_fprop_ragged(M, N, K, bn, monkeypatch):
    X = synth.activations_channel_outliers(M, K, seed=M + K)
    W = synth.weights(N, K, seed=N + K + 1)
    xq, xs = oracle.quant_1x128(X)
    wq, ws, _ = oracle.quant_128x128(W)
    ref, S = oracle.gemm(FPROP, xq, xs, wq, ws)
    check_gemm(run_gemm(FPROP, xq, xs, wq, ws, bn, monkeypatch), ref, S, f"fprop {M}x{N}x{K}")


@pytest.mark.parametrize("bn", list(CONFIGS))
@pytest.mark.parametrize("M,N,K", [(256, 512, 256), (333, 768, 640)])
def test_dgrad_ragged(M, N, K, bn, monkeypatch):
    dY = synth.output_grad(M, K, seed=M + K)
    W = synth.weights(K, N, seed=N + K + 2)
    gq, gs = oracle.quant_1x128(dY)
    wq, ws, _ = oracle.quant_128x128(W)
    ref, S = oracle.gemm(DGRAD, gq, gs, wq, ws)
    check_gemm(run_gemm(DGRAD, gq, gs, wq, ws, bn, monkeypatch), ref, S, f"dgrad {M}x{N}x{K}")


@pytest.mark.parametrize("bn", list(CONFIGS))
@pytest.mark.parametrize("T,Cout,Cin", [(512, 256, 512), (384, 384, 768)])
def test_wgrad(T, Cout, Cin, bn, monkeypatch):
    dY = synth.output_grad(T, Cout, seed=T + Cout)
    X = synth.activations_channel_outliers(T, Cin, seed=T + Cin + 3)
    gq, gs = oracle.quant_128x1_t(dY)
    xq, xs = oracle.quant_128x1_t(X)
    ref, S = oracle.gemm(WGRAD, gq, gs, xq, xs)
    check_gemm(run_gemm(WGRAD, gq, gs, xq, xs, bn, monkeypatch), ref, S, f"wgrad {T}x{Cout}x{Cin}",
               bf16_out=False)


def test_empty_rows_is_a_no_op():
    A = torch.zeros((0, 256), dtype=torch.uint8, device="cuda")
    sA = torch.zeros((2, 0), dtype=torch.float32, device="cuda")
    B = torch.zeros((128, 256), dtype=torch.uint8, device="cuda")
    sB = torch.ones((1, 2), dtype=torch.float32, device="cuda")
    out = ops.gemm_blockscaled(FPROP, A, sA, B, sB)
    assert out.shape == (0, 128)


# ------------------------------------------------------------------------------------------ #
# Full-size shapes (every output entry against the oracle)
# ------------------------------------------------------------------------------------------ #

_q = {}
_ref = {}


def quantised_layer():
    if not _q:
        d = linear_layer_inputs()
        _q["X"] = oracle.quant_1x128(d["X"])
        _q["dY"] = oracle.quant_1x128(d["dY"])
        _q["W"] = oracle.quant_128x128(d["W"])[:2]
        _q["Xt"] = oracle.quant_128x1_t(d["X"])
        _q["dYt"] = oracle.quant_128x1_t(d["dY"])
    return _q


def full_reference(key, mode, A, sA, B, sB):
    """The oracle's exact D and S of a full-size problem, computed once per key (a few seconds
    on the host's cores) and shared by every test of that problem."""
    if key not in _ref:
        _ref[key] = oracle.gemm(mode, A, sA, B, sB)
    return _ref[key]


def full_check(key, mode, A, sA, B, sB, got, what):
    """Every entry of a full-size result against the oracle."""
    ref, S = full_reference(key, mode, A, sA, B, sB)
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), f"{what}: unwritten or non-finite outputs"
    return check_gemm(got, ref, S, what, bf16_out=(mode != WGRAD))


def test_full_fprop_ffn_up():
    q = quantised_layer()
    (xq, xs), (wq, ws) = q["X"], q["W"]
    got = run_gemm(FPROP, xq, xs, wq, ws)
    full_check("fprop", FPROP, xq, xs, wq, ws, got, "fprop 4096x2048x7168")


def test_full_dgrad():
    q = quantised_layer()
    (gq, gs), (wq, ws) = q["dY"], q["W"]
    got = run_gemm(DGRAD, gq, gs, wq, ws)
    assert got.shape == (4096, 7168)
    full_check("dgrad", DGRAD, gq, gs, wq, ws, got, "dgrad 4096x7168x2048")


def test_full_wgrad():
    q = quantised_layer()
    (gq, gs), (xq, xs) = q["dYt"], q["Xt"]
    got = run_gemm(WGRAD, gq, gs, xq, xs)
    assert got.shape == (2048, 7168)
    full_check("wgrad", WGRAD, gq, gs, xq, xs, got, "wgrad 2048x7168x4096")
    # Accumulating into zeros adds each result to 0 exactly: bit-identical to the overwrite.
    acc = run_wgrad_acc(gq, gs, xq, xs, np.zeros((2048, 7168), np.float32), 1)
    assert np.array_equal(acc, got.astype(np.float64))


@pytest.mark.parametrize("N", [1536, 512])
def test_full_fprop_mla(N):
    q = quantised_layer()
    xq, xs = q["X"]
    W = synth.weights(N, 7168, seed=synth.SEED_BASE + 3 + N)
    wq, ws, _ = oracle.quant_128x128(W)
    got = run_gemm(FPROP, xq, xs, wq, ws)
    full_check(f"fprop_mla{N}", FPROP, xq, xs, wq, ws, got, f"fprop MLA 4096x{N}x7168")


@pytest.mark.parametrize("cfg", list(CONFIGS))
@pytest.mark.parametrize("mode", [FPROP, DGRAD, WGRAD])
def test_full_size_every_config_deterministic_and_within_tolerance(mode, cfg, monkeypatch):
    """Each kernel configuration is run twice at full size: the launches must be bitwise
    identical (a race would show here -- e.g. a shared-memory buffer refilled by the async proxy
    while threads still read it, or a stream-K partial read before it is published), and every
    entry of the result must match the oracle."""
    q = quantised_layer()
    (a, sa), (b, sb) = {FPROP: (q["X"], q["W"]), DGRAD: (q["dY"], q["W"]),
                        WGRAD: (q["dYt"], q["Xt"])}[mode]
    A, SA, B, SB = u8_dev(a), f32_dev(sa), u8_dev(b), f32_dev(sb)
    set_config(monkeypatch, cfg)
    first = ops.gemm_blockscaled(mode, A, SA, B, SB).clone()
    second = ops.gemm_blockscaled(mode, A, SA, B, SB)
    assert ops.device_status() == ops.DEV_OK
    assert torch.equal(first, second)
    key = {FPROP: "fprop", DGRAD: "dgrad", WGRAD: "wgrad"}[mode]
    full_check(key, mode, a, sa, b, sb, host(first), f"mode {mode} {cfg}")


def test_two_streams_default_workspace(monkeypatch):
    """Two stream-K GEMMs queued on two streams at once through the default binding (no explicit
    workspace): each stream gets its own cached workspace, so neither overwrites the other's
    partial tiles; both results match the oracle."""
    monkeypatch.setenv("FP8Q_GEMM_SCHED", "sk")
    cases = []
    for seed in (61, 62):
        X = synth.activations_channel_outliers(1024, 2048, seed=seed)
        W = synth.weights(768, 2048, seed=seed + 100)
        xq, xs = oracle.quant_1x128(X)
        wq, ws, _ = oracle.quant_128x128(W)
        cases.append((xq, xs, wq, ws, u8_dev(xq), f32_dev(xs), u8_dev(wq), f32_dev(ws)))
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [None, None]
    torch.cuda.synchronize()
    for rep in range(3):
        for i, s in enumerate(streams):
            with torch.cuda.stream(s):
                *_, A, SA, B, SB = cases[i]
                outs[i] = ops.gemm_blockscaled(FPROP, A, SA, B, SB)
        torch.cuda.synchronize()
        assert ops.device_status() == ops.DEV_OK
        for i in range(2):
            xq, xs, wq, ws = cases[i][:4]
            ref, S = oracle.gemm(FPROP, xq, xs, wq, ws)
            check_gemm(host(outs[i]), ref, S, f"stream {i}, repetition {rep}")

"""Pins for the oracle's block-scaled GEMM (Fprop, Dgrad, Wgrad and grouped Fprop).

All three GEMMs of a linear layer run in FP8 (DeepSeek-V3 report repost, paragraph 2 and
Figure 6); the per-group scales along the inner dimension are applied at each 128-element
promotion into FP32 (repost paragraphs 1 and 4; "DeepSeek-V3 Technical Report" summary page,
FP8 bullet).  The exact value of that computation is the dot product of the dequantised
operands, which the oracle evaluates in binary64.

Pins:
* brute force with dyadic inputs whose groups have power-of-two scales: every step is exact,
  so the oracle must equal numpy's float64 matmul of the ORIGINAL (unquantised) values
  bit for bit, in every mode -- this catches a transposed operand, a wrong scale index or a
  dropped term;
* one-hot activations select rows / columns of the dequantised weight exactly;
* against the unquantised binary64 product, the error stays inside the elementwise bound
  implied by E4M3's rounding error (and the RMS relative error is reported);
* grouped Fprop equals integer matmuls per expert, empty experts included.
"""
import numpy as np
import pytest

import oracle
from fp8_fine_grained_fp8q_b200 import synth


def bits(x):
    return synth.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def f32(h):
    return synth.bf16_bits_to_f32(h)


def dyadic_groups(shape, group_of, seed):
    """Integers in [-16, 16] times 2^j, with j fixed per group and one +-448*2^j in each
    group, so every group's scale is exactly 2^j and every code decodes to the input."""
    g = np.random.Generator(np.random.PCG64(seed))
    x = g.integers(-16, 17, size=shape).astype(np.float64)
    gid = group_of(np.indices(shape))
    ngroups = int(gid.max()) + 1
    j = g.integers(-3, 4, size=ngroups)
    # Put +-448 at the first element (in C order) of each group.
    flat = gid.reshape(-1)
    _, first = np.unique(flat, return_index=True)
    signs = np.where(g.random(first.size) < 0.5, -1.0, 1.0)
    x.reshape(-1)[first] = 448.0 * signs
    x *= np.exp2(j[gid])
    return x.astype(np.float32)


def rows_1x128(M, K):
    return lambda ij: ij[0] * (K // 128) + ij[1] // 128


def cols_128x1(T, C):
    return lambda ij: (ij[0] // 128) * C + ij[1]


def blocks_128(N, K):
    return lambda ij: (ij[0] // 128) * (K // 128) + ij[1] // 128


@pytest.mark.parametrize("M,N,K", [(128, 128, 128), (256, 128, 256), (128, 256, 384)])
def test_brute_force_fprop(M, N, K):
    X = dyadic_groups((M, K), rows_1x128(M, K), seed=M + 3 * N + 7 * K)
    W = dyadic_groups((N, K), blocks_128(N, K), seed=1 + M + N + K)
    xq, xs = oracle.quant_1x128(bits(X))
    wq, ws, _ = oracle.quant_128x128(bits(W))
    assert set(np.unique(xs)) <= {np.float32(2.0 ** j) for j in range(-3, 4)}
    D, S = oracle.gemm(oracle.FPROP, xq, xs, wq, ws)
    assert np.array_equal(D, X.astype(np.float64) @ W.astype(np.float64).T)
    assert np.array_equal(S, np.abs(X.astype(np.float64)) @ np.abs(W.astype(np.float64)).T)


@pytest.mark.parametrize("M,N,K", [(128, 128, 128), (256, 384, 128), (128, 256, 256)])
def test_brute_force_dgrad(M, N, K):
    # dX[M,N] = dY[M,K] . W[K,N], with W the forward weight [out=K, in=N] used transposed.
    dY = dyadic_groups((M, K), rows_1x128(M, K), seed=11 + M + N + K)
    W = dyadic_groups((K, N), blocks_128(K, N), seed=12 + M + N + K)
    gq, gs = oracle.quant_1x128(bits(dY))
    wq, ws, _ = oracle.quant_128x128(bits(W))
    D, _ = oracle.gemm(oracle.DGRAD, gq, gs, wq, ws)
    assert np.array_equal(D, dY.astype(np.float64) @ W.astype(np.float64))


@pytest.mark.parametrize("T,Cout,Cin", [(128, 128, 128), (256, 128, 384), (384, 256, 128)])
def test_brute_force_wgrad(T, Cout, Cin):
    # dW[Cout,Cin] = dY[T,Cout]^T . X[T,Cin], both quantised 128x1 along tokens.
    dY = dyadic_groups((T, Cout), cols_128x1(T, Cout), seed=21 + T + Cout + Cin)
    X = dyadic_groups((T, Cin), cols_128x1(T, Cin), seed=22 + T + Cout + Cin)
    gq, gs = oracle.quant_128x1_t(bits(dY))
    xq, xs = oracle.quant_128x1_t(bits(X))
    D, _ = oracle.gemm(oracle.WGRAD, gq, gs, xq, xs)
    assert np.array_equal(D, dY.astype(np.float64).T @ X.astype(np.float64))


def test_entries_match_full_product():
    d = synth.tiny_fprop()
    xq, xs = oracle.quant_1x128(d["X"])
    wq, ws, _ = oracle.quant_128x128(d["W"])
    D, S = oracle.gemm(oracle.FPROP, xq, xs, wq, ws)
    g = np.random.Generator(np.random.PCG64(5))
    ms = g.integers(0, D.shape[0], 300)
    ns = g.integers(0, D.shape[1], 300)
    e, s = oracle.gemm_entries(oracle.FPROP, xq, xs, wq, ws, ms, ns)
    assert np.array_equal(e, D[ms, ns]) and np.array_equal(s, S[ms, ns])


def test_one_hot_selects_weight_columns():
    """X = [448 I | 0] selects 448 * W_hat[n, m] (Fprop) exactly."""
    N, K = 256, 256
    X = np.zeros((128, K), dtype=np.float32)
    X[np.arange(128), np.arange(128)] = 448.0
    W = f32(synth.weights(N, K, seed=31))
    xq, xs = oracle.quant_1x128(bits(X))
    wq, ws, _ = oracle.quant_128x128(bits(W))
    D, _ = oracle.gemm(oracle.FPROP, xq, xs, wq, ws)
    w_hat = oracle.e4m3_decode(wq) * np.kron(ws.astype(np.float64), np.ones((128, 128)))
    assert np.array_equal(D, 448.0 * w_hat[:, :128].T)


def test_one_hot_selects_weight_rows_dgrad():
    """dY = [0 | 448 I] selects 448 * W_hat[128 + m, n] (Dgrad uses W transposed)."""
    Kout, Nin = 256, 384
    dY = np.zeros((128, Kout), dtype=np.float32)
    dY[np.arange(128), 128 + np.arange(128)] = 448.0
    W = f32(synth.weights(Kout, Nin, seed=32))
    gq, gs = oracle.quant_1x128(bits(dY))
    wq, ws, _ = oracle.quant_128x128(bits(W))
    D, _ = oracle.gemm(oracle.DGRAD, gq, gs, wq, ws)
    w_hat = oracle.e4m3_decode(wq) * np.kron(ws.astype(np.float64), np.ones((128, 128)))
    assert np.array_equal(D, 448.0 * w_hat[128:, :])


def _elem_err_bound(xf, dec_times_s, s_per_elem):
    """Bound on |x - dec(q) s| for nearest rounding, per element (see the quantiser pins)."""
    y = np.abs(xf) / s_per_elem
    slack = 1.0 + 2.0 ** -18
    return np.where(y >= 2.0 ** -6, 2.0 ** -4 * np.abs(xf) * slack, 2.0 ** -10 * s_per_elem * slack)


def test_bounded_quantisation_error_vs_unquantised():
    d = synth.tiny_fprop()
    X = f32(d["X"]).astype(np.float64)
    W = f32(d["W"]).astype(np.float64)
    xq, xs = oracle.quant_1x128(d["X"])
    wq, ws, _ = oracle.quant_128x128(d["W"])
    D, _ = oracle.gemm(oracle.FPROP, xq, xs, wq, ws)
    sx = np.repeat(xs.T.astype(np.float64), 128, axis=1)
    sw = np.kron(ws.astype(np.float64), np.ones((128, 128)))
    x_hat = oracle.e4m3_decode(xq) * sx
    w_hat = oracle.e4m3_decode(wq) * sw
    dx = _elem_err_bound(X, x_hat, sx)
    dw = _elem_err_bound(W, w_hat, sw)
    assert np.all(np.abs(X - x_hat) <= dx) and np.all(np.abs(W - w_hat) <= dw)
    exact = X @ W.T
    bound = np.abs(X) @ dw.T + dx @ np.abs(W).T + dx @ dw.T
    assert np.all(np.abs(D - exact) <= bound * (1 + 1e-12) + 1e-300)
    rel_rms = np.sqrt(np.mean((D - exact) ** 2) / np.mean(exact ** 2))
    # E4M3 keeps 3 fraction bits: errors around 2^-5 relative per element, averaging down.
    assert rel_rms < 0.05, rel_rms


def test_grouped_integer_brute_force():
    g = np.random.Generator(np.random.PCG64(41))
    E, N, K = 5, 128, 256
    counts = np.array([0, 3, 130, 0, 1])
    off = np.zeros(E + 1, dtype=np.int32)
    off[1:] = np.cumsum(counts)
    Mtot = int(off[-1])
    A = g.integers(-16, 17, size=(Mtot, K)).astype(np.float32)
    A[:, 0] = 448.0
    A[:, 128] = -448.0
    Bs = g.integers(-16, 17, size=(E, N, K)).astype(np.float32)
    Bs[:, 0, 0] = 448.0
    Bs[:, 0, 128] = 448.0
    aq, as_ = oracle.quant_1x128(bits(A))
    bq = np.empty((E, N, K), dtype=np.uint8)
    bs = np.empty((E, N // 128, K // 128), dtype=np.float32)
    for e in range(E):
        bq[e], bs[e], _ = oracle.quant_128x128(bits(Bs[e]))
    assert np.all(as_ == 1.0) and np.all(bs == 1.0)
    ms, ns = np.meshgrid(np.arange(Mtot), np.arange(N), indexing="ij")
    got, _ = oracle.grouped_entries(aq, as_, bq, bs, off, ms.reshape(-1), ns.reshape(-1))
    got = got.reshape(Mtot, N)
    for e in range(E):
        rows = slice(off[e], off[e + 1])
        ref = A[rows].astype(np.int64) @ Bs[e].astype(np.int64).T
        assert np.array_equal(got[rows], ref.astype(np.float64))

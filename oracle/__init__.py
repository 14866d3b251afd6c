"""CPU oracle for fine-grained FP8 quantisation and the block-scaled FP8 GEMM.

TEST INFRASTRUCTURE ONLY: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this package.  It shares no code with the CUDA path
(``fp8_fine_grained_fp8q_b200``) and neither imports the other.

What it computes, from the pages on the DeepSeek-V3 Technical Report (arXiv 2412.19437):

* E4M3 codes for every FP8 operand -- "DeepSeek-V3 Technical Report" summary page
  (xyznot.com), Key ideas, FP8 mixed-precision bullet; Questions, the answer on training FP8
  without divergence.
* 1x128 tile-wise activation scales and 128x128 block-wise weight scales -- same passages.
* 128x1 (token-direction) scales for the Wgrad operands: the groups run along the GEMM's inner
  dimension -- DeepSeek-V3 report repost (why-be.co.kr), paragraph 4; Wgrad runs in FP8 --
  paragraph 2 (Figure 6) and paragraph 3.
* The GEMM D = sum_k A(m,k) B(k,n) of the dequantised operands, with the per-128-K scales
  applied to each 128-wide partial sum at promotion -- repost paragraphs 1 and 4 (N_c = 128,
  Figure 7(b)); summary page FP8 bullet.  Mathematically that equals the plain dot product of
  the dequantised operands, which is what the oracle evaluates, exactly in binary64.
  Fprop and Dgrad outputs are bf16, the Wgrad output FP32 (repost paragraph 3: gradients in
  FP32).

Readings the pages leave open (OCP E4M3FN, round-to-nearest-even with saturation at 448,
max-abs scaling with an amax floor of 2^-100) are stated in ``fp8q_oracle.c``.

The quantisers also take ``scale_fmt="ue8m0"``: a power-of-two scale (the smallest power of two
not below the binary32 quotient a / 448), a separate mode the pages do not describe.  It is the
scale format the block-scaled tensor-core MMA accepts; the GEMM oracle needs no change for it,
since its scales are ordinary binary32 values.

The arithmetic lives in ``fp8q_oracle.c``; this module only marshals numpy arrays (and, for the
expert-grouped Wgrad operands, pads each expert's rows before calling it).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

FPROP, DGRAD, WGRAD = 0, 1, 2
SCALE_FORMATS = {"fp32": 0, "ue8m0": 1}

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_encode_array.argtypes = [P, I64, P]
        lib.oracle_e4m3_decode_array.argtypes = [P, I64, P]
        lib.oracle_quant_1x128_fmt.argtypes = [P, I64, I64, P, P, ctypes.c_int]
        lib.oracle_quant_128x1_t_fmt.argtypes = [P, I64, I64, P, P, ctypes.c_int]
        lib.oracle_quant_128x128_fmt.argtypes = [P, I64, I64, P, P, P, ctypes.c_int]
        lib.oracle_gemm.argtypes = [ctypes.c_int, P, P, P, P, I64, I64, I64, P, P, P, P]
        lib.oracle_gemm_entries.argtypes = [ctypes.c_int, P, P, P, P, I64, I64, I64, P, P,
                                            I64, P, P]
        lib.oracle_grouped_entries.argtypes = [P, P, P, P, P, ctypes.c_int32, I64, I64, I64,
                                               P, P, I64, P, P]
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    """Accept bf16 payloads as uint16 bit patterns (the seeded generators produce these)."""
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint16:
        raise TypeError("bf16 inputs are passed as uint16 bit patterns")
    return x


def num_threads() -> int:
    return int(_load().oracle_num_threads())


# ----------------------------------------------------------------------------------------- #
# E4M3 codec
# ----------------------------------------------------------------------------------------- #

def e4m3_encode(x) -> np.ndarray:
    """E4M3FN codes of binary32 values: round to nearest even, saturate at +-448."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    out = np.empty(x.shape, dtype=np.uint8)
    _load().oracle_e4m3_encode_array(_ptr(x), x.size, _ptr(out))
    return out


def e4m3_decode(c) -> np.ndarray:
    """Exact binary64 values of E4M3FN codes (NaN for 0x7F / 0xFF)."""
    c = np.ascontiguousarray(np.asarray(c, dtype=np.uint8))
    out = np.empty(c.shape, dtype=np.float64)
    _load().oracle_e4m3_decode_array(_ptr(c), c.size, _ptr(out))
    return out


# ----------------------------------------------------------------------------------------- #
# Quantisers
# ----------------------------------------------------------------------------------------- #

def _fmt(scale_fmt: str) -> int:
    """"fp32": the pages' max-abs scale a / 448.  "ue8m0": its power-of-two variant, the
    smallest power of two not below the binary32 quotient a / 448 (a separate mode the pages do
    not describe: the scale format of the block-scaled tensor-core MMA)."""
    try:
        return SCALE_FORMATS[scale_fmt]
    except KeyError:
        raise ValueError(f"scale_fmt must be one of {sorted(SCALE_FORMATS)}") from None


def quant_1x128(x_bits: np.ndarray, scale_fmt: str = "fp32"):
    """x[M,K] bf16 bits -> (q[M,K] uint8, s[K/128, M] float32)."""
    x = _bf16_bits(x_bits)
    M, K = x.shape
    q = np.empty((M, K), dtype=np.uint8)
    s = np.empty((K // 128, M), dtype=np.float32)
    _load().oracle_quant_1x128_fmt(_ptr(x), M, K, _ptr(q), _ptr(s), _fmt(scale_fmt))
    return q, s


def quant_128x1_t(x_bits: np.ndarray, scale_fmt: str = "fp32"):
    """x[T,C] bf16 bits -> (qt[C,T] uint8, s[T/128, C] float32)."""
    x = _bf16_bits(x_bits)
    T, C = x.shape
    qt = np.empty((C, T), dtype=np.uint8)
    s = np.empty((T // 128, C), dtype=np.float32)
    _load().oracle_quant_128x1_t_fmt(_ptr(x), T, C, _ptr(qt), _ptr(s), _fmt(scale_fmt))
    return qt, s


def quant_128x128(w_bits: np.ndarray, want_transposed: bool = False, scale_fmt: str = "fp32"):
    """w[N,K] bf16 bits -> (q[N,K], s[N/128, K/128], qt[K,N] or None)."""
    w = _bf16_bits(w_bits)
    N, K = w.shape
    q = np.empty((N, K), dtype=np.uint8)
    s = np.empty((N // 128, K // 128), dtype=np.float32)
    qt = np.empty((K, N), dtype=np.uint8) if want_transposed else None
    _load().oracle_quant_128x128_fmt(_ptr(w), N, K, _ptr(q), _ptr(s),
                                     _ptr(qt) if qt is not None else None, _fmt(scale_fmt))
    return q, s, qt


# ----------------------------------------------------------------------------------------- #
# GEMM
# ----------------------------------------------------------------------------------------- #

def _gemm_dims(mode, A, B):
    M, K = A.shape
    if mode == DGRAD:
        Kb, N = B.shape
    else:
        N, Kb = B.shape
    assert Kb == K, "inner dimensions differ"
    return M, N, K


def gemm(mode: int, A, sA, B, sB):
    """Exact binary64 D[M,N] and S[M,N] = sum_k |A(m,k) B(k,n)| of the dequantised operands.

    A: [M,K] codes, sA: [K/128, M].  B and sB per mode:
    FPROP  B = W[N,K],  sB = [N/128, K/128]
    DGRAD  B = W[K,N] (the forward weight, used transposed), sB = [K/128, N/128]
    WGRAD  B = X^T[N,K], sB = [K/128, N]
    """
    A = np.ascontiguousarray(A, dtype=np.uint8)
    B = np.ascontiguousarray(B, dtype=np.uint8)
    sA = np.ascontiguousarray(sA, dtype=np.float32)
    sB = np.ascontiguousarray(sB, dtype=np.float32)
    M, N, K = _gemm_dims(mode, A, B)
    D = np.empty((M, N), dtype=np.float64)
    S = np.empty((M, N), dtype=np.float64)
    wa = np.empty((M, K), dtype=np.float64)
    wb = np.empty((N, K), dtype=np.float64)
    _load().oracle_gemm(mode, _ptr(A), _ptr(sA), _ptr(B), _ptr(sB), M, N, K,
                        _ptr(D), _ptr(S), _ptr(wa), _ptr(wb))
    return D, S


def gemm_entries(mode: int, A, sA, B, sB, ms, ns):
    """D[ms[i], ns[i]] and S[ms[i], ns[i]] only (for full-size problems)."""
    A = np.ascontiguousarray(A, dtype=np.uint8)
    B = np.ascontiguousarray(B, dtype=np.uint8)
    sA = np.ascontiguousarray(sA, dtype=np.float32)
    sB = np.ascontiguousarray(sB, dtype=np.float32)
    M, N, K = _gemm_dims(mode, A, B)
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    assert ms.shape == ns.shape
    out = np.empty(ms.shape, dtype=np.float64)
    sabs = np.empty(ms.shape, dtype=np.float64)
    _load().oracle_gemm_entries(mode, _ptr(A), _ptr(sA), _ptr(B), _ptr(sB), M, N, K,
                                _ptr(ms), _ptr(ns), ms.size, _ptr(out), _ptr(sabs))
    return out, sabs


def grouped_entries(A, sA, B, sB, offsets, ms, ns):
    """Grouped Fprop entries: A[Mtot,K], sA[K/128,Mtot], B[E,N,K], sB[E,N/128,K/128],
    offsets[E+1] (rows of expert e are offsets[e]..offsets[e+1]-1)."""
    A = np.ascontiguousarray(A, dtype=np.uint8)
    B = np.ascontiguousarray(B, dtype=np.uint8)
    sA = np.ascontiguousarray(sA, dtype=np.float32)
    sB = np.ascontiguousarray(sB, dtype=np.float32)
    off = np.ascontiguousarray(offsets, dtype=np.int32)
    Mtot, K = A.shape
    E, N, Kb = B.shape
    assert Kb == K and off.size == E + 1
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    out = np.empty(ms.shape, dtype=np.float64)
    sabs = np.empty(ms.shape, dtype=np.float64)
    _load().oracle_grouped_entries(_ptr(A), _ptr(sA), _ptr(B), _ptr(sB), _ptr(off), E, Mtot,
                                   N, K, _ptr(ms), _ptr(ns), ms.size, _ptr(out), _ptr(sabs))
    return out, sabs


def ragged_group_prefix(offsets) -> np.ndarray:
    """P[e] = sum over e' < e of ceil(n_e' / 128): expert e's first 128-token group in the
    padded token axis of the grouped Wgrad operands (P[E] groups in all)."""
    off = np.asarray(offsets, dtype=np.int64)
    n = off[1:] - off[:-1]
    P = np.zeros(off.size, dtype=np.int64)
    np.cumsum((n + 127) // 128, out=P[1:])
    return P


def quant_128x1_t_ragged(x_bits: np.ndarray, offsets, scale_fmt: str = "fp32"):
    """128x1 groups along each expert's own tokens, for the grouped Wgrad dW_e = dY_e^T X_e.

    x[Mtot, C] bf16 bits with rows ordered by expert (rows offsets[e] .. offsets[e+1]-1 are
    expert e's).  Reading (the pages fix only that the groups run along the GEMM's inner, i.e.
    token, dimension -- repost paragraph 4): an expert's groups start at its first token; its last
    group holds the n_e mod 128 remaining tokens and takes its max-abs over those.  That is the
    plain 128x1 quantiser on the expert's rows zero-padded to a multiple of 128 (a zero changes
    neither the max-abs nor a dot product), which is how it is computed here.
    Returns qt[C, 128*P[E]] (expert e's tokens at columns 128*P[e] .., zero codes in its padding)
    and s[P[E], C]."""
    off = np.asarray(offsets, dtype=np.int64)
    C = x_bits.shape[1]
    P = ragged_group_prefix(off)
    qt = np.zeros((C, 128 * int(P[-1])), dtype=np.uint8)
    s = np.empty((int(P[-1]), C), dtype=np.float32)
    for e in range(off.size - 1):
        n = int(off[e + 1] - off[e])
        if n == 0:
            continue
        g = int(P[e + 1] - P[e])
        block = np.zeros((128 * g, C), dtype=x_bits.dtype)
        block[:n] = x_bits[off[e]:off[e + 1]]
        q, se = quant_128x1_t(block, scale_fmt=scale_fmt)
        qt[:, 128 * int(P[e]):128 * int(P[e + 1])] = q
        s[int(P[e]):int(P[e + 1])] = se
    return qt, s

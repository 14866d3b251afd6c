"""Seeded synthetic inputs shaped like DeepSeek-V3's FP8 linear-layer workloads.

This module holds input generation only -- no quantisation or GEMM arithmetic -- so that the
CUDA path's tests and the CPU oracle can be fed the same bytes.  Every tensor is returned as
host numpy arrays: bf16 payloads as ``uint16`` bit patterns (float32 rounded to nearest even).

Shapes follow the model dimensions on the pages (hidden size 7168 and the MLA compression widths
1536 / 512 in the wenxiaobai article's hyper-parameter paragraph; 256 routed experts with 8
active per token in the "DeepSeek-V3 Technical Report" summary page, Key ideas).  The value
distributions are the workload recipe of this library's benchmarks:

* activations ~ N(0, 1) with 0.1 % outliers x100 (individual entries for the tiny case, whole
  channels for the full-size case);
* weights ~ N(0, 0.02);
* output gradients ~ N(0, 1e-3) with 1 % of entries replaced by 1e-3 * Student-t(3) draws;
* MoE routing: 8 distinct experts per token drawn without replacement from Zipf(1.1)-skewed
  weights over the experts, with a seeded handful of experts given weight zero (so they are
  empty).
"""
from __future__ import annotations

import numpy as np

SEED_BASE = 0xF8F8


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round binary32 values to bf16 (nearest, ties to even); return the uint16 bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    b = x.view(np.uint32).astype(np.uint64)
    rounded = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    nan = np.isnan(x)
    out = rounded.astype(np.uint16)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def normal_bf16(shape, std: float, seed: int) -> np.ndarray:
    g = rng(seed)
    x = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return f32_to_bf16_bits(x)


def activations_entry_outliers(M: int, K: int, seed: int, frac: float = 1e-3,
                               factor: float = 100.0) -> np.ndarray:
    """X ~ N(0,1) with a seeded ``frac`` of individual entries multiplied by ``factor``."""
    g = rng(seed)
    x = g.standard_normal(size=(M, K), dtype=np.float32)
    n_out = int(round(frac * M * K))
    idx = g.choice(M * K, size=n_out, replace=False)
    x.reshape(-1)[idx] *= np.float32(factor)
    return f32_to_bf16_bits(x)


def activations_channel_outliers(M: int, K: int, seed: int, frac: float = 1e-3,
                                 factor: float = 100.0) -> np.ndarray:
    """X ~ N(0,1) with round(frac*K) seeded channels multiplied by ``factor`` for every token."""
    g = rng(seed)
    x = g.standard_normal(size=(M, K), dtype=np.float32)
    n_ch = max(1, int(round(frac * K)))
    ch = g.permutation(K)[:n_ch]
    x[:, ch] *= np.float32(factor)
    return f32_to_bf16_bits(x)


def output_grad(M: int, N: int, seed: int, std: float = 1e-3, frac_t: float = 0.01) -> np.ndarray:
    """dY ~ N(0, std) with a seeded ``frac_t`` of entries replaced by std * Student-t(3)."""
    g = rng(seed)
    y = g.standard_normal(size=(M, N), dtype=np.float32) * np.float32(std)
    n_t = int(round(frac_t * M * N))
    idx = g.choice(M * N, size=n_t, replace=False)
    y.reshape(-1)[idx] = (g.standard_t(3, size=n_t) * std).astype(np.float32)
    return f32_to_bf16_bits(y)


def weights(N: int, K: int, seed: int, std: float = 0.02) -> np.ndarray:
    return normal_bf16((N, K), std, seed)


# ------------------------------------------------------------------------------------------ #
# Named workloads
# ------------------------------------------------------------------------------------------ #

def tiny_fprop(seed: int = SEED_BASE + 0):
    """X[256,512] with 0.1 % entry outliers, W[512,512] ~ N(0,0.02)."""
    return {"X": activations_entry_outliers(256, 512, seed),
            "W": weights(512, 512, seed + 1000)}


def linear_layer(T: int = 4096, C_in: int = 7168, C_out: int = 2048,
                 seed: int = SEED_BASE + 1):
    """One linear layer's FP8 training operands: X[T,C_in], W[C_out,C_in], dY[T,C_out]."""
    return {"X": activations_channel_outliers(T, C_in, seed),
            "W": weights(C_out, C_in, seed + 1000),
            "dY": output_grad(T, C_out, seed + 2000)}


def moe_routing(tokens: int = 8192, experts: int = 256, top_k: int = 8, n_empty: int = 8,
                zipf_s: float = 1.1, seed: int = SEED_BASE + 4):
    """Route each token to ``top_k`` distinct experts.

    A seeded permutation gives each expert a popularity rank r (1..E) and weight r^-zipf_s;
    ``n_empty`` seeded experts get weight 0.  Each token draws ``top_k`` distinct experts by
    Gumbel-top-k on the log weights.  Returns (expert_of[tokens, top_k], counts[E]).
    """
    g = rng(seed)
    rank = g.permutation(experts) + 1
    w = rank.astype(np.float64) ** (-zipf_s)
    empty = g.choice(experts, size=n_empty, replace=False)
    w[empty] = 0.0
    logw = np.full(experts, -np.inf)
    nz = w > 0
    logw[nz] = np.log(w[nz])
    gumbel = g.gumbel(size=(tokens, experts))
    keys = logw[None, :] + gumbel
    top = np.argpartition(-keys, top_k - 1, axis=1)[:, :top_k]
    counts = np.bincount(top.reshape(-1), minlength=experts)
    return top.astype(np.int32), counts.astype(np.int64)


def moe_grouped_rows(expert_of: np.ndarray, experts: int):
    """Order the (token, slot) pairs by expert, then token.  Returns (token_index[Mtot],
    offsets[E+1] int32) so that rows offsets[e]..offsets[e+1]-1 belong to expert e."""
    tokens, k = expert_of.shape
    flat_e = expert_of.reshape(-1)
    flat_t = np.repeat(np.arange(tokens, dtype=np.int64), k)
    order = np.lexsort((flat_t, flat_e))
    counts = np.bincount(flat_e, minlength=experts)
    offsets = np.zeros(experts + 1, dtype=np.int64)
    np.cumsum(counts, out=offsets[1:])
    return flat_t[order], offsets.astype(np.int32)


def expert_weights(e: int, N: int = 2048, K: int = 7168, seed: int = SEED_BASE + 4):
    """W_e ~ N(0, 0.02), each expert from its own sub-seed so any expert regenerates alone."""
    return weights(N, K, seed * 1000 + 17 * e + 3)

"""Shared helpers for the parity tests: host <-> device marshalling and the GEMM tolerance.

The tolerance is the match criterion of this library's GEMM: elementwise
    B   = 2e-3 * S + 1e-2 * ulp_bf16(|ref|)                   (FP32 accumulator, FP32 D)
    B16 = B + 0.5 * ulp_bf16(|ref| + B)                       (bf16 D)
where ref is the oracle's exact binary64 result, S = sum_k |A^(m,k) B^(k,n)| and
ulp_bf16(x) = 2^(floor(log2 x) - 7) (2^-133 for x = 0).  B bounds the FP32 accumulator acc;
Fprop and Dgrad then round acc to bf16 (nearest even), which moves it by at most half a bf16 ulp
of |acc| <= |ref| + B, so the bf16 term depends on the oracle's values alone.  Without that term
even the correctly rounded bf16 of the exact value fails wherever one product dominates the dot
product (S close to |ref|), as with the outlier channels of the activation workload.
"""
from __future__ import annotations

import numpy as np
import torch

REL = 2e-3
ULP_FRAC = 1e-2


def bf16_dev(bits: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns -> torch.bfloat16 tensor on the device."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).to(device)


def u8_dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to(device)


def f32_dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def host(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.float().numpy().astype(np.float64)
    return t.numpy()


def ulp_bf16(x: np.ndarray) -> np.ndarray:
    ax = np.abs(np.asarray(x, dtype=np.float64))
    out = np.full(ax.shape, 2.0 ** -133)
    nz = ax > 0
    out[nz] = np.exp2(np.floor(np.log2(ax[nz])) - 7)
    return out


def tolerance(ref: np.ndarray, sabs: np.ndarray, bf16_out: bool = False) -> np.ndarray:
    """Elementwise bound from the oracle's result and sum of |products| only."""
    bound = REL * np.asarray(sabs, dtype=np.float64) + ULP_FRAC * ulp_bf16(ref)
    if bf16_out:
        bound = bound + 0.5 * ulp_bf16(np.abs(np.asarray(ref, dtype=np.float64)) + bound)
    return bound


def check_gemm(gpu: np.ndarray, ref: np.ndarray, sabs: np.ndarray, what: str = "",
               bf16_out: bool = True) -> float:
    """Assert the tolerance elementwise; return the worst |err| / bound.  bf16_out: D was
    rounded to bf16 (Fprop, Dgrad, grouped Fprop); False for the FP32 Wgrad output."""
    gpu = np.asarray(gpu, dtype=np.float64)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite outputs"
    err = np.abs(gpu - ref)
    bound = tolerance(ref, sabs, bf16_out)
    ratio = err / bound
    worst = float(ratio.max()) if ratio.size else 0.0
    if worst > 1.0:
        i = np.unravel_index(int(np.argmax(ratio)), ratio.shape)
        raise AssertionError(f"{what}: max err/bound {worst:.3g} at {i}: gpu {gpu[i]!r} "
                             f"ref {ref[i]!r} S {sabs[i]!r} ({int((ratio > 1).sum())} of "
                             f"{ratio.size} out of tolerance)")
    return worst


def cuda_ok() -> bool:
    return torch.cuda.is_available()


_layer_cache = {}


def linear_layer_inputs():
    """The full-size linear-layer operands (X [4096,7168], W [2048,7168], dY [4096,2048]),
    generated once per test session."""
    if "layer" not in _layer_cache:
        from fp8_fine_grained_fp8q_b200 import synth
        _layer_cache["layer"] = synth.linear_layer()
    return _layer_cache["layer"]

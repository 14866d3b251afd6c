"""ctypes binding of libfp8q.so (C ABI in include/fp8q.h).

Argument marshalling only: every step of the computation runs in the library's CUDA kernels.
PyTorch provides device memory and the current stream.  There is no fallback path: if the
library is missing or a call fails, an exception is raised.

Tensor conventions (all CUDA, contiguous):
  bf16 inputs are torch.bfloat16; E4M3 codes are torch.uint8 (view as torch.float8_e4m3fn if
  wanted); scales are torch.float32 with the group-major layouts the header documents.
"""
from __future__ import annotations

import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfp8q.so")

FPROP, DGRAD, WGRAD, WGRAD_ACC = 0, 1, 2, 3
DEV_OK, DEV_TIMEOUT, DEV_BAD_OFFSETS, DEV_BAD_SCALES = 0, 1, 2, 3
# Quantiser scale formats: the pages' max-abs scale a / 448, or the power-of-two (UE8M0) variant.
SCALE_FORMATS = {"fp32": 0, "ue8m0": 1}

_lib = None


class Fp8qError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status_string(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """Load libfp8q.so (built in-tree by fp8_fine_grained_fp8q_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m fp8_fine_grained_fp8q_b200.build` (needs nvcc)")
    L = ctypes.CDLL(LIB_PATH)
    P, I64, I32, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int
    L.fp8q_status_string.restype = ctypes.c_char_p
    L.fp8q_status_string.argtypes = [I]
    L.fp8q_abi_version.restype = I
    L.fp8q_abi_version.argtypes = []
    for name, args in {
        "fp8q_act_1x128": [P, I64, I64, P, P, P],
        "fp8q_act_128x1_transposed": [P, I64, I64, P, P, P],
        "fp8q_act_dual": [P, I64, I64, P, P, P, P, P],
        "fp8q_quant_forward": [P, I64, I64, P, P, P, P, P, I64, P, P, P, P],
        "fp8q_weight_128x128": [P, I64, I64, P, P, P, P],
        "fp8_gemm_blockscaled": [I, P, P, P, P, P, I64, I64, I64, P, ctypes.c_size_t, P],
        "fp8_gemm_blockscaled_quant": [I, P, P, P, P, P, P, P, I64, I64, I64, P, ctypes.c_size_t, P],
        "fp8_grouped_gemm_blockscaled": [P, P, P, P, P, I32, I64, I64, I64, P, P],
        "fp8_grouped_gemm_blockscaled_dgrad": [P, P, P, P, P, I32, I64, I64, I64, P, P],
        "fp8_grouped_gemm_blockscaled_wgrad": [P, P, P, P, P, I32, I64, I64, I64, I64, P, P],
        "fp8q_act_128x1_transposed_ragged": [P, P, I32, I64, I64, P, P, I64, P],
        "fp8q_device_status": [P, ctypes.POINTER(I)],
        "fp8q_act_1x128_fmt": [P, I64, I64, P, P, I, P],
        "fp8q_act_128x1_transposed_fmt": [P, I64, I64, P, P, I, P],
        "fp8q_act_dual_fmt": [P, I64, I64, P, P, P, P, I, P],
        "fp8q_quant_forward_fmt": [P, I64, I64, P, P, P, P, P, I64, P, P, P, I, P],
        "fp8q_weight_128x128_fmt": [P, I64, I64, P, P, P, I, P],
        "fp8_gemm_blockscaled_ue8m0": [I, P, P, P, P, P, I64, I64, I64, P, ctypes.c_size_t, P],
    }.items():
        fn = getattr(L, name)
        fn.restype = I
        fn.argtypes = args
    L.fp8q_selftest_wait_timeout.restype = I
    L.fp8q_selftest_wait_timeout.argtypes = [ctypes.c_uint64, P]
    L.fp8q_gemm_workspace_size.restype = ctypes.c_size_t
    L.fp8q_gemm_workspace_size.argtypes = [I, I64, I64, I64]
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().fp8q_status_string(int(status)).decode()


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(fn: str, status: int):
    if status != 0:
        raise Fp8qError(fn, status)


def _require(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got {t.dim()}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _out(t, shape, dtype, device, name):
    if t is None:
        return torch.empty(shape, dtype=dtype, device=device)
    _require(t, name, dtype, len(shape))
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _fmt(scale_fmt: str) -> int:
    try:
        return SCALE_FORMATS[scale_fmt]
    except KeyError:
        raise ValueError(f"scale_fmt must be one of {sorted(SCALE_FORMATS)}") from None


# ------------------------------------------------------------------------------------------ #
# Quantisers
# ------------------------------------------------------------------------------------------ #

def act_1x128(x: torch.Tensor, q: torch.Tensor | None = None, s: torch.Tensor | None = None,
              scale_fmt: str = "fp32"):
    """x[M,K] bf16 -> (q[M,K] uint8 E4M3 codes, s[K/128, M] fp32).  scale_fmt "ue8m0" selects the
    power-of-two scales (fp8q_act_1x128_fmt)."""
    _require(x, "x", torch.bfloat16, 2)
    M, K = x.shape
    q = _out(q, (M, K), torch.uint8, x.device, "q")
    s = _out(s, (K // 128, M), torch.float32, x.device, "s")
    if scale_fmt == "fp32":
        _check("fp8q_act_1x128", lib().fp8q_act_1x128(_p(x), M, K, _p(q), _p(s), _stream(x.device)))
    else:
        _check("fp8q_act_1x128_fmt", lib().fp8q_act_1x128_fmt(_p(x), M, K, _p(q), _p(s), _fmt(scale_fmt),
                                                              _stream(x.device)))
    return q, s


def act_128x1_transposed(x: torch.Tensor, qt: torch.Tensor | None = None,
                         s: torch.Tensor | None = None, scale_fmt: str = "fp32"):
    """x[T,C] bf16 -> (qt[C,T] uint8, s[T/128, C] fp32)."""
    _require(x, "x", torch.bfloat16, 2)
    T, C = x.shape
    qt = _out(qt, (C, T), torch.uint8, x.device, "qt")
    s = _out(s, (T // 128, C), torch.float32, x.device, "s")
    if scale_fmt == "fp32":
        _check("fp8q_act_128x1_transposed",
               lib().fp8q_act_128x1_transposed(_p(x), T, C, _p(qt), _p(s), _stream(x.device)))
    else:
        _check("fp8q_act_128x1_transposed_fmt",
               lib().fp8q_act_128x1_transposed_fmt(_p(x), T, C, _p(qt), _p(s), _fmt(scale_fmt), _stream(x.device)))
    return qt, s


def act_dual(x: torch.Tensor, q: torch.Tensor | None = None, s: torch.Tensor | None = None,
             qt: torch.Tensor | None = None, st: torch.Tensor | None = None, scale_fmt: str = "fp32"):
    """x[T,C] bf16 -> (q[T,C], s[C/128, T], qt[C,T], st[T/128, C]) in one pass over x: the
    outputs of act_1x128(x) and act_128x1_transposed(x), bit for bit."""
    _require(x, "x", torch.bfloat16, 2)
    T, C = x.shape
    q = _out(q, (T, C), torch.uint8, x.device, "q")
    s = _out(s, (C // 128, T), torch.float32, x.device, "s")
    qt = _out(qt, (C, T), torch.uint8, x.device, "qt")
    st = _out(st, (T // 128, C), torch.float32, x.device, "st")
    if scale_fmt == "fp32":
        _check("fp8q_act_dual",
               lib().fp8q_act_dual(_p(x), T, C, _p(q), _p(s), _p(qt), _p(st), _stream(x.device)))
    else:
        _check("fp8q_act_dual_fmt",
               lib().fp8q_act_dual_fmt(_p(x), T, C, _p(q), _p(s), _p(qt), _p(st), _fmt(scale_fmt),
                                       _stream(x.device)))
    return q, s, qt, st


def quant_forward(x: torch.Tensor, w: torch.Tensor, xq=None, xs=None, xqt=None, xst=None,
                  wq=None, ws=None, wqt=None, transposed_w: bool = False, scale_fmt: str = "fp32"):
    """x[T,C], w[N,C] bf16 -> ((xq, xs, xqt, xst), (wq, ws, wqt or None)) in one launch: the outputs of
    act_dual(x) and weight_128x128(w), bit for bit."""
    _require(x, "x", torch.bfloat16, 2)
    _require(w, "w", torch.bfloat16, 2)
    T, C = x.shape
    N, Cw = w.shape
    if Cw != C:
        raise ValueError("x and w must share the inner dimension")
    dev = x.device
    xq = _out(xq, (T, C), torch.uint8, dev, "xq")
    xs = _out(xs, (C // 128, T), torch.float32, dev, "xs")
    xqt = _out(xqt, (C, T), torch.uint8, dev, "xqt")
    xst = _out(xst, (T // 128, C), torch.float32, dev, "xst")
    wq = _out(wq, (N, C), torch.uint8, dev, "wq")
    ws = _out(ws, (N // 128, C // 128), torch.float32, dev, "ws")
    if transposed_w or wqt is not None:
        wqt = _out(wqt, (C, N), torch.uint8, dev, "wqt")
    if scale_fmt == "fp32":
        _check("fp8q_quant_forward",
               lib().fp8q_quant_forward(_p(x), T, C, _p(xq), _p(xs), _p(xqt), _p(xst), _p(w), N, _p(wq), _p(ws),
                                        _p(wqt), _stream(dev)))
    else:
        _check("fp8q_quant_forward_fmt",
               lib().fp8q_quant_forward_fmt(_p(x), T, C, _p(xq), _p(xs), _p(xqt), _p(xst), _p(w), N, _p(wq),
                                            _p(ws), _p(wqt), _fmt(scale_fmt), _stream(dev)))
    return (xq, xs, xqt, xst), (wq, ws, wqt)


def weight_128x128(w: torch.Tensor, q: torch.Tensor | None = None, s: torch.Tensor | None = None,
                   transposed: bool = False, qt: torch.Tensor | None = None, scale_fmt: str = "fp32"):
    """w[N,K] bf16 -> (q[N,K] uint8, s[N/128, K/128] fp32, qt[K,N] uint8 or None)."""
    _require(w, "w", torch.bfloat16, 2)
    N, K = w.shape
    q = _out(q, (N, K), torch.uint8, w.device, "q")
    s = _out(s, (N // 128, K // 128), torch.float32, w.device, "s")
    if transposed or qt is not None:
        qt = _out(qt, (K, N), torch.uint8, w.device, "qt")
    if scale_fmt == "fp32":
        _check("fp8q_weight_128x128",
               lib().fp8q_weight_128x128(_p(w), N, K, _p(q), _p(s), _p(qt), _stream(w.device)))
    else:
        _check("fp8q_weight_128x128_fmt",
               lib().fp8q_weight_128x128_fmt(_p(w), N, K, _p(q), _p(s), _p(qt), _fmt(scale_fmt), _stream(w.device)))
    return q, s, qt


# ------------------------------------------------------------------------------------------ #
# GEMMs
# ------------------------------------------------------------------------------------------ #

_workspaces: dict = {}


def gemm_workspace(mode: int, M: int, N: int, K: int, device: torch.device) -> torch.Tensor | None:
    """The stream-K workspace a call of this size may use (None if not needed).

    Cached per (device, current stream): calls queued on one stream run one after another and may
    share a workspace, calls on different streams may overlap on the GPU and get their own.  The
    cache holds the tensor, so a stream's workspace lives as long as the process (or until a
    larger call replaces it)."""
    nbytes = int(lib().fp8q_gemm_workspace_size(int(mode), M, N, K))
    if nbytes == 0:
        return None
    index = device.index if device.index is not None else torch.cuda.current_device()
    key = (index, torch.cuda.current_stream(index).cuda_stream)
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=torch.device("cuda", index))
        _workspaces[key] = ws
    return ws


def _gemm(entry: str, mode: int, A: torch.Tensor, sA: torch.Tensor, B: torch.Tensor, sB: torch.Tensor,
          out: torch.Tensor | None, workspace: torch.Tensor | None):
    """Shared marshalling of fp8_gemm_blockscaled and fp8_gemm_blockscaled_ue8m0 (same arguments)."""
    if mode == WGRAD_ACC and out is None:
        raise ValueError("WGRAD_ACC accumulates into `out`: pass the fp32 gradient to add to")
    _require(A, "A", torch.uint8, 2)
    _require(B, "B", torch.uint8, 2)
    _require(sA, "sA", torch.float32, 2)
    _require(sB, "sB", torch.float32, 2)
    M, K = A.shape
    N = B.shape[1] if mode == DGRAD else B.shape[0]
    Kb = B.shape[0] if mode == DGRAD else B.shape[1]
    if Kb != K:
        raise ValueError(f"inner dimensions differ: A has K={K}, B has {Kb}")
    dtype = torch.float32 if mode in (WGRAD, WGRAD_ACC) else torch.bfloat16
    out = _out(out, (M, N), dtype, A.device, "out")
    if workspace is None:
        workspace = gemm_workspace(mode, M, N, K, A.device)
    ws_ptr, ws_bytes = (None, 0) if workspace is None else (_p(workspace), workspace.numel())
    _check(entry, getattr(lib(), entry)(int(mode), _p(A), _p(sA), _p(B), _p(sB), _p(out), M, N, K,
                                        ws_ptr, ws_bytes, _stream(A.device)))
    return out


def gemm_blockscaled(mode: int, A: torch.Tensor, sA: torch.Tensor, B: torch.Tensor,
                     sB: torch.Tensor, out: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None):
    """Block-scaled FP8 GEMM.  FPROP: B = W[N,K]; DGRAD: B = W[K,N]; WGRAD: B = X^T[N,K];
    WGRAD_ACC: as WGRAD, added into `out` (required, fp32).
    Returns D[M,N] (bf16, or fp32 for WGRAD / WGRAD_ACC).  `workspace` (uint8, CUDA) enables the
    stream-K schedule; by default one workspace per (device, stream), sized by
    fp8q_gemm_workspace_size, is used.  A workspace passed explicitly must not be shared by GEMMs
    that may run concurrently."""
    return _gemm("fp8_gemm_blockscaled", mode, A, sA, B, sB, out, workspace)


def gemm_blockscaled_ue8m0(mode: int, A: torch.Tensor, sA: torch.Tensor, B: torch.Tensor,
                           sB: torch.Tensor, out: torch.Tensor | None = None,
                           workspace: torch.Tensor | None = None):
    """The GEMM of gemm_blockscaled for power-of-two scales (the scale_fmt="ue8m0" quantisers'):
    the tensor core applies them inside the MMA (tcgen05 kind::mxf8f6f4) and accumulates the
    whole K in FP32.  Same arguments and layouts; a scale that is not a power of two latches
    DEV_BAD_SCALES (see device_status)."""
    return _gemm("fp8_gemm_blockscaled_ue8m0", mode, A, sA, B, sB, out, workspace)


def gemm_blockscaled_quant(mode: int, A: torch.Tensor, sA: torch.Tensor, B: torch.Tensor,
                           sB: torch.Tensor, out: torch.Tensor | None = None, q: torch.Tensor | None = None,
                           s: torch.Tensor | None = None, store_out: bool = True,
                           workspace: torch.Tensor | None = None):
    """FPROP / DGRAD that also returns the 1x128 E4M3 codes and scales of its bf16 output (as
    act_1x128 would compute them from it).  Returns (D or None, q[M,N] uint8, s[N/128, M] fp32);
    store_out=False skips writing the bf16 D."""
    if mode not in (FPROP, DGRAD):
        raise ValueError("the fused output quantisation exists for FPROP and DGRAD")
    _require(A, "A", torch.uint8, 2)
    _require(B, "B", torch.uint8, 2)
    _require(sA, "sA", torch.float32, 2)
    _require(sB, "sB", torch.float32, 2)
    M, K = A.shape
    N = B.shape[1] if mode == DGRAD else B.shape[0]
    dev = A.device
    if store_out:
        out = _out(out, (M, N), torch.bfloat16, dev, "out")
    else:
        out = None
    q = _out(q, (M, N), torch.uint8, dev, "q")
    s = _out(s, (N // 128, M), torch.float32, dev, "s")
    if workspace is None:
        workspace = gemm_workspace(mode, M, N, K, dev)
    ws_ptr, ws_bytes = (None, 0) if workspace is None else (_p(workspace), workspace.numel())
    _check("fp8_gemm_blockscaled_quant",
           lib().fp8_gemm_blockscaled_quant(int(mode), _p(A), _p(sA), _p(B), _p(sB), _p(out), _p(q), _p(s),
                                            M, N, K, ws_ptr, ws_bytes, _stream(dev)))
    return out, q, s


def grouped_gemm_blockscaled(A: torch.Tensor, sA: torch.Tensor, B: torch.Tensor,
                             sB: torch.Tensor, offsets: torch.Tensor,
                             out: torch.Tensor | None = None):
    """Grouped Fprop: A[Mtot,K], sA[K/128,Mtot], B[E,N,K], sB[E,N/128,K/128],
    offsets int32[E+1] on the device.  Returns D[Mtot,N] bf16."""
    _require(A, "A", torch.uint8, 2)
    _require(B, "B", torch.uint8, 3)
    _require(sA, "sA", torch.float32, 2)
    _require(sB, "sB", torch.float32, 3)
    _require(offsets, "offsets", torch.int32, 1)
    Mtot, K = A.shape
    E, N, Kb = B.shape
    if Kb != K:
        raise ValueError("inner dimensions differ")
    if offsets.numel() != E + 1:
        raise ValueError("offsets must have E+1 entries")
    out = _out(out, (Mtot, N), torch.bfloat16, A.device, "out")
    _check("fp8_grouped_gemm_blockscaled",
           lib().fp8_grouped_gemm_blockscaled(_p(A), _p(sA), _p(B), _p(sB), _p(offsets), E, Mtot,
                                              N, K, _p(out), _stream(A.device)))
    return out


def grouped_gemm_blockscaled_dgrad(A: torch.Tensor, sA: torch.Tensor, B: torch.Tensor,
                                   sB: torch.Tensor, offsets: torch.Tensor,
                                   out: torch.Tensor | None = None):
    """Grouped Dgrad: A = dY codes [Mtot,K], sA[K/128,Mtot], B = forward expert weights
    [E,K,N] (out = K, in = N), sB[E,K/128,N/128], offsets int32[E+1] on the device.
    Returns dX[Mtot,N] bf16."""
    _require(A, "A", torch.uint8, 2)
    _require(B, "B", torch.uint8, 3)
    _require(sA, "sA", torch.float32, 2)
    _require(sB, "sB", torch.float32, 3)
    _require(offsets, "offsets", torch.int32, 1)
    Mtot, K = A.shape
    E, Kb, N = B.shape
    if Kb != K:
        raise ValueError("inner dimensions differ")
    if offsets.numel() != E + 1:
        raise ValueError("offsets must have E+1 entries")
    out = _out(out, (Mtot, N), torch.bfloat16, A.device, "out")
    _check("fp8_grouped_gemm_blockscaled_dgrad",
           lib().fp8_grouped_gemm_blockscaled_dgrad(_p(A), _p(sA), _p(B), _p(sB), _p(offsets), E, Mtot,
                                                    N, K, _p(out), _stream(A.device)))
    return out


def ragged_capacity(Mtot: int, E: int) -> int:
    """A padded token extent that fits any routing of Mtot rows over E experts."""
    return 128 * ((Mtot + 127) // 128 + E)


def act_128x1_transposed_ragged(x: torch.Tensor, offsets: torch.Tensor, Kcap: int | None = None,
                                qt: torch.Tensor | None = None, s: torch.Tensor | None = None):
    """x[Mtot,C] bf16 rows grouped by expert (offsets int32[E+1] on the device) ->
    (qt[C,Kcap] uint8, s[Kcap/128, C] fp32), each expert's 128-token groups padded to whole groups."""
    _require(x, "x", torch.bfloat16, 2)
    _require(offsets, "offsets", torch.int32, 1)
    Mtot, C = x.shape
    E = offsets.numel() - 1
    Kcap = ragged_capacity(Mtot, E) if Kcap is None else Kcap
    qt = _out(qt, (C, Kcap), torch.uint8, x.device, "qt")
    s = _out(s, (Kcap // 128, C), torch.float32, x.device, "s")
    _check("fp8q_act_128x1_transposed_ragged",
           lib().fp8q_act_128x1_transposed_ragged(_p(x), _p(offsets), E, Mtot, C, _p(qt), _p(s), Kcap,
                                                  _stream(x.device)))
    return qt, s


def grouped_gemm_blockscaled_wgrad(A: torch.Tensor, sA: torch.Tensor, B: torch.Tensor,
                                   sB: torch.Tensor, offsets: torch.Tensor, Mtot: int,
                                   out: torch.Tensor | None = None):
    """Grouped Wgrad: A = dY^T codes [M,Kcap], sA[Kcap/128,M], B = X^T codes [N,Kcap],
    sB[Kcap/128,N] (both from act_128x1_transposed_ragged with the same offsets over Mtot
    tokens).  Returns dW[E,M,N] fp32."""
    _require(A, "A", torch.uint8, 2)
    _require(B, "B", torch.uint8, 2)
    _require(sA, "sA", torch.float32, 2)
    _require(sB, "sB", torch.float32, 2)
    _require(offsets, "offsets", torch.int32, 1)
    M, Kcap = A.shape
    N, Kb = B.shape
    if Kb != Kcap:
        raise ValueError("A and B must share the padded token extent")
    E = offsets.numel() - 1
    out = _out(out, (E, M, N), torch.float32, A.device, "out")
    _check("fp8_grouped_gemm_blockscaled_wgrad",
           lib().fp8_grouped_gemm_blockscaled_wgrad(_p(A), _p(sA), _p(B), _p(sB), _p(offsets), E, Mtot, M, N,
                                                    Kcap, _p(out), _stream(A.device)))
    return out


def device_status(device: torch.device | None = None) -> int:
    """Synchronise the current stream and return (and clear) the device status word."""
    device = device or torch.device("cuda", torch.cuda.current_device())
    v = ctypes.c_int(-1)
    _check("fp8q_device_status", lib().fp8q_device_status(_stream(device), ctypes.byref(v)))
    return int(v.value)


def selftest_wait_timeout(limit_ns: int = 10_000_000, device: torch.device | None = None) -> None:
    """Launch the timeout self-test kernel (see include/fp8q.h)."""
    device = device or torch.device("cuda", torch.cuda.current_device())
    _check("fp8q_selftest_wait_timeout",
           lib().fp8q_selftest_wait_timeout(int(limit_ns), _stream(device)))

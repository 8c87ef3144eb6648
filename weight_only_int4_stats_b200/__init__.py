"""AWQ hot path on B200: a thin Python binding over libawq_b200.so (include/awq.h).

Every function here only marshals arguments: it checks dtypes, allocates outputs and the
workspace with PyTorch (device memory and the current stream are PyTorch's), and calls the
C entry point of the same name. All arithmetic runs in the library's CUDA kernels. There is
no fallback: if the library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "AwqError", "lib", "load_library", "library_path", "GROUP",
    "awq_act_stats", "awq_act_stats_noalloc", "awq_quantize_pack", "awq_search_scale", "awq_gemm_w4a16",
    "awq_silu_mul_gemm",
    "awq_check_error", "packed_words_per_row", "WEIGHTS_READY", "BF16",
]

GROUP = 128
_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libawq_b200.so")

STATUS = {0: "AWQ_OK", 1: "AWQ_ERR_INVALID_ARG", 2: "AWQ_ERR_UNSUPPORTED",
          3: "AWQ_ERR_WORKSPACE", 4: "AWQ_ERR_CUDA", 5: "AWQ_ERR_TIMEOUT", 6: "AWQ_ERR_BOUNDS"}


class AwqError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)}")
        self.code = code
        self.status = STATUS.get(code, str(code))


_lib = None


def load_library(path: str) -> ctypes.CDLL:
    """Loads a build of the library (the release build, or the bounds-checking debug build)
    and declares every entry point's signature. Raises ImportError if it is missing."""
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with "
            "`python -m weight_only_int4_stats_b200.build` (there is no CPU fallback)")
    L = ctypes.CDLL(path)
    P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    sig = {
        "awq_status_string": (ctypes.c_char_p, [I32]),
        "awq_abi_version": (I32, []),
        "awq_check_error": (I32, [P]),
        "awq_selftest_timeout": (I32, [P, P]),
        "awq_selftest_bounds": (I32, [P, P]),
        "awq_trace_reset": (I32, []),
        "awq_trace_read": (I32, [P, I64, P]),
        "awq_act_stats_workspace_size": (SZ, [I64, I64]),
        "awq_act_stats": (I32, [P, I64, I64, P, P, SZ, P]),
        "awq_act_stats_noalloc": (I32, [P, I64, I64, P, P]),
        "awq_quantize_pack": (I32, [P, I64, I64, P, I32, I32, P, P, P, P]),
        "awq_search_scale_workspace_size": (SZ, [I64, I64, I64, I32]),
        "awq_search_scale": (I32, [P, I64, I64, P, I64, P, P, I32, I32, I32, P, P, P, P, P,
                                   P, P, SZ, P]),
        "awq_gemm_workspace_size": (SZ, [I64, I64, I64, I32]),
        "awq_silu_mul_gemm": (I32, [P, I64, P, P, I64, I64, P, P]),
        "awq_gemm_w4a16": (I32, [P, I64, P, P, P, I64, I64, I32, I32, P, ctypes.c_uint, P,
                                 P, SZ, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


def lib() -> ctypes.CDLL:
    """The loaded CUDA library (loaded on first use; raises if it was never built)."""
    global _lib
    if _lib is None:
        _lib = load_library(library_path)
    return _lib


def use_library(path: str) -> ctypes.CDLL:
    """Makes the build at `path` (e.g. the trace build) the one every call of this module
    goes through, and returns it."""
    global _lib
    _lib = load_library(path)
    return _lib


def trace_read(max_ctas: int = 1 << 16):
    """The trace build's per-CTA timeline records since the last awq_trace_reset, as a
    [n, AWQ_TRACE_WORDS] uint64 numpy array (see include/awq.h). Raises AwqError with
    AWQ_ERR_UNSUPPORTED on a build without the timeline."""
    import numpy as np
    words = 32
    out = np.zeros((max_ctas, words), dtype=np.uint64)
    n = ctypes.c_int64(0)
    _check("awq_trace_read", lib().awq_trace_read(ctypes.c_void_p(out.ctypes.data), max_ctas,
                                                  ctypes.byref(n)))
    return out[:min(n.value, max_ctas)]


def trace_reset():
    """Clears the trace build's timeline records."""
    _check("awq_trace_reset", lib().awq_trace_reset())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn: str, code: int):
    if code != 0:
        raise AwqError(fn, code)


def _need(t, dtype, name):
    if t is None:
        return
    if t.dtype != dtype or not t.is_cuda or not t.is_contiguous():
        raise TypeError(f"{name}: expected a contiguous CUDA tensor of {dtype}, got "
                        f"{t.dtype} on {t.device} (contiguous={t.is_contiguous()})")


def _workspace(nbytes: int, device):
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


def packed_words_per_row(K: int, bits: int) -> int:
    return K // 8 if bits == 4 else 3 * K // 32


def awq_check_error(stream=None) -> None:
    _check("awq_check_error", lib().awq_check_error(_stream(stream)))


def awq_act_stats(X: torch.Tensor, out: torch.Tensor | None = None, workspace=None,
                  stream=None) -> torch.Tensor:
    """s_x[k] = mean_m |X[m, k]| (fp32 [K]) for fp16 X [M, K]."""
    _need(X, torch.float16, "X")
    M, K = X.shape
    s_x = torch.empty(K, dtype=torch.float32, device=X.device) if out is None else out
    _need(s_x, torch.float32, "out")
    ws_bytes = lib().awq_act_stats_workspace_size(M, K)
    ws = _workspace(ws_bytes, X.device) if workspace is None else workspace
    _check("awq_act_stats", lib().awq_act_stats(_ptr(X), M, K, _ptr(s_x), _ptr(ws),
                                                ws.numel() * ws.element_size(), _stream(stream)))
    return s_x


def awq_act_stats_noalloc(X: torch.Tensor, out: torch.Tensor | None = None,
                          stream=None) -> torch.Tensor:
    """awq_act_stats without a workspace: the library's own fixed device array holds the
    partial sums (K <= 65536; calls that overlap on the GPU race on that array)."""
    _need(X, torch.float16, "X")
    M, K = X.shape
    s_x = torch.empty(K, dtype=torch.float32, device=X.device) if out is None else out
    _need(s_x, torch.float32, "out")
    _check("awq_act_stats_noalloc",
           lib().awq_act_stats_noalloc(_ptr(X), M, K, _ptr(s_x), _stream(stream)))
    return s_x


def awq_quantize_pack(W: torch.Tensor, s: torch.Tensor | None, bits: int = 4,
                      group: int = GROUP, out=None, stream=None):
    """Quantize W diag(s) group-wise and pack: (qweight uint32 as int32, scales fp16 [G, N],
    zeros uint8 [G, N])."""
    _need(W, torch.float16, "W")
    _need(s, torch.float32, "s")
    N, K = W.shape
    dev = W.device
    if out is None:
        qweight = torch.empty(N, packed_words_per_row(K, bits), dtype=torch.int32, device=dev)
        scales = torch.empty(K // group, N, dtype=torch.float16, device=dev)
        zeros = torch.empty(K // group, N, dtype=torch.uint8, device=dev)
    else:
        qweight, scales, zeros = out
    _check("awq_quantize_pack", lib().awq_quantize_pack(
        _ptr(W), N, K, _ptr(s), bits, group, _ptr(qweight), _ptr(scales), _ptr(zeros),
        _stream(stream)))
    return qweight, scales, zeros


def awq_search_scale(W: torch.Tensor, X: torch.Tensor, s_x: torch.Tensor | None,
                     alphas: torch.Tensor | None, bits: int = 4, group: int = GROUP,
                     s_table: torch.Tensor | None = None, row_losses: bool = False,
                     workspace=None, stream=None, inv: bool = False):
    """Grid search of the per-channel scale. Returns (losses fp64 [A], best_idx int32 [1],
    best_s fp32 [K], row_losses fp64 [A, N] or None), and with ``inv=True`` a fifth item,
    best_inv_s fp32 [K] = 1 / best_s (the GEMM's inv_s for a layer packed with best_s)."""
    _need(W, torch.float16, "W")
    _need(X, torch.float16, "X")
    _need(s_x, torch.float32, "s_x")
    _need(alphas, torch.float32, "alphas")
    _need(s_table, torch.float32, "s_table")
    N, K = W.shape
    M = X.shape[0]
    A = alphas.numel() if alphas is not None else s_table.shape[0]
    dev = W.device
    losses = torch.empty(A, dtype=torch.float64, device=dev)
    best_idx = torch.empty(4, dtype=torch.int32, device=dev)
    best_s = torch.empty(K, dtype=torch.float32, device=dev)
    rl = torch.empty(A, N, dtype=torch.float64, device=dev) if row_losses else None
    best_inv = torch.empty(K, dtype=torch.float32, device=dev) if inv else None
    ws_bytes = lib().awq_search_scale_workspace_size(M, N, K, A)
    ws = _workspace(ws_bytes, dev) if workspace is None else workspace
    _check("awq_search_scale", lib().awq_search_scale(
        _ptr(W), N, K, _ptr(X), M, _ptr(s_x), _ptr(alphas), A, bits, group, _ptr(s_table),
        _ptr(losses), _ptr(best_idx), _ptr(best_s), _ptr(best_inv), _ptr(rl), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))
    if inv:
        return losses, best_idx[:1], best_s, rl, best_inv
    return losses, best_idx[:1], best_s, rl


WEIGHTS_READY = 1   # AWQ_GEMM_WEIGHTS_READY
BF16 = 2            # AWQ_GEMM_BF16


def awq_gemm_w4a16(X: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor,
                   zeros: torch.Tensor, N: int, K: int, bits: int = 4, group: int = GROUP,
                   inv_s: torch.Tensor | None = None, out: torch.Tensor | None = None,
                   workspace=None, stream=None, weights_ready: bool = False) -> torch.Tensor:
    """Y = X deq(W)^T ([M, N], X's dtype) with the dequantization fused into the kernel.

    X may be fp16 or bf16 (AWQ_GEMM_BF16); Y has X's dtype. ``weights_ready=True`` passes
    AWQ_GEMM_WEIGHTS_READY: the packed weights are not written by the kernel launched just
    before this call on the stream, so the kernel may start reading them while that kernel
    still runs."""
    bf16 = X.dtype == torch.bfloat16
    _need(X, torch.bfloat16 if bf16 else torch.float16, "X")
    _need(scales, torch.float16, "scales")
    _need(zeros, torch.uint8, "zeros")
    _need(inv_s, torch.float32, "inv_s")
    M = X.shape[0]
    Y = torch.empty(M, N, dtype=X.dtype, device=X.device) if out is None else out
    _need(Y, X.dtype, "out")
    ws = workspace
    if ws is None:
        need = lib().awq_gemm_workspace_size(M, N, K, bits)
        ws = _workspace(need, X.device) if need > 0 else None
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("awq_gemm_w4a16", lib().awq_gemm_w4a16(
        _ptr(X), M, _ptr(qweight), _ptr(scales), _ptr(zeros), N, K, bits, group, _ptr(inv_s),
        (WEIGHTS_READY if weights_ready else 0) | (BF16 if bf16 else 0), _ptr(Y), _ptr(ws),
        ws_bytes, _stream(stream)))
    return Y


def awq_silu_mul_gemm(X: torch.Tensor, W_gate: torch.Tensor, W_up: torch.Tensor,
                      out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """H = silu(X W_gate^T) * (X W_up^T) (fp16 [M, I]): the input of a gated MLP's down
    projection, computed from the full-precision weights for calibration."""
    _need(X, torch.float16, "X")
    _need(W_gate, torch.float16, "W_gate")
    _need(W_up, torch.float16, "W_up")
    M, K = X.shape
    I = W_gate.shape[0]
    if W_up.shape != W_gate.shape or W_gate.shape[1] != K:
        raise ValueError("W_gate and W_up must both be [I, K]")
    H = torch.empty(M, I, dtype=torch.float16, device=X.device) if out is None else out
    _need(H, torch.float16, "out")
    _check("awq_silu_mul_gemm", lib().awq_silu_mul_gemm(
        _ptr(X), M, _ptr(W_gate), _ptr(W_up), I, K, _ptr(H), _stream(stream)))
    return H

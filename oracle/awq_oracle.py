"""Plain, slow CPU definition of the AWQ hot path.

TEST INFRASTRUCTURE ONLY. Nothing in the product library imports or calls this module;
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may.
It shares no code with the CUDA path.

Sources (the pages are the authority on what is computed):

* robotsatlas.com "AWQ", section "How it works": a calibration set is passed through the
  layer and the activation magnitude of every input channel is measured; salient channels'
  weights are multiplied by a per-channel scale and the matching activation divided by it,
  which leaves the matmul unchanged; the scale is picked by a grid search that minimises the
  layer's output error; the weights are then quantized group-wise to 4 bits.
* robotsatlas.com "AWQ", section "Components" (Activation saliency analysis, Per-channel
  scaling, Group-wise 4-bit quantization: groups of e.g. 128 with a per-group scale) and
  section "Hyperparameters" (bit width 4 or 3, group size 128).
* builderai.tools "AWQ", section "About": the repository writes real INT4 weights and ships
  kernels for 4-bit weights with 16-bit activations.

The pages leave the exact formulas open. The readings taken here (each is stated where it
is used): s_x = mean |x| over all calibration tokens; s = max(s_x, 1e-4)^alpha on the grid
alpha_i = i/20, i = 0..19; asymmetric codes with an integer zero point per (row, group);
the per-group scale is rounded to fp16 and the codes are made with that rounded value;
round-half-to-even everywhere; the output error is the squared Frobenius norm
||Q(W diag(s)) diag(1/s) X^T - W X^T||^2 summed over every row of the searched weight.

Precision: statistics, dequantized weights, losses and GEMM outputs are exact or fp64.
The quantizer's decisions (min/max, scale, zero point, codes) are taken in IEEE fp32 with
one rounding per operation, in the order written below, because those decisions are
integers and both sides of a parity check must take them in the same precision.

Packed layouts (this library's convention; the pages fix only "group-wise 4-bit with a
per-group scale"):

* 4-bit: ``qweight`` uint32 [N, K/8]; word j of row n holds k = 8j..8j+7. Code of k-offset
  i (0..7) sits in nibble position p = i//2 + 4*(i%2) (bits 4p..4p+3), so nibble positions
  0..7 hold k-offsets 0,2,4,6,1,3,5,7: a mask of 0x000F000F picks the pair (k0, k1) into
  the two 16-bit halves of the word, 0x00F000F0 picks (k2, k3), and the same masks on the
  word shifted right by 8 pick (k4, k5) and (k6, k7).
* 3-bit: ``qweight`` uint32 [N, 3K/32]; each block of 32 consecutive k takes three words.
  Word 0 holds the low two bits of k-offsets 0..15, word 1 those of 16..31, each offset i
  (taken mod 16) at bits 2p..2p+1 with p = i//2 + 8*(i%2); word 2 holds bit 2 of all 32
  offsets, offset i at bit p = i//2 + 16*(i%2).
* ``scales`` float16 [K/g, N] and ``zeros`` uint8 [K/g, N], group-major.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "alpha_grid",
    "act_stats",
    "scale_candidates",
    "quantize",
    "dequantize",
    "pack",
    "unpack",
    "quantize_pack",
    "output_error",
    "search_losses",
    "search_scale",
    "gemm_w4a16",
    "silu_mul",
    "packed_words_per_row",
]

S_X_FLOOR = np.float32(1e-4)     # dead channels: s_x is clamped before the power
SCALE_FLOOR = np.float32(1e-5)   # degenerate groups (max == min)


def alpha_grid(n: int = 20) -> np.ndarray:
    """The search grid alpha_i = i / n, i = 0..n-1, each an fp32 quotient."""
    return np.arange(n, dtype=np.float32) / np.float32(n)


def act_stats(X: np.ndarray) -> np.ndarray:
    """Per-input-channel activation magnitude s_x[k] = (1/M) sum_m |x[m, k]|.

    robotsatlas "AWQ", "How it works" / "Components: Activation saliency analysis". The sum
    and the division are fp64; the result is rounded once to fp32.
    """
    X = np.asarray(X)
    assert X.ndim == 2 and X.shape[0] > 0
    total = np.abs(X.astype(np.float64)).sum(axis=0)
    return (total / np.float64(X.shape[0])).astype(np.float32)


def scale_candidates(s_x: np.ndarray, alphas: np.ndarray) -> np.ndarray:
    """s_alpha[k] = max(s_x[k], 1e-4)^alpha for every grid point, fp32 [n_alpha, K].

    robotsatlas "AWQ", "How it works" ("For each channel it derives a scaling factor") and
    "Key mechanisms" (grid search over scales). The power is taken in fp64 and rounded once
    to fp32; alpha = 0 gives exactly 1.
    """
    base = np.maximum(np.asarray(s_x, np.float32), S_X_FLOOR).astype(np.float64)
    a = np.asarray(alphas, np.float32).astype(np.float64)
    return np.power(base[None, :], a[:, None]).astype(np.float32)


def quantize(W: np.ndarray, s: np.ndarray | None, bits: int, group: int):
    """Group-wise asymmetric quantization of W diag(s).

    robotsatlas "AWQ", "Components: Group-wise 4-bit quantization" (groups of e.g. 128, one
    scale per group) and "Hyperparameters" (4 or 3 bits). Per row n and group j of ``group``
    consecutive input channels, in fp32 with one rounding per operation:

        w'    = w * s[k]                       (s = 1 when ``s`` is None: plain RTN)
        mx,mn = max and min of w' over the group
        scale = max((mx - mn) / qmax, 1e-5),  qmax = 2^bits - 1
        sc    = fp32(fp16(scale))              (the stored scale is the one used)
        z     = clamp(rint(-mn / sc), 0, qmax)
        q     = clamp(rint(w' / sc) + z, 0, qmax)

    Returns codes uint8 [N, K], scales float16 [K/g, N], zeros uint8 [K/g, N].
    """
    W = np.asarray(W)
    N, K = W.shape
    assert bits in (3, 4) and K % group == 0
    qmax = np.float32(2 ** bits - 1)
    w = W.astype(np.float32)
    if s is not None:
        w = w * np.asarray(s, np.float32)[None, :]
    wg = w.reshape(N, K // group, group)
    mx = wg.max(axis=2)
    mn = wg.min(axis=2)
    scale = (mx - mn) / qmax
    scale = np.maximum(scale, SCALE_FLOOR)
    scale_h = scale.astype(np.float16)
    sc = scale_h.astype(np.float32)
    z = np.clip(np.rint(-mn / sc), np.float32(0), qmax)
    q = np.clip(np.rint(wg / sc[:, :, None]) + z[:, :, None], np.float32(0), qmax)
    codes = q.reshape(N, K).astype(np.uint8)
    return codes, np.ascontiguousarray(scale_h.T), np.ascontiguousarray(z.T.astype(np.uint8))


def dequantize(codes: np.ndarray, scales: np.ndarray, zeros: np.ndarray, group: int) -> np.ndarray:
    """deq[n, k] = (q[n, k] - z[j, n]) * scale[j, n] with j = k // group, exact in fp64."""
    N, K = codes.shape
    G = K // group
    sc = np.asarray(scales).astype(np.float64).T.reshape(N, G, 1)
    zz = np.asarray(zeros).astype(np.float64).T.reshape(N, G, 1)
    q = codes.astype(np.float64).reshape(N, G, group)
    return ((q - zz) * sc).reshape(N, K)


def packed_words_per_row(K: int, bits: int) -> int:
    return K // 8 if bits == 4 else 3 * K // 32


def _nibble_position(i: int) -> int:
    return i // 2 + 4 * (i % 2)


def _crumb_position(i: int) -> int:          # 2-bit field index inside a 3-bit low word
    return i // 2 + 8 * (i % 2)


def _plane_position(i: int) -> int:          # bit index inside the 3-bit high-bit word
    return i // 2 + 16 * (i % 2)


def pack(codes: np.ndarray, bits: int) -> np.ndarray:
    """Pack codes [N, K] (values < 2^bits) into the uint32 layout described at module top.

    builderai.tools "AWQ", "About": the method writes real INT4 weights.
    """
    codes = np.asarray(codes, dtype=np.uint32)
    N, K = codes.shape
    if bits == 4:
        assert K % 8 == 0
        c = codes.reshape(N, K // 8, 8)
        out = np.zeros((N, K // 8), np.uint32)
        for i in range(8):
            out |= c[:, :, i] << np.uint32(4 * _nibble_position(i))
        return out
    assert bits == 3 and K % 32 == 0
    c = codes.reshape(N, K // 32, 32)
    out = np.zeros((N, K // 32, 3), np.uint32)
    for i in range(32):
        lo = c[:, :, i] & np.uint32(3)
        hi = (c[:, :, i] >> np.uint32(2)) & np.uint32(1)
        out[:, :, i // 16] |= lo << np.uint32(2 * _crumb_position(i % 16))
        out[:, :, 2] |= hi << np.uint32(_plane_position(i))
    return out.reshape(N, 3 * K // 32)


def unpack(qweight: np.ndarray, bits: int, K: int) -> np.ndarray:
    """Inverse of :func:`pack`: uint8 codes [N, K]."""
    qweight = np.asarray(qweight, dtype=np.uint32)
    N = qweight.shape[0]
    if bits == 4:
        out = np.zeros((N, K // 8, 8), np.uint8)
        for i in range(8):
            out[:, :, i] = (qweight >> np.uint32(4 * _nibble_position(i))) & np.uint32(15)
        return out.reshape(N, K)
    w = qweight.reshape(N, K // 32, 3)
    out = np.zeros((N, K // 32, 32), np.uint8)
    for i in range(32):
        lo = (w[:, :, i // 16] >> np.uint32(2 * _crumb_position(i % 16))) & np.uint32(3)
        hi = (w[:, :, 2] >> np.uint32(_plane_position(i))) & np.uint32(1)
        out[:, :, i] = lo | (hi << np.uint32(2))
    return out.reshape(N, K)


def quantize_pack(W: np.ndarray, s: np.ndarray | None, bits: int, group: int):
    """quantize() followed by pack(): (qweight uint32, scales fp16 [G, N], zeros u8 [G, N])."""
    codes, scales, zeros = quantize(W, s, bits, group)
    return pack(codes, bits), scales, zeros


def output_error(W: np.ndarray, X: np.ndarray, Wq_scaled: np.ndarray, s: np.ndarray,
                 per_row: bool = False):
    """Layer output error of a (quantized) scaled weight, fp64.

    robotsatlas "AWQ", "How it works": the salient channel's weight is multiplied by the
    scale and the activation divided by it, so the scaled layer computes
    (Wq_scaled diag(1/s)) X^T; the error is its squared distance to W X^T:

        L = sum_m sum_n ( sum_k (Wq_scaled[n,k] / s[k] - w[n,k]) * x[m,k] )^2

    With ``per_row`` the sum over m only is returned, one value per row n.
    """
    E = np.asarray(Wq_scaled, np.float64) / np.asarray(s, np.float32).astype(np.float64)[None, :]
    E -= np.asarray(W).astype(np.float64)
    Y = np.asarray(X).astype(np.float64) @ E.T            # [M, N]
    sq = Y * Y
    return sq.sum(axis=0) if per_row else float(sq.sum())


def search_losses(W, X, s_x, alphas, bits: int, group: int, s_table=None, per_row=False):
    """Output error at every grid point: L_i = output_error(W, X, deq(Q(W diag(s_i))), s_i).

    robotsatlas "AWQ", "How it works" and "Key mechanisms": grid search over scales that
    minimises the layer's output error. ``s_table`` [n_alpha, K] replaces the powers of s_x
    (the same fp32 scales can then be fed to both sides of a parity check).
    """
    alphas = np.asarray(alphas, np.float32)
    S = np.asarray(s_table, np.float32) if s_table is not None else scale_candidates(s_x, alphas)
    out = []
    for i in range(len(alphas)):
        codes, scales, zeros = quantize(W, S[i], bits, group)
        deq = dequantize(codes, scales, zeros, group)
        out.append(output_error(W, X, deq, S[i], per_row=per_row))
    return np.array(out, dtype=np.float64)


def search_scale(W, X, s_x, alphas, bits: int, group: int, s_table=None):
    """The grid search: (losses fp64 [n_alpha], best index, best_s fp32 [K]).

    The best index is the first minimum (ties go to the smaller alpha).
    """
    alphas = np.asarray(alphas, np.float32)
    S = np.asarray(s_table, np.float32) if s_table is not None else scale_candidates(s_x, alphas)
    losses = search_losses(W, X, s_x, alphas, bits, group, s_table=S)
    best = int(np.argmin(losses))
    return losses, best, S[best].copy()


def gemm_w4a16(X, qweight, scales, zeros, N: int, K: int, bits: int, group: int, inv_s=None):
    """Y[m, n] = sum_k x[m, k] * deq[n, k] in fp64 (builderai.tools "AWQ", "About": kernels for
    4-bit weights with 16-bit activations). With ``inv_s`` the activation columns are first
    multiplied by it (the activation side of the per-channel scaling, robotsatlas "AWQ",
    "How it works")."""
    codes = unpack(qweight, bits, K)
    deq = dequantize(codes, scales, zeros, group)
    x = np.asarray(X).astype(np.float64)
    if inv_s is not None:
        x = x * np.asarray(inv_s, np.float32).astype(np.float64)[None, :]
    return x @ deq.T


def silu_mul(X, W_gate, W_up):
    """Input of a gated MLP's down projection: h = silu(g) * u with g = X W_gate^T,
    u = X W_up^T and silu(g) = g / (1 + exp(-g)), all in fp64 from the fp16 operands.

    robotsatlas "AWQ", "How it works": the calibration set is passed through the model, so each
    linear layer is calibrated on the activations that actually reach it. In the 7B-shaped
    decoder layer's MLP (a SiLU-gated MLP: this library's reading of the layer, which the
    pages do not spell out) the activations reaching down_proj are this gated product of the
    full-precision gate_proj and up_proj outputs.
    """
    x = np.asarray(X).astype(np.float64)
    g = x @ np.asarray(W_gate).astype(np.float64).T
    u = x @ np.asarray(W_up).astype(np.float64).T
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g)) * u

"""Plausible mistakes planted in the CPU oracle, to show that its pins catch them.

Each mutant replaces one oracle function (or helper) with a copy that differs by one slip
of the kind a reimplementation makes: a dropped absolute value, a flipped sign, an
off-by-one level count, a wrong bit position, a missing factor, a reversed comparison.
``install(name)`` patches the oracle module and the ``oracle`` package in place; it is
only called from ``tests/conftest.py`` when ``AWQ_ORACLE_MUTANT`` is set, in a separate
pytest process started by ``tests/test_oracle_mutations.py``. Nothing here runs on a GPU.
"""
import numpy as np

import oracle
from oracle import awq_oracle as A


def _quantize_variant(zero_sign=1.0, levels_offset=0, fp16_scale=True, rounding=np.rint,
                      clamp=True, scale_floor=True):
    """The oracle's quantizer with one step altered (see quantize() for the reference)."""
    def quantize(W, s, bits, group):
        W = np.asarray(W)
        N, K = W.shape
        qmax = np.float32(2 ** bits - 1)
        w = W.astype(np.float32)
        if s is not None:
            w = w * np.asarray(s, np.float32)[None, :]
        wg = w.reshape(N, K // group, group)
        mx = wg.max(axis=2)
        mn = wg.min(axis=2)
        scale = (mx - mn) / (qmax + np.float32(levels_offset))
        if scale_floor:
            scale = np.maximum(scale, A.SCALE_FLOOR)
        scale_h = scale.astype(np.float16)
        sc = scale_h.astype(np.float32) if fp16_scale else scale.astype(np.float32)
        with np.errstate(divide="ignore", invalid="ignore"):
            z = rounding(np.float32(zero_sign) * -mn / sc)
            q = rounding(wg / sc[:, :, None]) + z[:, :, None]
        if clamp:
            z = np.clip(z, np.float32(0), qmax)
            q = np.clip(rounding(wg / sc[:, :, None]) + z[:, :, None], np.float32(0), qmax)
        z = np.nan_to_num(z)
        q = np.nan_to_num(q)
        codes = q.reshape(N, K).astype(np.int64).astype(np.uint8)
        return (codes, np.ascontiguousarray(scale_h.T),
                np.ascontiguousarray(z.T.astype(np.int64).astype(np.uint8)))
    return quantize


def _act_stats_no_abs(X):
    X = np.asarray(X)
    return (X.astype(np.float64).sum(axis=0) / np.float64(X.shape[0])).astype(np.float32)


def _act_stats_m_minus_1(X):
    X = np.asarray(X)
    total = np.abs(X.astype(np.float64)).sum(axis=0)
    return (total / np.float64(max(X.shape[0] - 1, 1))).astype(np.float32)


def _scale_candidates_flipped(s_x, alphas):
    base = np.maximum(np.asarray(s_x, np.float32), A.S_X_FLOOR).astype(np.float64)
    a = np.asarray(alphas, np.float32).astype(np.float64)
    return np.power(base[None, :], 1.0 - a[:, None]).astype(np.float32)


def _scale_candidates_no_floor(s_x, alphas):
    base = np.asarray(s_x, np.float32).astype(np.float64)
    a = np.asarray(alphas, np.float32).astype(np.float64)
    with np.errstate(divide="ignore"):
        return np.power(base[None, :], a[:, None]).astype(np.float32)


def _dequantize_no_zero(codes, scales, zeros, group):
    N, K = codes.shape
    G = K // group
    sc = np.asarray(scales).astype(np.float64).T.reshape(N, G, 1)
    q = codes.astype(np.float64).reshape(N, G, group)
    return (q * sc).reshape(N, K)


def _dequantize_group_shift(codes, scales, zeros, group):
    # scales and zeros of group j applied to the next group's columns (an index slip)
    N, K = codes.shape
    G = K // group
    sc = np.roll(np.asarray(scales).astype(np.float64).T, 1, axis=1).reshape(N, G, 1)
    zz = np.roll(np.asarray(zeros).astype(np.float64).T, 1, axis=1).reshape(N, G, 1)
    q = codes.astype(np.float64).reshape(N, G, group)
    return ((q - zz) * sc).reshape(N, K)


def _output_error_no_inverse(W, X, Wq_scaled, s, per_row=False):
    E = np.asarray(Wq_scaled, np.float64) - np.asarray(W).astype(np.float64)
    Y = np.asarray(X).astype(np.float64) @ E.T
    sq = Y * Y
    return sq.sum(axis=0) if per_row else float(sq.sum())


def _output_error_weight_space(W, X, Wq_scaled, s, per_row=False):
    # the weight error alone, without the activations
    E = np.asarray(Wq_scaled, np.float64) / np.asarray(s, np.float32).astype(np.float64)[None, :]
    E -= np.asarray(W).astype(np.float64)
    sq = E * E
    return sq.sum(axis=1) if per_row else float(sq.sum())


def _search_scale_argmax(W, X, s_x, alphas, bits, group, s_table=None):
    alphas = np.asarray(alphas, np.float32)
    S = np.asarray(s_table, np.float32) if s_table is not None else A.scale_candidates(s_x, alphas)
    losses = A.search_losses(W, X, s_x, alphas, bits, group, s_table=S)
    best = int(np.argmax(losses))
    return losses, best, S[best].copy()


def _search_scale_last_minimum(W, X, s_x, alphas, bits, group, s_table=None):
    alphas = np.asarray(alphas, np.float32)
    S = np.asarray(s_table, np.float32) if s_table is not None else A.scale_candidates(s_x, alphas)
    losses = A.search_losses(W, X, s_x, alphas, bits, group, s_table=S)
    best = int(len(losses) - 1 - np.argmin(losses[::-1]))
    return losses, best, S[best].copy()


def _gemm_inv_s_ignored(X, qweight, scales, zeros, N, K, bits, group, inv_s=None):
    codes = A.unpack(qweight, bits, K)
    deq = A.dequantize(codes, scales, zeros, group)
    return np.asarray(X).astype(np.float64) @ deq.T


def _silu_mul_sign_slip(X, W_gate, W_up):
    # exp(+g) in the logistic: g * sigmoid(-g) instead of g * sigmoid(g)
    x = np.asarray(X).astype(np.float64)
    g = x @ np.asarray(W_gate).astype(np.float64).T
    u = x @ np.asarray(W_up).astype(np.float64).T
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(g)) * u


def _silu_mul_gate_up_swapped(X, W_gate, W_up):
    # the SiLU applied to up_proj's output instead of gate_proj's
    return A.__dict__["_silu_mul_reference"](X, W_up, W_gate)


MUTANTS = {
    "act_stats_abs_dropped": {"act_stats": _act_stats_no_abs},
    "act_stats_divides_by_m_minus_1": {"act_stats": _act_stats_m_minus_1},
    "scale_power_flipped": {"scale_candidates": _scale_candidates_flipped},
    "scale_floor_dropped": {"scale_candidates": _scale_candidates_no_floor},
    "zero_point_sign_flipped": {"quantize": _quantize_variant(zero_sign=-1.0)},
    "one_level_too_many": {"quantize": _quantize_variant(levels_offset=1)},
    "fp32_scale_used_not_stored_fp16": {"quantize": _quantize_variant(fp16_scale=False)},
    "floor_instead_of_round": {"quantize": _quantize_variant(rounding=np.floor)},
    "codes_not_clamped": {"quantize": _quantize_variant(clamp=False)},
    "scale_floor_missing": {"quantize": _quantize_variant(scale_floor=False)},
    "nibbles_not_interleaved": {"_nibble_position": lambda i: i},
    "crumbs_not_interleaved": {"_crumb_position": lambda i: i},
    "high_bits_not_interleaved": {"_plane_position": lambda i: i},
    "dequant_zero_point_ignored": {"dequantize": _dequantize_no_zero},
    "dequant_group_index_slip": {"dequantize": _dequantize_group_shift},
    "error_without_inverse_scale": {"output_error": _output_error_no_inverse},
    "error_in_weight_space": {"output_error": _output_error_weight_space},
    "search_picks_largest_loss": {"search_scale": _search_scale_argmax},
    "search_ties_go_to_largest_alpha": {"search_scale": _search_scale_last_minimum},
    "gemm_ignores_inv_s": {"gemm_w4a16": _gemm_inv_s_ignored},
    "silu_sign_slip": {"silu_mul": _silu_mul_sign_slip},
    "silu_on_up_not_gate": {"silu_mul": _silu_mul_gate_up_swapped},
}


def install(name: str) -> None:
    """Patch the named mutant into the oracle module and package."""
    if name == "none":
        return
    A._silu_mul_reference = A.silu_mul   # the unmutated function, for mutants that wrap it
    for attr, fn in MUTANTS[name].items():
        assert hasattr(A, attr), attr
        setattr(A, attr, fn)
        if hasattr(oracle, attr):
            setattr(oracle, attr, fn)

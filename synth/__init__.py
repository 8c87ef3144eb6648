"""Seeded synthetic inputs shaped like the Llama/Qwen-class layers the AWQ pages discuss.

This module only draws random numbers; it holds none of the method's arithmetic (no
statistics, no scales, no quantization). Both the CPU oracle's tests and the CUDA path's
tests and benchmark take their inputs from here, so the two sides see identical bytes.

Every generator uses ``numpy.random.default_rng`` on a ``SeedSequence`` built from the
workload's seed and the layer shape, and draws in the order its docstring lists. Normal
draws are made in float32 and cast to float16 (round to nearest even).

Workloads (names follow the pages' notation: W is [N, K] with N output features and K
input channels, X is [M, K] with M calibration or decode tokens):

* ``single_layer``      -- one 512x512 layer, 256 calibration tokens (seed 0).
* ``decode_layer``      -- decode GEMV shapes, M in {1, 4, 16} (seed 1).
* ``batched_layer``     -- batched decode / small prefill, M in {32..256} (seed 2).
* ``prefill_layer``     -- compute-bound prefill GEMMs, M in {2048..8192} (seed 3).
* ``decoder_layer``     -- one 7B-shaped decoder layer with its calibration batch (seed 4).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "channel_magnitudes",
    "single_layer",
    "decode_layer",
    "batched_layer",
    "prefill_layer",
    "decoder_layer_weights",
    "decoder_layer_activations",
    "random_weight",
    "random_activations",
    "DECODE_SHAPES",
    "DECODE_M",
    "BATCHED_SHAPES",
    "BATCHED_M",
    "PREFILL_SHAPES",
    "PREFILL_M",
]

DECODE_SHAPES = [(4096, 4096), (11008, 4096), (4096, 11008)]
DECODE_M = [1, 4, 16]
BATCHED_SHAPES = [(14336, 4096), (4096, 14336), (6144, 4096)]
BATCHED_M = [32, 64, 128, 256]
PREFILL_SHAPES = [(28672, 8192), (8192, 28672), (10240, 8192)]
PREFILL_M = [2048, 4096, 8192]


def _rng(*key: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(k) for k in key]))


def random_weight(rng: np.random.Generator, n: int, k: int, sigma: float) -> np.ndarray:
    """W ~ N(0, sigma^2) as float16 [n, k] (float32 draws, then cast)."""
    w = rng.standard_normal((n, k), dtype=np.float32)
    w *= np.float32(sigma)
    return w.astype(np.float16)


def channel_magnitudes(rng: np.random.Generator, k: int, sigma: float,
                       outlier_frac: float = 0.01, outlier_gain=(20.0, 20.0),
                       n_outliers: int | None = None) -> np.ndarray:
    """Per-input-channel magnitudes m_k ~ lognormal(0, sigma), float32 [k].

    A fraction ``outlier_frac`` of the channels (rounded, or exactly ``n_outliers``) is
    chosen without replacement and multiplied by a gain drawn uniformly from
    ``outlier_gain`` (a fixed gain when both ends are equal). Draw order: magnitudes,
    outlier indices, gains.
    """
    m = rng.lognormal(0.0, sigma, k)
    n_out = int(round(outlier_frac * k)) if n_outliers is None else int(n_outliers)
    idx = rng.choice(k, n_out, replace=False) if n_out > 0 else np.zeros(0, np.int64)
    lo, hi = outlier_gain
    gain = rng.uniform(lo, hi, n_out) if hi > lo else np.full(n_out, lo)
    m[idx] *= gain
    return m.astype(np.float32)


def random_activations(rng: np.random.Generator, m_rows: int, mag: np.ndarray | None,
                       chunk: int = 1 << 14) -> np.ndarray:
    """X = N(0, 1) [m_rows, k] times the channel magnitudes (if given), as float16.

    Rows are drawn in chunks (same stream order as a single draw) to bound host memory.
    """
    k = mag.shape[0] if mag is not None else None
    assert k is not None
    out = np.empty((m_rows, k), dtype=np.float16)
    for r0 in range(0, m_rows, chunk):
        r1 = min(m_rows, r0 + chunk)
        x = rng.standard_normal((r1 - r0, k), dtype=np.float32)
        x *= mag[None, :]
        out[r0:r1] = x.astype(np.float16)
    return out


def single_layer():
    """Seed 0: W [512, 512] ~ N(0, 0.02^2); m ~ lognormal(0, 0.5) [512] with 5 channels x20;
    X [256, 512] = N(0, 1) * m. Draw order: W, m, outlier indices, X."""
    rng = _rng(0, 512, 512)
    W = random_weight(rng, 512, 512, 0.02)
    m = channel_magnitudes(rng, 512, 0.5, n_outliers=5)
    X = random_activations(rng, 256, m)
    return W, X, m


def decode_layer(n: int, k: int, m_max: int = 16):
    """Seed 1, per shape [n, k]: W ~ N(0, 0.02^2); m ~ lognormal(0, 0.5) [k] with
    round(0.01 k) channels x20 (the per-channel scale s = m^0.5 is formed by the caller);
    X [m_max, k] ~ N(0, 1) (decode with M < m_max uses the first M rows)."""
    rng = _rng(1, n, k)
    W = random_weight(rng, n, k, 0.02)
    m = channel_magnitudes(rng, k, 0.5)
    X = random_activations(rng, m_max, np.ones(k, np.float32))
    return W, m, X


def batched_layer(n: int, k: int, m_max: int = 256):
    """Seed 2, per shape [n, k]: W ~ N(0, 0.02^2); m ~ lognormal(0, 0.5) with 1% of the
    channels x20; X [m_max, k] = N(0, 1) * m (smaller M use the first rows)."""
    rng = _rng(2, n, k)
    W = random_weight(rng, n, k, 0.02)
    m = channel_magnitudes(rng, k, 0.5)
    X = random_activations(rng, m_max, m)
    return W, m, X


def prefill_layer(n: int, k: int, m_rows: int):
    """Seed 3, per shape [n, k]: W ~ N(0, 0.015^2); m ~ lognormal(0, 0.5) with 1% x20
    (used for the quantization scale); X [m_rows, k] ~ N(0, 1)."""
    rng = _rng(3, n, k)
    W = random_weight(rng, n, k, 0.015)
    m = channel_magnitudes(rng, k, 0.5)
    X = random_activations(rng, m_rows, np.ones(k, np.float32))
    return W, m, X


_DECODER_LINEARS = [
    ("q_proj", 4096, 4096), ("k_proj", 4096, 4096), ("v_proj", 4096, 4096),
    ("o_proj", 4096, 4096), ("gate_proj", 11008, 4096), ("up_proj", 11008, 4096),
    ("down_proj", 4096, 11008),
]


def decoder_layer_weights(hidden: int = 4096, mlp: int = 11008):
    """Seed 4: the seven linears of a 7B-shaped decoder layer, all ~ N(0, 0.02^2), drawn
    in the order q, k, v, o, gate, up, down. Returns {name: W [N, K] float16}."""
    rng = _rng(4, hidden, mlp)
    shapes = {"q_proj": (hidden, hidden), "k_proj": (hidden, hidden),
              "v_proj": (hidden, hidden), "o_proj": (hidden, hidden),
              "gate_proj": (mlp, hidden), "up_proj": (mlp, hidden),
              "down_proj": (hidden, mlp)}
    return {name: random_weight(rng, *shapes[name], 0.02) for name, _, _ in _DECODER_LINEARS}


def decoder_layer_activations(tokens: int = 128 * 512, hidden: int = 4096, mlp: int = 11008,
                              names=("hidden", "o_in", "down_in"), rows: int | None = None):
    """Seed 4: the layer's three calibration inputs of ``tokens`` rows, each N(0, 1) times its
    own lognormal(0, 0.7) channel magnitudes with round(0.01 K) outlier channels multiplied
    by U(10, 50): the hidden state X (input of q/k/v and gate/up), X_o (input of o_proj) and
    X_d (input of down_proj). Each input has its own stream (SeedSequence [4, tokens, K, i],
    i = 0, 1, 2 in that order), drawing magnitudes, outlier indices, gains, then X, so any
    subset can be generated alone. ``rows`` draws only the first rows of the same inputs
    (normal draws fill row by row, so they are exactly the leading rows of the full batch)."""
    dims = {"hidden": (0, hidden), "o_in": (1, hidden), "down_in": (2, mlp)}
    out = {}
    for name in names:
        idx, k = dims[name]
        rng = _rng(4, tokens, k, idx)
        m = channel_magnitudes(rng, k, 0.7, outlier_gain=(10.0, 50.0))
        out[name] = random_activations(rng, tokens if rows is None else rows, m)
    return out

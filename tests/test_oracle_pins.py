"""Pins for the CPU oracle: each check ties it to something other than itself.

The pages print no worked example, so the pins are closed forms, exact invariants that the
pages state in words (the per-channel scaling leaves the matmul unchanged; the grid search
picks the lowest output error; AWQ is at least as good as plain rounding), hand-derived
values (tests/golden), library routines on special cases, and brute force on tiny inputs.
"""
import json
import math
import os
import struct

import numpy as np
import pytest
import torch

import oracle as O
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _f16(x: float) -> float:
    return struct.unpack("e", struct.pack("e", x))[0]


def _f32(x: float) -> float:
    return struct.unpack("f", struct.pack("f", x))[0]


# ----------------------------------------------------------------------------- act_stats

def test_act_stats_closed_form():
    # x[m, k] = (-1)^m (k + 1): the mean magnitude of column k is exactly k + 1.
    M, K = 6, 40
    m = np.arange(M)[:, None]
    k = np.arange(K)[None, :]
    X = (((-1.0) ** m) * (k + 1)).astype(np.float16)
    s = O.act_stats(X)
    assert s.dtype == np.float32
    np.testing.assert_array_equal(s, np.arange(1, K + 1, dtype=np.float32))


def test_act_stats_zero_column_and_brute_force():
    rng = np.random.default_rng(11)
    X = (rng.standard_normal((9, 16)) * 3).astype(np.float16)
    X[:, 5] = 0
    s = O.act_stats(X)
    assert s[5] == 0.0
    for k in range(16):
        col = [abs(float(X[i, k])) for i in range(9)]
        exact = math.fsum(col) / 9
        assert s[k] == np.float32(exact)


# ----------------------------------------------------------------------------- scale grid

def test_alpha_grid():
    a = O.alpha_grid(20)
    assert a.dtype == np.float32 and a.shape == (20,)
    assert a[0] == 0.0
    for i in range(20):
        assert a[i] == np.float32(np.float32(i) / np.float32(20))
    assert abs(float(a[19]) - 0.95) < 1e-7


def test_scale_candidates_special_cases():
    rng = np.random.default_rng(3)
    s_x = rng.lognormal(0, 1, 64).astype(np.float32)
    s_x[3] = 0.0                                   # dead channel
    S = O.scale_candidates(s_x, np.array([0.0, 1.0, 0.5], np.float32))
    assert np.all(S[0] == 1.0)                     # alpha = 0: no scaling at all
    base = np.maximum(s_x, np.float32(1e-4))
    np.testing.assert_array_equal(S[1], base)      # alpha = 1: s = s_x
    np.testing.assert_array_equal(S[2], np.sqrt(base.astype(np.float64)).astype(np.float32))
    assert S[1][3] == np.float32(1e-4)


# ----------------------------------------------------------------------------- quantizer

def _ramp_group():
    return np.array([[(k - 64) / 64 for k in range(128)]], np.float16)


@pytest.mark.parametrize("bits", [4, 3])
def test_quantize_handworked_group(bits):
    g = _load("handworked_group.json")["bits%d" % bits]
    W = _ramp_group()
    codes, scales, zeros = O.quantize(W, None, bits, 128)
    assert scales.shape == (1, 1) and zeros.shape == (1, 1)
    assert float(scales[0, 0]) == g["scale_fp16"]
    assert int(zeros[0, 0]) == g["zero"]
    for k, q in g["codes_at"].items():
        assert int(codes[0, int(k)]) == q, k
    deq = O.dequantize(codes, scales, zeros, 128)
    err = np.abs(deq - W.astype(np.float64)).max()
    assert err == g["max_abs_error"]
    assert err <= g["half_step"]
    if bits == 4:
        assert deq[0, 0] == g["deq_0"] and deq[0, 127] == g["deq_127"]
        word = O.pack(codes, 4)[0, 0]
        assert word == int(g["first_packed_word"], 16)


def _groups_straddling_zero(Wf, group):
    N, K = Wf.shape
    wg = Wf.reshape(N, K // group, group)
    return (wg.max(axis=2) >= 0) & (wg.min(axis=2) <= 0)


@pytest.mark.parametrize("bits", [4, 3])
@pytest.mark.parametrize("scaled", [False, True])
def test_quantize_invariants(bits, scaled):
    rng = np.random.default_rng(5 + bits)
    N, K, g = 24, 512, 128
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    s = rng.lognormal(0, 0.8, K).astype(np.float32) if scaled else None
    codes, scales, zeros = O.quantize(W, s, bits, g)
    qmax = 2 ** bits - 1
    assert codes.dtype == np.uint8 and codes.max() <= qmax
    assert scales.shape == (K // g, N) and zeros.shape == (K // g, N)
    assert zeros.max() <= qmax
    wprime = W.astype(np.float32) * (s if s is not None else np.float32(1))
    wp = wprime.astype(np.float64)
    deq = O.dequantize(codes, scales, zeros, g)
    sc = np.repeat(scales.astype(np.float64).T, g, axis=1)       # [N, K]
    zz = np.repeat(zeros.astype(np.float64).T, g, axis=1)
    # 1. the stored scale is the fp16 rounding of the fp32 (max - min) / qmax
    wg = wprime.reshape(N, K // g, g)
    for n in range(N):
        for j in range(K // g):
            span = _f32(float(wg[n, j].max()) - float(wg[n, j].min()))
            want = _f16(max(_f32(span / qmax), _f32(1e-5)))
            assert float(scales[j, n]) == want
    # 2. reconstruction error at most half a step in every group that straddles zero, for
    #    every code the clamp did not move; a clamped end of the range may lie further out
    #    only by the amount the fp16-rounded step falls short of (max - min) / qmax.
    strad = np.repeat(_groups_straddling_zero(wprime, g), g, axis=1)
    err = np.abs(deq - wp)
    unclamped = np.abs(np.rint(wp / sc) + zz - codes) == 0
    assert np.all(err[strad & unclamped] <= sc[strad & unclamped] / 2 * (1 + 2.0 ** -20))
    span = (wg.max(axis=2) - wg.min(axis=2)).astype(np.float64)
    short = np.repeat(np.maximum(0.0, span - qmax * scales.astype(np.float64).T), g, axis=1)
    assert np.all(short <= qmax * sc * 2.0 ** -11)
    assert np.all(err[strad] <= (sc / 2 + short)[strad] * (1 + 2.0 ** -20))
    # 3. each code is the nearest level: moving it by one never gets closer
    for d in (-1, 1):
        alt = codes.astype(np.float64) + d
        ok = (alt >= 0) & (alt <= qmax)
        alt_err = np.abs((alt - zz) * sc - wp)
        assert np.all(err[ok] <= alt_err[ok] * (1 + 2.0 ** -20) + 1e-12)
    # 4. the zero point sits within half a step of -min/scale (integer grid contains 0)
    mn = wprime.reshape(N, K // g, g).min(axis=2).T.astype(np.float64)
    assert np.all(np.abs(zeros * scales.astype(np.float64) + mn) <=
                  scales.astype(np.float64) / 2 * (1 + 2.0 ** -20))


def test_quantize_alpha_zero_is_plain_rtn():
    W, X, m = synth.single_layer()
    s0 = O.scale_candidates(O.act_stats(X), np.zeros(1, np.float32))[0]
    a = O.quantize(W, s0, 4, 128)
    b = O.quantize(W, None, 4, 128)
    for u, v in zip(a, b):
        np.testing.assert_array_equal(u, v)


def test_quantize_degenerate_groups():
    W = np.zeros((3, 128), np.float16)
    W[1, :] = 0.5                                  # constant positive group
    W[2, :] = -0.25                                # constant negative group
    codes, scales, zeros = O.quantize(W, None, 4, 128)
    floor16 = _f16(_f32(1e-5))
    assert np.all(scales.astype(np.float64) == floor16)
    assert zeros[0, 0] == 0 and np.all(codes[0] == 0)             # all-zero: exact
    assert np.all(O.dequantize(codes, scales, zeros, 128)[0] == 0.0)
    assert zeros[0, 1] == 0 and np.all(codes[1] == 15)            # clamps at qmax
    assert zeros[0, 2] == 15 and np.all(codes[2] == 0)            # clamps at 0


# ----------------------------------------------------------------------------- packing

def test_pack_golden_words():
    g = _load("packing_words.json")
    q = np.array([g["bits4_ramp"]["codes"]], np.uint8)
    assert O.pack(q, 4)[0, 0] == int(g["bits4_ramp"]["word"], 16)
    q = np.array([g["bits4_first_of_group"]["codes"]], np.uint8)
    assert O.pack(q, 4)[0, 0] == int(g["bits4_first_of_group"]["word"], 16)
    q = np.array([[i % 8 for i in range(32)]], np.uint8)
    words = O.pack(q, 3)[0]
    assert [int(w) for w in words] == [int(w, 16) for w in g["bits3_mod8"]["words"]]


@pytest.mark.parametrize("bits", [4, 3])
def test_pack_roundtrip_and_bit_positions(bits):
    rng = np.random.default_rng(17)
    N, K = 5, 256
    q = rng.integers(0, 2 ** bits, (N, K)).astype(np.uint8)
    pw = O.pack(q, bits)
    assert pw.dtype == np.uint32 and pw.shape == (N, O.packed_words_per_row(K, bits))
    np.testing.assert_array_equal(O.unpack(pw, bits, K), q)
    # read every field back through the raw little-endian bit stream
    bitstream = np.unpackbits(pw.view(np.uint8), axis=1, bitorder="little")
    for n in range(N):
        for k in range(K):
            i = k % (8 if bits == 4 else 32)
            if bits == 4:
                base = (k // 8) * 32 + 4 * (i // 2 + 4 * (i % 2))
                v = sum(int(bitstream[n, base + b]) << b for b in range(4))
            else:
                blk = (k // 32) * 96
                lo_base = blk + 32 * (i // 16) + 2 * ((i % 16) // 2 + 8 * (i % 2))
                hi_bit = blk + 64 + (i // 2 + 16 * (i % 2))
                v = int(bitstream[n, lo_base]) | (int(bitstream[n, lo_base + 1]) << 1) | \
                    (int(bitstream[n, hi_bit]) << 2)
            assert v == q[n, k]


@pytest.mark.parametrize("bits,expect", [(4, 4.1875), (3, 3.1875)])
def test_storage_bits_per_weight(bits, expect):
    # "~4.x bits per weight" (robotsatlas "AWQ", "Computational complexity")
    N, K = 64, 1024
    W = np.random.default_rng(0).standard_normal((N, K)).astype(np.float16)
    qw, sc, z = O.quantize_pack(W, None, bits, 128)
    bits_total = 8 * (qw.nbytes + sc.nbytes + z.nbytes)
    assert bits_total / (N * K) == expect


# ----------------------------------------------------------------------------- output error

def test_scaling_leaves_the_matmul_unchanged():
    # robotsatlas "AWQ", "How it works": weight x s and activation / s preserve the result.
    rng = np.random.default_rng(2)
    W = (rng.standard_normal((16, 256)) * 0.02).astype(np.float16)
    X = rng.standard_normal((8, 256)).astype(np.float16)
    s = rng.lognormal(0, 1.0, 256).astype(np.float32)
    Ws = W.astype(np.float64) * s.astype(np.float64)[None, :]
    assert O.output_error(W, X, Ws, s) == 0.0
    ref = X.astype(np.float64) @ W.astype(np.float64).T
    scaled = (X.astype(np.float64) / s.astype(np.float64)) @ Ws.T
    assert np.abs(scaled - ref).max() <= 1e-12 * np.abs(ref).max()


def test_output_error_brute_force():
    rng = np.random.default_rng(4)
    N, K, M = 3, 8, 4
    W = (rng.standard_normal((N, K)) * 0.1).astype(np.float16)
    X = rng.standard_normal((M, K)).astype(np.float16)
    s = rng.lognormal(0, 0.5, K).astype(np.float32)
    Wq = rng.standard_normal((N, K)) * 0.1
    total = []
    for m in range(M):
        for n in range(N):
            yq = math.fsum(Wq[n, k] / float(s[k]) * float(X[m, k]) for k in range(K))
            yr = math.fsum(float(W[n, k]) * float(X[m, k]) for k in range(K))
            total.append((yq - yr) ** 2)
    want = math.fsum(total)
    got = O.output_error(W, X, Wq, s)
    assert abs(got - want) <= 1e-12 * want


# ----------------------------------------------------------------------------- search

def _tiny_layer(seed, N, K, M):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    m = rng.lognormal(0, 0.5, K)
    m[rng.integers(0, K)] *= 25.0                  # one outlier channel
    X = (rng.standard_normal((M, K)) * m).astype(np.float16)
    return W, X


@pytest.mark.parametrize("N,K,M", [(8, 128, 4), (32, 256, 16), (8, 256, 16), (32, 128, 4)])
def test_search_matches_brute_force(N, K, M):
    W, X = _tiny_layer(N * K + M, N, K, M)
    s_x = O.act_stats(X)
    alphas = O.alpha_grid(20)
    losses, best, best_s = O.search_scale(W, X, s_x, alphas, 4, 128)
    # brute force: re-derive every candidate and compare the explicit outputs Y_q and Y_ref
    x = X.astype(np.float64)
    yref = x @ W.astype(np.float64).T
    brute = []
    for a in alphas:
        s = np.float32(1.0) * np.array(
            [_f32(max(float(v), _f32(1e-4)) ** float(a)) for v in s_x], np.float32)
        codes, sc, z = O.quantize(W, s, 4, 128)
        deq = O.dequantize(codes, sc, z, 128)
        yq = (x / s.astype(np.float64)) @ deq.T
        brute.append(math.fsum(((yq - yref) ** 2).ravel()))
    brute = np.array(brute)
    np.testing.assert_allclose(losses, brute, rtol=1e-9)
    assert best == int(np.argmin(brute))
    assert losses[best] <= losses[0]               # never worse than plain rounding
    np.testing.assert_array_equal(best_s, O.scale_candidates(s_x, alphas)[best])


def test_search_helps_on_outlier_channels():
    # The premise of the method: scaling the channels with large activations beats plain
    # round-to-nearest (builderai.tools "AWQ", "About"; robotsatlas "AWQ", "Benchmark notes").
    W, X, _ = synth.single_layer()
    s_x = O.act_stats(X)
    losses, best, _ = O.search_scale(W, X, s_x, O.alpha_grid(20), 4, 128)
    assert best > 0
    assert losses[best] < 0.9 * losses[0]


def test_search_ties_go_to_smallest_alpha():
    rng = np.random.default_rng(9)
    W = (rng.standard_normal((4, 128)) * 0.02).astype(np.float16)
    X = np.ones((3, 128), np.float16)              # s_x == 1 -> every candidate is s == 1
    losses, best, best_s = O.search_scale(W, X, O.act_stats(X), O.alpha_grid(20), 4, 128)
    assert np.all(losses == losses[0]) and best == 0 and np.all(best_s == 1.0)


def test_joint_search_is_sum_of_parts():
    rng = np.random.default_rng(21)
    parts = [(rng.standard_normal((n, 256)) * 0.02).astype(np.float16) for n in (8, 8, 16)]
    X = (rng.standard_normal((12, 256)) * rng.lognormal(0, 0.7, 256)).astype(np.float16)
    s_x = O.act_stats(X)
    a = O.alpha_grid(20)
    joint = O.search_losses(np.concatenate(parts, axis=0), X, s_x, a, 4, 128)
    summed = sum(O.search_losses(p, X, s_x, a, 4, 128) for p in parts)
    np.testing.assert_allclose(joint, summed, rtol=1e-12)


def test_search_s_table_overrides_powers():
    W, X = _tiny_layer(1, 8, 256, 8)
    rng = np.random.default_rng(8)
    table = rng.lognormal(0, 0.3, (5, 256)).astype(np.float32)
    a = O.alpha_grid(5)
    losses = O.search_losses(W, X, O.act_stats(X), a, 4, 128, s_table=table)
    for i in range(5):
        c, sc, z = O.quantize(W, table[i], 4, 128)
        want = O.output_error(W, X, O.dequantize(c, sc, z, 128), table[i])
        assert losses[i] == want


def test_per_row_losses_sum_to_total():
    W, X = _tiny_layer(2, 16, 256, 8)
    a = O.alpha_grid(4)
    s_x = O.act_stats(X)
    rows = O.search_losses(W, X, s_x, a, 4, 128, per_row=True)
    tot = O.search_losses(W, X, s_x, a, 4, 128)
    assert rows.shape == (4, 16)
    np.testing.assert_allclose(rows.sum(axis=1), tot, rtol=1e-12)


# ----------------------------------------------------------------------------- GEMM

@pytest.mark.parametrize("bits", [4, 3])
def test_gemm_reduces_to_plain_matmul(bits):
    # Weights built from codes dequantize exactly, so the GEMM is a plain matmul.
    rng = np.random.default_rng(30 + bits)
    N, K, M = 48, 384, 7
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    qw, sc, z = O.quantize_pack(W, None, bits, 128)
    deq = O.dequantize(O.unpack(qw, bits, K), sc, z, 128)
    X = rng.standard_normal((M, K)).astype(np.float16)
    Y = O.gemm_w4a16(X, qw, sc, z, N, K, bits, 128)
    ref = torch.matmul(torch.from_numpy(X.astype(np.float64)),
                       torch.from_numpy(deq).T).numpy()
    np.testing.assert_allclose(Y, ref, rtol=1e-12, atol=1e-12)
    inv_s = rng.lognormal(0, 0.5, K).astype(np.float32)
    Y2 = O.gemm_w4a16(X, qw, sc, z, N, K, bits, 128, inv_s=inv_s)
    ref2 = torch.matmul(torch.from_numpy(X.astype(np.float64) * inv_s.astype(np.float64)),
                        torch.from_numpy(deq).T).numpy()
    np.testing.assert_allclose(Y2, ref2, rtol=1e-12, atol=1e-12)


def test_gemm_brute_force_tiny():
    rng = np.random.default_rng(40)
    N, K, M = 3, 128, 2
    W = (rng.standard_normal((N, K)) * 0.05).astype(np.float16)
    qw, sc, z = O.quantize_pack(W, None, 4, 128)
    codes = O.unpack(qw, 4, K)
    X = rng.standard_normal((M, K)).astype(np.float16)
    Y = O.gemm_w4a16(X, qw, sc, z, N, K, 4, 128)
    for m in range(M):
        for n in range(N):
            want = math.fsum(float(X[m, k]) * (int(codes[n, k]) - int(z[0, n])) * float(sc[0, n])
                             for k in range(K))
            assert abs(Y[m, n] - want) <= 1e-13 * max(1.0, abs(want))


# ----------------------------------------------------------------------------- silu_mul

def _select(rows, k):
    """fp16 weight whose row i picks input channel rows[i] (a one-hot row), [len(rows), k]."""
    W = np.zeros((len(rows), k), np.float16)
    for i, c in enumerate(rows):
        W[i, c] = 1.0
    return W


def test_silu_mul_closed_forms():
    # One token whose channels hold g-values with closed-form SiLU: silu(0) = 0,
    # silu(1) = e / (e + 1), silu(-1) = 1 / (e + 1) * -1, silu(ln 3) = (3/4) ln 3 (the logistic
    # of ln 3 is 3/4), silu(-ln 3) = -(1/4) ln 3. W_gate selects channel i into output i; W_up
    # selects the channel holding 1 (u = 1) or the channel holding 2 (u = 2).
    ln3 = math.log(3.0)
    e = math.e
    gvals = [0.0, 1.0, -1.0, float(np.float16(ln3)), float(np.float16(-ln3))]
    x = np.array([gvals + [1.0, 2.0]], np.float16)
    K = x.shape[1]
    Wg = _select(range(5), K)
    h1 = O.silu_mul(x, Wg, _select([5] * 5, K))[0]
    h2 = O.silu_mul(x, Wg, _select([6] * 5, K))[0]
    l3 = gvals[3]
    want = [0.0, e / (e + 1.0), -1.0 / (e + 1.0), l3 * 0.75, gvals[4] * 0.25]
    # fp16(ln 3) is not ln 3: its logistic is 3/4 only to within |fp16(ln3) - ln3| / 4
    tol = [1e-15, 1e-15, 1e-15, abs(l3 - ln3), abs(l3 - ln3)]
    for got, w, t in zip(h1, want, tol):
        assert abs(got - w) <= t + 1e-15
    np.testing.assert_allclose(h2, 2.0 * h1, rtol=1e-15, atol=0)


def test_silu_mul_odd_part_and_large_gates():
    # silu(g) - silu(-g) = g for every g (the logistic satisfies s(g) + s(-g) = 1), and
    # silu(g) -> g for large g, -> 0 for very negative g; u scales h linearly
    rng = np.random.default_rng(7)
    K = 64
    x = (rng.standard_normal((16, K), dtype=np.float32) * 3).astype(np.float16)
    Wg = (rng.standard_normal((24, K), dtype=np.float32) * 0.1).astype(np.float16)
    zero_part = np.zeros((24, K), np.float16)
    x1 = np.concatenate([x, np.ones((16, 1), np.float16)], axis=1)
    Wg1 = np.concatenate([Wg, np.zeros((24, 1), np.float16)], axis=1)
    Wu1 = np.concatenate([zero_part, np.ones((24, 1), np.float16)], axis=1)   # u = 1
    hp = O.silu_mul(x1, Wg1, Wu1)
    hn = O.silu_mul(x1, -Wg1, Wu1)
    g = x1.astype(np.float64) @ Wg1.astype(np.float64).T
    np.testing.assert_allclose(hp - hn, g, rtol=1e-12, atol=1e-12)
    big = np.array([[60.0, 1.0]], np.float16)
    Wbig = np.array([[1.0, 0.0], [-1.0, 0.0]], np.float16)
    Wone = np.array([[0.0, 1.0], [0.0, 1.0]], np.float16)
    hb = O.silu_mul(big, Wbig, Wone)[0]
    assert abs(hb[0] - 60.0) < 1e-20 * 60 + 60 * math.exp(-60) * 1.01
    assert 0.0 >= hb[1] > -60.0 * math.exp(-60) * 1.01
    np.testing.assert_array_equal(O.silu_mul(x1, Wg1, np.zeros_like(Wu1)), 0.0)


def test_silu_mul_brute_force_tiny():
    rng = np.random.default_rng(8)
    M, I, K = 3, 4, 40
    x = rng.standard_normal((M, K), dtype=np.float32).astype(np.float16)
    Wg = (rng.standard_normal((I, K), dtype=np.float32) * 0.3).astype(np.float16)
    Wu = (rng.standard_normal((I, K), dtype=np.float32) * 0.3).astype(np.float16)
    got = O.silu_mul(x, Wg, Wu)
    for m in range(M):
        for i in range(I):
            g = math.fsum(float(x[m, k]) * float(Wg[i, k]) for k in range(K))
            u = math.fsum(float(x[m, k]) * float(Wu[i, k]) for k in range(K))
            want = g * u / (1.0 + math.exp(-g))
            assert abs(got[m, i] - want) <= 1e-12 * (abs(want) + 1e-12)

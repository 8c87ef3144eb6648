"""Out-of-bounds writes, caught without a memory checker.

Every output and every workspace of every entry point is placed inside a larger device
buffer whose surrounding bytes hold a sentinel pattern; after the call, no byte outside the
region the call may write can have changed. The shapes are small and ragged so that the
code paths that write near buffer ends all run: N not a multiple of 16 (register decode
kernel, scales and zeros read by the builders), N not a multiple of 128 (search padding
rows, partial output tiles), M * N not a multiple of 4 (split-K reduction), few output
tiles (split-K partial sums in the workspace), 3-bit codes, and inv_s. Each call's result is
also checked against the oracle, so a guard that passes because nothing was written fails.

The same cases run against the debug build of the library (compiled with AWQ_DEBUG_BOUNDS,
where the kernels check their indices against the shapes and record a violation in the
device status word instead of making the access): awq_check_error must report no violation.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
from test_gpu_parity import GEMM_RTOL, assert_losses_match, rand_layer, rel_fro

pytestmark = pytest.mark.gpu

GUARD = 4096                 # sentinel bytes on each side (a multiple of 16)
SENTINEL = 0xA5
P, I64 = ctypes.c_void_p, ctypes.c_int64


def _load(debug):
    from weight_only_int4_stats_b200 import build
    path = build.build(debug=debug)
    import weight_only_int4_stats_b200 as awq
    return awq.load_library(path)


@pytest.fixture(scope="module", params=[False, True], ids=["release", "debug_bounds"])
def L(request):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return _load(request.param)


class Guarded:
    """`nbytes` of device memory (16-byte aligned) with GUARD sentinel bytes on each side."""

    def __init__(self, nbytes, fill=None):
        self.n = int(nbytes)
        self.buf = torch.full((GUARD + ((self.n + 15) // 16) * 16 + GUARD,), SENTINEL,
                              dtype=torch.uint8, device="cuda")
        if fill is not None:
            raw = np.ascontiguousarray(fill).view(np.uint8).reshape(-1)
            assert raw.size == self.n
            self.inner()[:] = torch.from_numpy(raw).cuda()

    def inner(self):
        return self.buf[GUARD:GUARD + self.n]

    @property
    def ptr(self):
        return P(self.buf.data_ptr() + GUARD)

    def host(self, dtype):
        return self.inner().cpu().numpy().view(dtype)

    def assert_intact(self, what):
        b = self.buf.cpu().numpy()
        bad_lo = np.nonzero(b[:GUARD] != SENTINEL)[0]
        bad_hi = np.nonzero(b[GUARD + self.n:] != SENTINEL)[0]
        assert bad_lo.size == 0, f"{what}: {bad_lo.size} bytes before the buffer changed"
        assert bad_hi.size == 0, f"{what}: {bad_hi.size} bytes after the buffer changed " \
                                 f"(first at +{bad_hi[0]})"


def _stream():
    return P(torch.cuda.current_stream().cuda_stream)


def _ok(L, rc):
    assert rc == 0, L.awq_status_string(rc)


def _no_violation(L):
    rc = L.awq_check_error(_stream())
    assert rc == 0, L.awq_status_string(rc)


@pytest.mark.parametrize("M,K", [(37, 264), (1, 8), (130, 1024)])
def test_act_stats_guarded(L, M, K):
    _, X, _ = rand_layer(M * K, 1, K, M)
    x = Guarded(X.nbytes, X)
    out = Guarded(4 * K)
    ws = Guarded(L.awq_act_stats_workspace_size(M, K))
    _ok(L, L.awq_act_stats(x.ptr, M, K, out.ptr, ws.ptr, ws.n, _stream()))
    out2 = Guarded(4 * K)
    _ok(L, L.awq_act_stats_noalloc(x.ptr, M, K, out2.ptr, _stream()))
    _no_violation(L)
    for g, what in ((out, "s_x"), (ws, "workspace"), (out2, "s_x (no-alloc)"), (x, "X")):
        g.assert_intact(what)
    np.testing.assert_array_equal(out.host(np.float32), O.act_stats(X))
    np.testing.assert_array_equal(out2.host(np.float32), O.act_stats(X))


@pytest.mark.parametrize("bits", [4, 3])
@pytest.mark.parametrize("N,K", [(37, 384), (1, 128), (130, 256)])
def test_quantize_pack_guarded(L, bits, N, K):
    W, _, m = rand_layer(N + K, N, K, 1)
    s = np.sqrt(m).astype(np.float32)
    w, sd = Guarded(W.nbytes, W), Guarded(s.nbytes, s)
    wpr = O.packed_words_per_row(K, bits)
    G = K // 128
    qw, sc, z = Guarded(4 * N * wpr), Guarded(2 * G * N), Guarded(G * N)
    _ok(L, L.awq_quantize_pack(w.ptr, N, K, sd.ptr, bits, 128, qw.ptr, sc.ptr, z.ptr,
                               _stream()))
    _no_violation(L)
    for g, what in ((qw, "qweight"), (sc, "scales"), (z, "zeros")):
        g.assert_intact(what)
    oq, osc, oz = O.quantize_pack(W, s, bits, 128)
    np.testing.assert_array_equal(qw.host(np.uint32).reshape(N, wpr), oq)
    np.testing.assert_array_equal(sc.host(np.uint16).reshape(G, N), osc.view(np.uint16))
    np.testing.assert_array_equal(z.host(np.uint8).reshape(G, N), oz)


@pytest.mark.parametrize("N,K,M", [(37, 256, 40), (130, 128, 300), (8, 384, 5)])
def test_search_guarded(L, N, K, M):
    W, X, _ = rand_layer(N * K + M, N, K, M)
    a = O.alpha_grid(20)
    sx = O.act_stats(X)
    w, x = Guarded(W.nbytes, W), Guarded(X.nbytes, X)
    sxd, ad = Guarded(sx.nbytes, sx), Guarded(a.nbytes, a)
    A = len(a)
    losses, best = Guarded(8 * A), Guarded(4)
    best_s, best_inv, rows = Guarded(4 * K), Guarded(4 * K), Guarded(8 * A * N)
    ws = Guarded(L.awq_search_scale_workspace_size(M, N, K, A))
    _ok(L, L.awq_search_scale(w.ptr, N, K, x.ptr, M, sxd.ptr, ad.ptr, A, 4, 128, None,
                              losses.ptr, best.ptr, best_s.ptr, best_inv.ptr, rows.ptr, ws.ptr,
                              ws.n, _stream()))
    _no_violation(L)
    for g, what in ((losses, "losses"), (best, "best_idx"), (best_s, "best_s"),
                    (best_inv, "best_inv_s"), (rows, "row_losses"), (ws, "workspace")):
        g.assert_intact(what)
    ol = O.search_losses(W, X, sx, a, 4, 128)
    assert_losses_match(losses.host(np.float64), ol, K, M=M)
    np.testing.assert_allclose(rows.host(np.float64).reshape(A, N).sum(axis=1),
                               losses.host(np.float64), rtol=1e-12)
    b = int(best.host(np.int32)[0])
    assert b == int(np.argmin(losses.host(np.float64)))
    S = O.scale_candidates(sx, a)
    np.testing.assert_allclose(best_s.host(np.float32), S[b], rtol=2 ** -23)
    np.testing.assert_array_equal(best_inv.host(np.float32),
                                  np.float32(1.0) / best_s.host(np.float32))


# (M, N, K, bits, inv_s): decode (streaming and register kernels), tensor-core with split-K and
# a ragged M * N, 3-bit, and a multi-tile prefill-like call
GEMM_CASES = [(1, 48, 256, 4, False), (5, 40, 384, 4, True), (16, 96, 512, 4, True),
              (33, 130, 1024, 4, True), (17, 258, 2048, 3, False), (300, 200, 384, 4, True),
              (3, 64, 768, 3, False)]


@pytest.mark.parametrize("M,N,K,bits,with_inv", GEMM_CASES)
def test_gemm_guarded(L, M, N, K, bits, with_inv):
    W, X, m = rand_layer(M + N + K + bits, N, K, M)
    s = np.sqrt(m).astype(np.float32)
    oq, osc, oz = O.quantize_pack(W, s, bits, 128)
    inv = (np.float32(1.0) / s).astype(np.float32) if with_inv else None
    x, q = Guarded(X.nbytes, X), Guarded(oq.nbytes, oq)
    sc, z = Guarded(osc.nbytes, osc), Guarded(oz.nbytes, oz)
    invd = Guarded(inv.nbytes, inv) if with_inv else None
    y = Guarded(2 * M * N)
    need = L.awq_gemm_workspace_size(M, N, K, bits)
    ws = Guarded(need) if need > 0 else None
    for flags in (0, 1):
        _ok(L, L.awq_gemm_w4a16(x.ptr, M, q.ptr, sc.ptr, z.ptr, N, K, bits, 128,
                                invd.ptr if invd else None, flags, y.ptr,
                                ws.ptr if ws else None, ws.n if ws else 0, _stream()))
        _no_violation(L)
        y.assert_intact("Y")
        if ws is not None:
            ws.assert_intact("workspace")
        want = O.gemm_w4a16(X, oq, osc, oz, N, K, bits, 128, inv_s=inv)
        got = y.host(np.float16).reshape(M, N).astype(np.float64)
        assert rel_fro(got, want) <= GEMM_RTOL


def test_debug_bounds_check_reports_a_violation():
    # The debug build's self-test computes an index one past a 4-element buffer; the bounds
    # check records the violation and skips the store (nothing outside the buffer is
    # touched), and awq_check_error reports AWQ_ERR_BOUNDS once, then clears it.
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = _load(True)
    buf = Guarded(16)
    assert L.awq_check_error(_stream()) == 0
    _ok(L, L.awq_selftest_bounds(buf.ptr, _stream()))
    assert L.awq_check_error(_stream()) == 6          # AWQ_ERR_BOUNDS
    assert L.awq_check_error(_stream()) == 0
    buf.assert_intact("self-test buffer")
    np.testing.assert_array_equal(buf.host(np.int32), np.arange(4, dtype=np.int32))
    # the release build has no bounds checks: its self-test reports that
    R = _load(False)
    assert R.awq_selftest_bounds(buf.ptr, _stream()) == 2   # AWQ_ERR_UNSUPPORTED

"""awq_act_stats_noalloc: the activation statistics for callers that cannot allocate.

Some callers of this library cannot hand it a workspace -- for example a plugin inside
another framework's engine that only receives its input and output pointers, or a
latency-critical path that must not call cudaMalloc. awq_act_stats_noalloc serves them by
keeping its partial sums in a fixed array of device memory owned by the library. This file
is collected last so that a failing run that stops at the first failure has already run
every other test; it passes both on its own and after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from weight_only_int4_stats_b200 import build
    build.build()
    import weight_only_int4_stats_b200 as awq
    return awq.lib()


def _workspace_version(L, X, K, stream):
    M = X.shape[0]
    out = torch.empty(K, dtype=torch.float32, device="cuda")
    ws_bytes = L.awq_act_stats_workspace_size(M, K)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    rc = L.awq_act_stats(ctypes.c_void_p(X.data_ptr()), M, K, ctypes.c_void_p(out.data_ptr()),
                         ctypes.c_void_p(ws.data_ptr()), ws.numel(), stream)
    assert rc == 0, L.awq_status_string(rc)
    return out


def _noalloc_version(L, X, K, stream):
    out = torch.empty(K, dtype=torch.float32, device="cuda")
    rc = L.awq_act_stats_noalloc(ctypes.c_void_p(X.data_ptr()), X.shape[0], K,
                                 ctypes.c_void_p(out.data_ptr()), stream)
    assert rc == 0, L.awq_status_string(rc)
    return out


def _activations(M, K, seed):
    rng = np.random.default_rng(seed)
    mag = rng.lognormal(0.0, 0.7, K).astype(np.float32)
    return torch.from_numpy((rng.standard_normal((M, K), dtype=np.float32) * mag)
                            .astype(np.float16)).cuda()


# On a 148-SM B200 the array (2^17 doubles) caps the row split at 2^17 / K slices: the
# 4097 x 4096 and 65536 x 4096 calls want 65 and 74 slices and get 32, the 2048 x 65536
# call wants 5 and gets 2; the 256 x 512 call (4 slices) is below its cap of 256.
@pytest.mark.parametrize("M,K", [(256, 512), (4097, 4096), (65536, 4096), (2048, 65536)])
def test_noalloc_matches_workspace_entry_point_twice(lib, M, K):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    X = _activations(M, K, M + K)
    want = _workspace_version(lib, X, K, stream).cpu().numpy()
    # two calls in a row: the second runs on the array the first one left behind
    first = _noalloc_version(lib, X, K, stream).cpu().numpy()
    second = _noalloc_version(lib, X, K, stream).cpu().numpy()
    np.testing.assert_array_equal(first, want)
    np.testing.assert_array_equal(second, want)


def test_noalloc_small_call_after_large_call_on_other_data(lib):
    # A large call fills most of the array with its partial sums; a smaller call on different
    # data (fewer slices, smaller K) must not pick any of them up.
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    big = _activations(65536, 4096, 11)
    small = _activations(300, 1024, 12)
    want_big = _workspace_version(lib, big, 4096, stream).cpu().numpy()
    want_small = _workspace_version(lib, small, 1024, stream).cpu().numpy()
    got_big = _noalloc_version(lib, big, 4096, stream).cpu().numpy()
    got_small = _noalloc_version(lib, small, 1024, stream).cpu().numpy()
    np.testing.assert_array_equal(got_big, want_big)
    np.testing.assert_array_equal(got_small, want_small)


def test_noalloc_rejects_k_beyond_its_array(lib):
    X = torch.zeros(2, 65536 + 8, dtype=torch.float16, device="cuda")
    out = torch.empty(65536 + 8, dtype=torch.float32, device="cuda")
    rc = lib.awq_act_stats_noalloc(ctypes.c_void_p(X.data_ptr()), 2, 65536 + 8,
                                   ctypes.c_void_p(out.data_ptr()), None)
    assert rc == 1   # AWQ_ERR_INVALID_ARG, nothing launched

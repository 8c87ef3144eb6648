"""The trace build (libawq_b200_trace.so): the streaming decode kernel computes the same result
as the release build (checked against the oracle) and leaves one timeline record per CTA whose
stamps are in causal order."""
import numpy as np
import pytest
import torch

import oracle as O
from test_gpu_parity import GEMM_RTOL, cu, rand_layer, rel_fro

pytestmark = pytest.mark.gpu


@pytest.fixture()
def traced():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from weight_only_int4_stats_b200 import build
    import weight_only_int4_stats_b200 as awq
    build.build()
    awq.use_library(build.build(trace=True))
    yield awq
    awq.use_library(build.LIB)   # later tests go through the release build again


@pytest.mark.parametrize("N,K", [(4096, 4096), (1040, 11008)])
def test_trace_records_one_ordered_record_per_cta(traced, N, K):
    awq = traced
    W, X, m = rand_layer(N + K, N, K, 1, outliers=False)
    qw, sc, z = O.quantize_pack(W, np.sqrt(m).astype(np.float32), 4, 128)
    Xd, q, s_, zd = cu(X), cu(qw), cu(sc), cu(z)
    awq.awq_gemm_w4a16(Xd, q, s_, zd, N, K, 4)            # first call: module load
    torch.cuda.synchronize()
    awq.trace_reset()
    Y = awq.awq_gemm_w4a16(Xd, q, s_, zd, N, K, 4)
    torch.cuda.synchronize()
    want = O.gemm_w4a16(X, qw, sc, z, N, K, 4, 128)
    assert rel_fro(Y.float().cpu().numpy(), want) <= GEMM_RTOL
    R = awq.trace_read().astype(np.int64)
    tiles, chunks = N // 16, -(-K // 2048)
    grid = len(R)
    assert 1 <= grid <= tiles
    assert sorted(R[:, 6].tolist()) == list(range(grid))   # every CTA once
    assert (R[:, 0] == N).all()
    assert R[:, 1].sum() == tiles * chunks                 # units cover every (tile, chunk)
    start, waited, staged, end = R[:, 2], R[:, 3], R[:, 4], R[:, 5]
    assert (start <= waited).all() and (waited <= staged).all() and (staged <= end).all()
    for rec in R:
        k = int(min(rec[1], 24))
        landed = rec[8:8 + k]
        assert (np.diff(landed) >= 0).all() and landed[0] >= rec[2] and landed[-1] <= rec[5]

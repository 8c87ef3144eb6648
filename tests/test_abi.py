"""The C-ABI library builds, loads without a GPU, exports every entry point that include/*.h
declares, and rejects bad arguments on the host before any launch."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _lib():
    from weight_only_int4_stats_b200 import build
    build.build()
    import weight_only_int4_stats_b200 as awq
    return awq.lib()


def _declared():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names += re.findall(r"^AWQ_API\s+[\w\s\*]+?\b(awq_\w+)\s*\(", text, flags=re.M)
    return names


def test_header_declares_the_boundary():
    names = set(_declared())
    for want in ("awq_act_stats", "awq_search_scale", "awq_quantize_pack", "awq_gemm_w4a16",
                 "awq_act_stats_workspace_size", "awq_search_scale_workspace_size",
                 "awq_gemm_workspace_size", "awq_check_error", "awq_status_string",
                 "awq_abi_version"):
        assert want in names


def test_library_exports_every_declared_symbol():
    L = _lib()
    for name in _declared():
        assert hasattr(L, name), name


def test_status_strings_and_version():
    L = _lib()
    for code, name in enumerate(["AWQ_OK", "AWQ_ERR_INVALID_ARG", "AWQ_ERR_UNSUPPORTED",
                                 "AWQ_ERR_WORKSPACE", "AWQ_ERR_CUDA", "AWQ_ERR_TIMEOUT",
                                 "AWQ_ERR_BOUNDS"]):
        assert L.awq_status_string(code).decode() == name
    assert L.awq_abi_version() == 2


def test_host_validation_rejects_before_launch():
    L = _lib()
    P = ctypes.c_void_p
    fake = P(1 << 20)          # never dereferenced: every call below fails validation first
    odd = P((1 << 20) + 2)     # misaligned
    # act_stats: null X, M = 0, K not a multiple of 8
    assert L.awq_act_stats(None, 4, 8, fake, fake, 1 << 20, None) == 1
    assert L.awq_act_stats(fake, 0, 8, fake, fake, 1 << 20, None) == 1
    assert L.awq_act_stats(fake, 4, 12, fake, fake, 1 << 20, None) == 1
    assert L.awq_act_stats(odd, 4, 8, fake, fake, 1 << 20, None) == 1
    # quantize_pack: bad bits, bad group, K not a multiple of 128; N = 0 is a no-op
    assert L.awq_quantize_pack(fake, 4, 128, None, 5, 128, fake, fake, fake, None) == 1
    assert L.awq_quantize_pack(fake, 4, 128, None, 4, 64, fake, fake, fake, None) == 1
    assert L.awq_quantize_pack(fake, 4, 200, None, 4, 128, fake, fake, fake, None) == 1
    assert L.awq_quantize_pack(fake, 0, 128, None, 4, 128, fake, fake, fake, None) == 0
    # gemm: M = 0 and N = 0 are no-ops; misaligned Y; bits 2
    assert L.awq_gemm_w4a16(fake, 0, fake, fake, fake, 8, 128, 4, 128, None, 0, fake, None, 0,
                            None) == 0
    assert L.awq_gemm_w4a16(fake, 1, fake, fake, fake, 0, 128, 4, 128, None, 0, fake, None, 0,
                            None) == 0
    assert L.awq_gemm_w4a16(fake, 1, fake, fake, fake, 8, 128, 4, 128, None, 0, odd, None, 0,
                            None) == 1
    assert L.awq_gemm_w4a16(fake, 1, fake, fake, fake, 8, 128, 2, 128, None, 0, fake, None, 0,
                            None) == 1
    # unknown flag bits
    assert L.awq_gemm_w4a16(fake, 1, fake, fake, fake, 8, 128, 4, 128, None, 6, fake, None, 0,
                            None) == 1
    # search: n_alpha out of range, too-small workspace
    assert L.awq_search_scale(fake, 8, 128, fake, 4, fake, fake, 0, 4, 128, None, fake, fake,
                              fake, None, None, fake, 1 << 30, None) == 1
    assert L.awq_search_scale(fake, 8, 128, fake, 4, fake, fake, 20, 4, 128, None, fake, fake,
                              fake, None, None, fake, 16, None) == 3
    assert L.awq_search_scale(fake, 8, 128, fake, 4, fake, fake, 20, 4, 128, None, fake, fake,
                              fake, odd, None, fake, 1 << 30, None) == 1


def test_workspace_queries():
    L = _lib()
    assert L.awq_search_scale_workspace_size(256, 512, 512, 20) >= 20 * 512 * 512 * 2
    assert L.awq_gemm_workspace_size(1, 4096, 4096, 4) == 0
    # enough output tiles for every SM: no split-K, no workspace (inv_s needs none)
    assert L.awq_gemm_workspace_size(2048, 4096, 4096, 4) == 0
    assert L.awq_act_stats_workspace_size(0, 16) == 0


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import weight_only_int4_stats_b200 as awq
    monkeypatch.setattr(awq, "library_path", str(tmp_path / "missing.so"))
    monkeypatch.setattr(awq, "_lib", None)
    with pytest.raises(ImportError):
        awq.lib()


def test_gemm_workspace_follows_the_chosen_kernel():
    # the decode kernels need no workspace; an 8 < M <= 16 call whose X does not fit the
    # streaming kernel's shared memory takes the tensor-core path, which with so few output
    # tiles splits K and needs room for fp32 partial sums (at least two slices of M x N)
    L = _lib()
    assert L.awq_gemm_workspace_size(1, 4096, 11008, 4) == 0
    assert L.awq_gemm_workspace_size(8, 4096, 11008, 4) == 0
    assert L.awq_gemm_workspace_size(16, 4096, 4096, 4) == 0
    for M, N, K in [(16, 4096, 11008), (16, 4104, 4096), (64, 4096, 4096)]:  # 4104: N % 16
        ws = L.awq_gemm_workspace_size(M, N, K, 4)
        assert ws >= 2 * M * N * 4 and ws % 256 == 0, (M, N, K, ws)


@pytest.mark.parametrize("N,K,M,slices", [
    (14336, 4096, 32, 1), (14336, 4096, 64, 1), (14336, 4096, 128, 1), (14336, 4096, 256, 1),
    (4096, 14336, 32, 4), (4096, 14336, 64, 4), (4096, 14336, 128, 4), (4096, 14336, 256, 4),
    (6144, 4096, 32, 3), (6144, 4096, 64, 3), (6144, 4096, 128, 3), (6144, 4096, 256, 2),
])
def test_split_k_choice_on_the_batched_shapes(N, K, M, slices):
    # the split-K chooser on 148 SMs (the count the library assumes without a device, and a
    # B200's): a larger split has to win by 12 % per extra slice. On B200 this beat 2, 6, 40
    # and 60 %: [14336, 4096] at M = 32 / 64 runs unsplit (26.6 -> 24.3, 29.4 -> 26.2 us
    # against 5 slices), [4096, 14336] takes 4 slices, not 9 (2 or 3 were 20-60 % slower).
    # The workspace holds one fp32 partial M x N per slice when K is split, nothing otherwise.
    ws = _lib().awq_gemm_workspace_size(M, N, K, 4)
    want = 0 if slices == 1 else -(-slices * M * N * 4 // 256) * 256
    assert ws == want, (N, K, M, ws, want)


def test_gemm_workspace_is_checked_before_launch():
    # the tensor-core path with few output tiles needs room for split-K partial sums; a
    # missing or short workspace is rejected on the host (AWQ_ERR_WORKSPACE) before anything
    # is launched
    L = _lib()
    P = ctypes.c_void_p
    fake = P(1 << 20)
    need = L.awq_gemm_workspace_size(64, 4096, 4096, 4)
    assert need >= 2 * 64 * 4096 * 4
    assert L.awq_gemm_w4a16(fake, 64, fake, fake, fake, 4096, 4096, 4, 128, fake, 0, fake,
                            None, 0, None) == 3
    assert L.awq_gemm_w4a16(fake, 64, fake, fake, fake, 4096, 4096, 4, 128, fake, 0, fake,
                            fake, need - 16, None) == 3


def test_debug_build_exports_the_same_symbols():
    # the bounds-checking build is the same library with index checks compiled in
    from weight_only_int4_stats_b200 import build
    import weight_only_int4_stats_b200 as awq
    D = awq.load_library(build.build(debug=True))
    for name in _declared():
        assert hasattr(D, name), name
    assert D.awq_abi_version() == 2
    # the release build refuses the bounds self-test without launching anything
    assert _lib().awq_selftest_bounds(ctypes.c_void_p(1 << 20), None) == 2


def test_trace_build_exports_the_same_symbols():
    # the timeline build is the same library with %globaltimer stamps in the decode kernel;
    # the release and debug builds decline the trace calls without touching the GPU
    from weight_only_int4_stats_b200 import build
    import weight_only_int4_stats_b200 as awq
    T = awq.load_library(build.build(trace=True))
    for name in _declared():
        assert hasattr(T, name), name
    assert T.awq_abi_version() == 2
    n = ctypes.c_int64(0)
    out = (ctypes.c_ulonglong * 32)()
    assert _lib().awq_trace_reset() == 2
    assert _lib().awq_trace_read(out, 1, ctypes.byref(n)) == 2
    D = awq.load_library(build.build(debug=True))
    assert D.awq_trace_reset() == 2

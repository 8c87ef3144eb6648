"""Host logic of bench.py that the reported numbers rest on: the executed tensor flops of a
search call in each form, the lookup of a kernel's profiled DRAM traffic (and its refusal
once the kernel's sources change), and the splitting of the trace build's records into
launches."""
import hashlib
import importlib.util
import os

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_search_flops_direct_form(bench):
    # M < 2K: both fp16 parts of the error operand against X, rows padded to 128
    ex, form = bench.search_executed_flops(1000, 130, 4096, 20)
    assert form == "direct"
    assert ex == 2 * 20 * 2 * 1000 * 256 * 4096


def test_search_flops_gram_form_counts_the_upper_tiles(bench):
    # M >= 2K: G from its 128 x 256 tiles that reach the diagonal, then three MMAs per k step
    # of the two-part operand against G. Tile (r, c) covers rows [128 r, 128 r + 128) and
    # columns [256 c, 256 c + 256); it is skipped when every row lies below every column.
    M, N, K, A = 65536, 22016, 4096, 20
    ex, form = bench.search_executed_flops(M, N, K, A)
    assert form == "gram"
    kept = 0
    for r in range(K // 128):
        for c in range(K // 256):
            rows = range(128 * r, 128 * r + 128)
            cols = range(256 * c, 256 * c + 256)
            if min(rows) <= max(cols):       # some element on or above the diagonal
                kept += 1
    assert kept == 272                       # of 512 at K = 4096
    assert ex == 2 * M * 128 * 256 * kept + A * 3 * 2 * 22016 * K * K
    # K = 11008: 86 row tiles, 43 column tiles
    ex2, _ = bench.search_executed_flops(65536, 4096, 11008, 20)
    kept2 = sum(1 for r in range(86) for c in range(43) if 128 * r <= 256 * c + 255)
    assert ex2 == 2 * 65536 * 128 * 256 * kept2 + 20 * 3 * 2 * 4096 * 11008 * 11008


def test_gemm_bytes(bench):
    # packed codes + fp16 scales and uint8 zeros per group + X in + Y out
    assert bench.gemm_bytes(1, 4096, 4096) == 4096 * 4096 // 2 + 4096 * 32 * 3 + 2 * 4096 + 2 * 4096
    assert bench.gemm_bytes(16, 11008, 4096, 3) == (11008 * 4096 * 3 // 8 + 11008 * 32 * 3
                                                   + 2 * 16 * 4096 + 2 * 16 * 11008)


def _tree(tmp_path, gemv, common, line):
    csrc = tmp_path / "weight_only_int4_stats_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "gemv.cuh").write_bytes(gemv)
    (csrc / "common.cuh").write_bytes(common)
    prof = tmp_path / "profiles"
    prof.mkdir()
    if line is not None:
        (prof / "decode.md").write_text(f"# summary\n\n`{line}`\n")


def test_profiled_traffic_follows_the_source_hash(bench, tmp_path, monkeypatch):
    gemv, common = b"kernel source\n", b"helpers\n"
    h = hashlib.sha256(gemv + common).hexdigest()[:16]
    _tree(tmp_path, gemv, common, f"bench-traffic: gemv_stream_decode_M1 12345 {h}")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.source_hash("gemv_stream_decode_M1") == h
    assert bench.profiled_traffic("gemv_stream_decode_M1") == (12345.0, "profiles/decode.md")
    # the sources change after the capture: the figure is refused, with the reason
    (tmp_path / "weight_only_int4_stats_b200" / "csrc" / "gemv.cuh").write_bytes(b"changed\n")
    v, why = bench.profiled_traffic("gemv_stream_decode_M1")
    assert v is None and "changed" in why


def test_profiled_traffic_without_a_capture(bench, tmp_path, monkeypatch):
    _tree(tmp_path, b"a", b"b", None)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("gemv_stream_decode_M1") == (None, "no ncu capture")


def test_segment_launches_splits_where_a_block_repeats(bench):
    def rec(block, n):
        r = np.zeros(32, dtype=np.int64)
        r[0], r[6] = n, block
        return r
    # three launches of 3, 2 and 3 CTAs, CTAs of a launch in any start order
    records = [rec(b, 4096) for b in (2, 0, 1)] + [rec(b, 11008) for b in (1, 0)] + \
              [rec(b, 4096) for b in (0, 2, 1)]
    launches = bench.segment_launches(np.array(records))
    assert [len(l) for l in launches] == [3, 2, 3]
    assert [int(l[0][0]) for l in launches] == [4096, 11008, 4096]
    assert bench.segment_launches(np.zeros((0, 32), dtype=np.int64)) == []

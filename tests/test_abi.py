"""C-ABI checks that need no GPU: the library loads, exports every symbol that
include/ispa.h declares, rejects bad arguments on the host before any launch,
and its host bookkeeping matches the oracle bit for bit."""
import ctypes
import os
import re

import numpy as np

import pytest

from ar_video_diffusion_b200 import build as ispa_build
from ar_video_diffusion_b200 import ispa
from oracle import ispa_oracle as orc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    ispa_build.build()
    return ispa.lib()


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "ispa.h")).read()
    return sorted(set(re.findall(r"ISPA_API\s+[\w\s\*]+?\b(ispa_\w+)\s*\(", text)))


def test_header_declares_the_four_hot_path_entry_points():
    names = _declared_symbols()
    for n in ("ispa_dual_attention", "ispa_gram_accumulate", "ispa_absorb_solve", "ispa_local_attention_project"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    names = _declared_symbols()
    assert names, "no declarations found"
    for n in names:
        assert hasattr(L, n), f"{n} not exported"
    assert set(names) == set(ispa.EXPORTED)


def test_version_and_status_strings(L):
    assert ispa.ispa_version() >= 100
    assert ispa.ispa_status_string(0) == "ok"
    assert "positive definite" in ispa.ispa_status_string(4)


def test_host_validation_rejects_before_launch(L):
    # NULL q -> invalid argument, no CUDA call needed
    r = L.ispa_dual_attention(None, 10, 128, 1, 128, 0, 0.0, None, 0, None, 0, None, None, None, None, None, None,
                              None)
    assert r == 1 and "q is NULL" in L.ispa_last_error().decode()
    # unsupported head_dim
    r = L.ispa_dual_attention(ctypes.c_void_p(256), 10, 96, 1, 96, 0, 0.0, None, 0, None, 0, None, None, None, None,
                              None, None, None)
    assert r == 2
    # unsupported dtype
    r = L.ispa_gram_accumulate(None, None, 4, 128, 128, 7, None, None, 0, None)
    assert r == 2
    # workspace too small
    r = L.ispa_absorb_solve(ctypes.c_void_p(256), ctypes.c_void_p(256), ctypes.c_void_p(256), 0, 128, 0.0, 0.01,
                            ctypes.c_void_p(256), None, ctypes.c_void_p(256), 16, None, None)
    assert r == 6
    # d_model not a multiple of 64
    r = L.ispa_absorb_solve(ctypes.c_void_p(256), ctypes.c_void_p(256), ctypes.c_void_p(256), 0, 100, 0.0, 0.01,
                            ctypes.c_void_p(256), None, ctypes.c_void_p(256), 1 << 20, None, None)
    assert r == 2
    # misaligned projection input
    r = L.ispa_project(ctypes.c_void_p(258), 4, 128, 128, 128, 0, ctypes.c_void_p(256), ctypes.c_void_p(256), None)
    assert r == 1


def test_workspace_size_formula(L):
    for D in (64, 128, 1536, 5120):
        assert ispa.ispa_absorb_workspace_bytes(D) >= 4 * D * D + 4 * 64 * D + 8


@pytest.mark.parametrize("chunk", [0, 1, 2, 7, 23])
def test_chunk_token_ranges_bit_exact(L, chunk):
    for F, cf, sf in [(1560, 3, 1), (16, 4, 1), (7, 2, 2)]:
        got = ispa.ispa_chunk_token_ranges(chunk, F, cf, sf)
        assert got == orc.chunk_token_ranges(chunk, F, cf, sf)


def test_chunk_token_ranges_rejects_a_sink_that_overlaps_the_current_chunk(L):
    # chunk 1 of 3-frame chunks starts at frame 3: a 4-frame sink would overlap it
    for args in [(1, 1560, 3, 4), (2, 16, 1, 3), (1, 7, 2, 3)]:
        with pytest.raises(ispa.IspaError) as e:
            ispa.ispa_chunk_token_ranges(*args)
        assert e.value.code == 1
        with pytest.raises(ValueError):
            orc.chunk_token_ranges(*args)
        with pytest.raises(ispa.IspaError):
            ispa.ispa_kv_bytes(args[0], 4, 0b0101, True, args[1], args[2], 128, 2, args[3])
    # the boundary case (the sink fills every frame before the chunk) and chunk 0 are valid
    assert ispa.ispa_chunk_token_ranges(1, 16, 3, 3) == orc.chunk_token_ranges(1, 16, 3, 3)
    assert ispa.ispa_chunk_token_ranges(0, 16, 3, 9) == orc.chunk_token_ranges(0, 16, 3, 9)


def test_kv_bytes_bit_exact(L):
    mask = orc.layer_mask(30, range(0, 30, 2))
    for chunk in range(24):
        for trans in (False, True):
            for m in (0, mask, (1 << 30) - 1):
                assert ispa.ispa_kv_bytes(chunk, 30, m, trans, 1560, 3, 1536, 2) == \
                    orc.kv_bytes(chunk, 30, m, trans, 1560, 3, 1536, 2)
    assert ispa.ispa_kv_bytes(23, 30, mask, True, 1560, 3, 1536, 2) == 15 * 112320 * 6144 + 15 * 6240 * 6144


def test_layer_selection_host_logic_bit_exact(L):
    # the library's selection against the oracle's on random errors with ties and NaN
    rng = np.random.default_rng(91)
    for trial in range(200):
        n = int(rng.integers(0, 40))
        eps = [float(x) for x in rng.choice([0.01, 0.02, 0.05, 0.3, 1.0, 2.5], size=n)]
        for j in range(n):
            if rng.random() < 0.1:
                eps[j] = float("nan")
        k = int(rng.integers(0, n + 1))
        assert ispa.select_layers(eps, k) == orc.select_layers(eps, k), (eps, k)


def test_layer_selection_entry_points_reject_before_launch(L):
    arr = (ctypes.c_double * 4)(0.1, 0.2, 0.3, 0.4)
    sel = (ctypes.c_uint8 * 4)()
    assert L.ispa_select_layers(arr, 4, 5, sel) == 1     # k > n_layers
    assert L.ispa_select_layers(arr, -1, 0, sel) == 1
    assert L.ispa_select_layers(None, 4, 2, sel) == 1
    # layer error: NULL matrix, short workspace, unsupported dtype
    p = ctypes.c_void_p(256)
    assert L.ispa_layer_error(None, p, p, p, 0, p, 128, p, 1 << 20, p, None) == 1
    assert L.ispa_layer_error(p, p, p, p, 0, p, 128, p, 16, p, None) == 6
    assert L.ispa_layer_error(p, p, p, p, 9, p, 128, p, 1 << 20, p, None) == 2
    assert ispa.ispa_layer_error_workspace_bytes(1536) == 32 * 1536 * 1536
    # symmetric statistics: bf16 needs d_model % 128 == 0; NULL E
    assert L.ispa_sym_gram_accumulate(p, 10, 96, 96, 0, p, 0, None) == 2
    assert L.ispa_sym_gram_accumulate(p, 10, 128, 128, 0, None, 0, None) == 1


def test_segment_limit_and_empty_queries_rejected_before_launch(L):
    seg_t = ispa.KVSegment
    p = 256  # aligned fake device address: validation runs before any launch
    def segs(n, tokens=16):
        arr = (seg_t * max(n, 1))()
        for i in range(n):
            arr[i] = seg_t(p, p, tokens, 128)
        return arr
    q = ctypes.c_void_p(p)
    out = ctypes.c_void_p(p)
    # 4 local + 5 history non-empty segments: one more than ISPA_MAX_SEGMENTS
    r = L.ispa_dual_attention(q, 10, 128, 1, 128, 0, 0.0, segs(4), 4, segs(5), 5, out, out, None, None, None, None,
                              None)
    assert r == 2 and "segments" in L.ispa_last_error().decode()
    # no query rows
    r = L.ispa_dual_attention(q, 0, 128, 1, 128, 0, 0.0, segs(1), 1, segs(1), 1, out, out, None, None, None, None,
                              None)
    assert r == 1
    # dual mode with an empty local set
    r = L.ispa_dual_attention(q, 10, 128, 1, 128, 0, 0.0, segs(1, 0), 1, segs(1), 1, out, out, None, None, None, None,
                              None)
    assert r == 1 and "local" in L.ispa_last_error().decode()


def test_w8a8_entry_points_reject_before_launch(L):
    p, odd = ctypes.c_void_p(256), ctypes.c_void_p(264)
    # activations: fp32 is unsupported, k must be a multiple of 16, NULL codes, misaligned rows
    assert L.ispa_quantize_e4m3_rows(p, 4, 128, 128, 1, p, p, None) == 2
    assert L.ispa_quantize_e4m3_rows(p, 4, 120, 120, 0, p, p, None) == 2
    assert L.ispa_quantize_e4m3_rows(p, 4, 128, 128, 0, None, p, None) == 1
    assert L.ispa_quantize_e4m3_rows(p, 4, 128, 132, 0, p, p, None) == 1
    assert L.ispa_quantize_e4m3_rows(odd, 4, 128, 128, 0, p, p, None) == 1
    # weight: sizes off the multiples, NULL scales
    assert L.ispa_quantize_e4m3_weight(p, 100, 128, 0, p, p, None) == 2
    assert L.ispa_quantize_e4m3_weight(p, 128, 128, 0, p, None, None) == 1
    # projection: d_out % 128, misaligned codes, non-positive rows
    assert L.ispa_project_w8a8(p, p, 4, 128, p, p, 192, p, None) == 2
    assert L.ispa_project_w8a8(odd, p, 4, 128, p, p, 128, p, None) == 1
    assert L.ispa_project_w8a8(p, p, 0, 128, p, p, 128, p, None) == 1
    # L-layer W8A8: missing code buffers
    assert L.ispa_local_attention_project_w8a8(p, 4, 128, 1, 128, 0, 0.0, None, 0, p, p, p, p, None, p, None,
                                               None) == 1

"""The algorithmic units behind every roofline fraction the bench reports,
pinned to their closed forms at the Wan-1.3B shapes (CPU only)."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from ar_video_diffusion_b200 import synth  # noqa: E402

W13 = synth.WORKLOADS["wan1.3b"]


def test_attention_flops_of_the_wan13b_chunk():
    # QK^T and PV over 1560 sink + 4680 current + 18720 history keys, 12 heads of 128
    assert bench.attn_flops(W13) == 4 * 4680 * 24960 * 128 * 12 == 717_697_843_200


def test_statistics_flops_count_the_symmetric_half_once():
    D = 1536
    assert bench.gram_flops(W13, 4680) == 4680 * D * (D + 1) + 2 * 4680 * D * D
    assert bench.gram_flops(W13, 4680) == pytest.approx(33.1e9, rel=2e-3)


def test_solve_flops_and_launch_count():
    D = 1536
    assert bench.solve_flops(D) == pytest.approx(D ** 3 / 3 + 2 * D ** 3 + 2 * D ** 3)
    assert bench.solve_flops(D) == pytest.approx(15.7e9, rel=3e-3)
    nb = D // 64
    # tensor-core form: split of R, [0 | I] fill, S = R W, trace, shift, the
    # first diagonal step; nb panel applications, nb-1 further diagonal steps
    # (side stream) and nb-1 update products; the split of [L^-1 S | L^-1],
    # dW = (L^-1)^T (L^-1 S), W_new (an ncu launch list shows 24
    # diag_step_kernel and 24 panel_apply_kernel launches per D = 1536 solve).
    assert bench.absorb_launches(D) == 6 + nb + 2 * (nb - 1) + 3 == 79


def test_chunk_rooflines_are_the_tensor_time_of_their_contractions():
    peak = 1644.2
    r = bench.chunk_roofline_ms(W13, peak)
    proj = 2 * 4680 * 1536 * 1536
    local = 4 * 4680 * 6240 * 128 * 12
    to_ms = lambda f: f / (peak * 1e12) * 1e3
    assert r["l_layer"] == pytest.approx(to_ms(local + proj))
    assert r["f_layer"] == pytest.approx(to_ms(bench.attn_flops(W13) + proj))
    assert r["warmup_f_layer"] == pytest.approx(to_ms(bench.attn_flops(W13) + proj + bench.gram_flops(W13, 4680)))


def test_e2e_bytes_per_step():
    # host -> device: the chunk's Q and current K, V (bf16); device -> host: A_full (bf16) and LSE_full (fp32)
    n, D, H = 4680, 1536, 12
    assert 3 * n * D * 2 == 43_130_880
    assert n * D * 2 + H * n * 4 == 14_601_600

"""GPU parity of the streaming rollout (1.3B shapes, 4 layers, layers 0 and 2
absorbed, 4 warm-up chunks then 2 post-transition chunks): sampled rows of
each checked layer output against the oracle, dW of both absorbed layers
against the oracle absorb fed the exact A_loc / delta rows the GPU statistics
consumed, and the KV bookkeeping bit for bit."""
import dataclasses

import numpy as np
import pytest
import torch

from ar_video_diffusion_b200 import build as ispa_build
from ar_video_diffusion_b200 import ispa, synth
from ar_video_diffusion_b200.rollout import Rollout
from oracle import ispa_oracle as orc
from helpers import ATTN_MAX_REL, DW_REL_BF16, fro_rel, host, max_rel

pytestmark = pytest.mark.gpu

CHECK = {(0, 0), (1, 2), (2, 3), (0, 4), (1, 4), (2, 5), (3, 5)}
N_ROWS = 32


def test_rollout_layers_absorb_and_kv_bookkeeping():
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    ispa_build.build()
    w = dataclasses.replace(synth.WORKLOADS["rollout"], n_layers=4, post_chunks=2)
    absorbed = [0, 2]
    rows = np.sort(np.random.default_rng(7).choice(w.n_q, N_ROWS, replace=False))
    rows[-1] = w.n_q - 1
    stats = {l: ([], []) for l in absorbed}
    checks = []

    def on_layer(l, c, info):
        if c < w.warm_chunks and l in absorbed:
            stats[l][0].append(host(info["out"]["a_loc"]))
            stats[l][1].append(host(info["out"]["a_delta"]))
        if (l, c) in CHECK:
            torch.cuda.synchronize()
            cat = lambda segs, i: np.concatenate([host(s[i]) for s in segs]) if segs else np.zeros((0, w.d_model))
            checks.append({"l": l, "c": c, "mode": info["mode"], "q": host(info["q"])[rows],
                           "k_loc": cat(info["local"], 0), "v_loc": cat(info["local"], 1),
                           "k_hist": cat(info["hist"], 0), "v_hist": cat(info["hist"], 1),
                           "W": host(info["W"]), "y": host(info["y"])[rows]})

    ro = Rollout(w, absorbed=absorbed, on_layer=on_layer)
    reports = ro.run()

    # KV bookkeeping: bit-exact against the oracle's integer arithmetic
    mask = orc.layer_mask(w.n_layers, absorbed)
    for rep in reports:
        trans = rep.chunk >= w.warm_chunks
        assert rep.kv_bytes == orc.kv_bytes(rep.chunk, w.n_layers, mask, trans, w.frame_tokens, w.chunk_frames,
                                            w.d_model, 2)
        assert rep.kv_bytes_all_f == orc.kv_bytes(rep.chunk, w.n_layers, 0, trans, w.frame_tokens,
                                                  w.chunk_frames, w.d_model, 2)
    # L-layers really dropped their history: sink + one chunk of K/V remain
    for l in absorbed:
        assert ro.k[l].shape[0] == w.frame_tokens + w.n_q

    # absorb: dW against the oracle solve of the rows the statistics consumed
    for l in absorbed:
        A, Dl = np.concatenate(stats[l][0]), np.concatenate(stats[l][1])
        G, R = orc.gram(A, Dl)
        W = host(ro.W[l])
        dW_ref = orc.absorb(G, R, W, orc.ridge_lambda(G))
        assert fro_rel(host(ro.dW[l]), dW_ref) <= DW_REL_BF16

    # sampled layer outputs
    assert len(checks) == len(CHECK)
    for ck in checks:
        a_loc, _ = orc.attention(ck["q"], ck["k_loc"], ck["v_loc"], w.n_heads)
        if ck["mode"] == "L":
            a = a_loc
        else:
            a, _ = orc.attention(ck["q"], np.concatenate([ck["k_loc"], ck["k_hist"]]),
                                 np.concatenate([ck["v_loc"], ck["v_hist"]]), w.n_heads)
        y_ref = orc.project(a, ck["W"])
        assert max_rel(ck["y"], y_ref) <= ATTN_MAX_REL, (ck["l"], ck["c"], ck["mode"])
    modes = {(ck["l"], ck["c"]): ck["mode"] for ck in checks}
    assert modes[(0, 4)] == "L" and modes[(1, 4)] == "F" and modes[(0, 0)] == "F"

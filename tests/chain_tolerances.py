"""Oracle-only simulation behind the chained tolerances of the GPU tests.

TEST INFRASTRUCTURE: imports the oracle and the seeded input generator only.

A chained GPU test compares the end of a GPU chain (attention -> statistics
-> absorb, or attention -> W8A8 projection) with the oracle's own chain run
from the same seeded inputs.  The GPU chain consumes its own bf16 attention
outputs, which differ from the oracle's fp64 ones by the attention error
(bf16 operands: about 2^-9 relative) and by the bf16 rounding of the stored
outputs.  This module replays that perturbation inside the oracle:

  * A_loc and A_full of every warm-up row get 2^-9 relative Gaussian noise and
    are rounded to bf16 (delta = bf16(A_full~ - A_loc~), as the GPU writes it);
  * the statistics, lambda, dW and the reconstruction error are recomputed
    from the perturbed rows and compared with the unperturbed chain;
  * for the W8A8 L-layer, A_loc gets the same noise before its bf16 rounding
    and the e4m3 projection is recomputed.

The figures it prints are the basis of CHAIN_DW_REL, CHAIN_EPS_REL,
CHAIN_W8A8_FRO and CHAIN_W8A8_MAX in tests/helpers.py;
tests/test_chain_tolerances.py re-runs the small cases and checks that every
bound keeps at least a factor of two over the simulated movement.

    python tests/chain_tolerances.py          # small rollout + W8A8 L-layer
    python tests/chain_tolerances.py --full   # also one 1.3B-shaped rollout layer (minutes)
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from ar_video_diffusion_b200 import synth  # noqa: E402  (seeded generator only)
from oracle import ispa_oracle as orc  # noqa: E402
from oracle import w8a8_oracle as w8  # noqa: E402

NOISE = 2.0 ** -9


def rollout_warmup_rows(w: synth.Workload, layer: int, rows_per_chunk=None):
    """The oracle's A_loc and A_full over the warm-up chunks of one rollout
    layer (host generator, the rollout's chunk schedule: chunk 0 holds the sink
    frame in its own current chunk; chunk c >= 1 sees sink = frame 0, history =
    frames 1..3c-1, current = frames 3c..3c+2)."""
    a_loc, a_full = [], []
    cf = w.chunk_frames
    for c in range(w.warm_chunks):
        q = synth.chunk_q(w, layer, c)
        if rows_per_chunk is not None:
            q = q[:rows_per_chunk]
        if c == 0:
            sink, hist, cur = [], [], list(range(0, cf))
        else:
            sink, hist, cur = [0], list(range(w.sink_frames, cf * c)), list(range(cf * c, cf * c + cf))
        ks, vs = synth.frames_kv(w, layer, sink)
        kh, vh = synth.frames_kv(w, layer, hist)
        kc, vc = synth.frames_kv(w, layer, cur)
        kl, vl = np.concatenate([ks, kc]), np.concatenate([vs, vc])
        loc, _ = orc.attention(q, kl, vl, w.n_heads)
        full, _ = orc.attention(q, np.concatenate([kl, kh]), np.concatenate([vl, vh]), w.n_heads)
        a_loc.append(loc)
        a_full.append(full)
    return np.concatenate(a_loc), np.concatenate(a_full)


def perturb(a_loc, a_full, rng):
    """The GPU-like copies: 2^-9 relative noise, bf16 storage of A_loc and delta."""
    an = a_loc * (1 + NOISE * rng.standard_normal(a_loc.shape))
    fn = a_full * (1 + NOISE * rng.standard_normal(a_full.shape))
    ab = synth.round_bf16(an.astype(np.float32)).astype(np.float64)
    db = synth.round_bf16((fn - an).astype(np.float32)).astype(np.float64)
    return ab, ab + db


def absorb_chain_sensitivity(w: synth.Workload, layers, seed: int = 0, rows_per_chunk=None) -> list:
    """Per layer: relative Frobenius movement of dW and relative movement of
    the reconstruction error eps under the GPU-like perturbation."""
    rng = np.random.default_rng(seed)
    out = []
    for layer in layers:
        a_loc, a_full = rollout_warmup_rows(w, layer, rows_per_chunk)
        W = synth.weight(w, layer).astype(np.float64)
        G, R = orc.gram(a_loc, a_full - a_loc)
        dW = orc.absorb(G, R, W, orc.ridge_lambda(G))
        eps = orc.reconstruction_error(a_loc, a_full, W, dW)
        pl, pf = perturb(a_loc, a_full, rng)
        Gp, Rp = orc.gram(pl, pf - pl)
        dWp = orc.absorb(Gp, Rp, W, orc.ridge_lambda(Gp))
        epsp = orc.reconstruction_error(pl, pf, W, dWp)
        out.append({"layer": layer, "rows": len(a_loc),
                    "dw_rel": float(np.linalg.norm(dWp - dW) / np.linalg.norm(dW)),
                    "eps": eps, "eps_rel": abs(epsp - eps) / eps})
    return out


def w8a8_chain_sensitivity(draws: int = 3, n_rows: int = 48, seed: int = 1, project=w8.project_w8a8) -> list:
    """W8A8 L-layer of the Wan-1.3B shapes on sampled rows: relative Frobenius
    error and largest element error / max|y| of the e4m3 projection (the
    per-token form, or with project=w8.project_mx_rows the MX form) when A_loc
    carries the GPU-like perturbation before its bf16 rounding."""
    w = synth.WORKLOADS["wan1.3b"]
    x = synth.single_layer_inputs(w, 1)
    W = synth.weight(w, 0)
    rows = np.sort(np.random.default_rng(5).choice(w.n_q, n_rows, replace=False))
    rows[-1] = w.n_q - 1
    a_ref, _ = orc.attention(x["q"][rows], np.concatenate([x["k_sink"], x["k_cur"]]),
                             np.concatenate([x["v_sink"], x["v_cur"]]), w.n_heads)
    y_ref = project(synth.round_bf16(a_ref.astype(np.float32)), W)
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(draws):
        an = a_ref * (1 + NOISE * rng.standard_normal(a_ref.shape))
        y = synth.round_bf16(project(synth.round_bf16(an.astype(np.float32)), W).astype(np.float32))
        out.append({"fro": float(np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref)),
                    "max": float(np.max(np.abs(y - y_ref)) / np.max(np.abs(y_ref)))})
    return out


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--full", action="store_true", help="also one absorbed layer of the 1.3B-shaped rollout")
    args = ap.parse_args()
    for r in absorb_chain_sensitivity(synth.WORKLOADS["rollout_small"], [0, 1, 2, 3]):
        print(f"rollout_small layer {r['layer']}: {r['rows']} rows, dW moves {r['dw_rel']:.2e}, "
              f"eps {r['eps']:.4f} moves {r['eps_rel']:.2e} (relative)")
    for name, proj in (("per-token", w8.project_w8a8), ("MX", w8.project_mx_rows)):
        for i, r in enumerate(w8a8_chain_sensitivity(project=proj)):
            print(f"W8A8 ({name}) L-layer draw {i}: y relative Frobenius {r['fro']:.2e}, "
                  f"largest element {r['max']:.2e}")
    if args.full:
        for r in absorb_chain_sensitivity(synth.WORKLOADS["rollout"], [0]):
            print(f"rollout (1.3B shapes) layer {r['layer']}: {r['rows']} rows, dW moves {r['dw_rel']:.2e}, "
                  f"eps {r['eps']:.4f} moves {r['eps_rel']:.2e}")


if __name__ == "__main__":
    main()

"""fp64 CPU oracle for the ISPA hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The product path (the CUDA library and
its Python binding) never imports, calls or links anything here, and this
module imports nothing from the product package.

Method: "Towards Memory-Efficient Autoregressive Video Generation via
Instance-Specific Parametric Absorption" (ISPA).  Citations name the page and
its section:
  [gist §2.1]  gist.science technical summary, section 2, stage 1
               "Dual-Stream Warmup" (A_full, A_loc, Decomposable Attention)
  [gist §2.2]  same page, stage 2 "Layer Absorb", the ridge objective and its
               closed-form minimiser
  [gist §2.3]  same page, stage 3 "Memory-Efficient Inference" (W_new = W + dW,
               eviction of K_hist, V_hist for the K selected layers)
  [gist §3]    same page, "Key Contributions" item 2 (online-softmax grounding)
  [gist sel]   same page, "Dynamic Layer Selection" (all layers ranked by
               their reconstruction error after the warm-up; the lowest are
               converted to L-layers)
  [abstract]   mlsanity.com arXiv abstract (up to 50% of the KV cache removed)

Everything is plain numpy in float64: attention materialises the score matrix
(one head and one block of query rows at a time, to bound memory); the ridge
problem is a dense LU solve of the normal equations.  No blocking, fusion or
reordering beyond that.

Readings of points the pages leave open (each is also a named constant or
argument below):
  * softmax scale 1/sqrt(head_dim) (SOFTMAX_SCALE);
  * no mask inside a chunk: block-causal streaming, every query of a chunk sees
    the sink, the history and the whole current chunk;
  * LSE is the natural log of the sum of exp of the scaled scores;
  * "A" is the concatenated multi-head attention output [n, D], the input of
    the output projection W [D_in, D_out] with y = A @ W;
  * the matrix norm of the objective is Frobenius;
  * lambda = lambda_abs + lambda_rel * trace(G) / D, G the un-normalised sum;
  * a layer's reconstruction error is the relative squared Frobenius error of
    the absorbed local stream over the warm-up rows,
    ||A_loc (W + dW) - A_full W||^2 / ||A_full W||^2, and selection takes the
    K smallest with ties to the lower layer index.
Pinned by tests/test_oracle.py (closed forms, special cases, a library
attention routine, brute-force minimisation of the objective, invariants).
"""
from __future__ import annotations

import math
from typing import Dict, List, Sequence, Tuple

import numpy as np

LAMBDA_REL = 1e-2     # lambda = LAMBDA_REL * trace(G) / D  (the pages give no value)


def SOFTMAX_SCALE(head_dim: int) -> float:
    return 1.0 / math.sqrt(head_dim)


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------
# Attention [gist §2.1]
# --------------------------------------------------------------------------
def attention(q, k, v, n_heads: int, scale: float | None = None,
              row_block: int = 512) -> Tuple[np.ndarray, np.ndarray]:
    """Softmax attention of every query row over the key set (k, v).

    q [n_q, D], k/v [n_k, D] with heads interleaved (D = n_heads * head_dim).
    Per head h and row i: s_ij = scale * <q_i, k_j>;  m_i = max_j s_ij;
    LSE_i = m_i + log sum_j exp(s_ij - m_i);  o_i = sum_j exp(s_ij - LSE_i) v_j.
    Returns o [n_q, D] and lse [n_heads, n_q]; an empty key set gives o = 0 and
    lse = -inf.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    n_q, D = q.shape
    d = D // n_heads
    s = SOFTMAX_SCALE(d) if scale is None else float(scale)
    o = np.zeros((n_q, D))
    lse = np.full((n_heads, n_q), -np.inf)
    if k.shape[0] == 0:
        return o, lse
    for h in range(n_heads):
        qh, kh, vh = q[:, h * d:(h + 1) * d], k[:, h * d:(h + 1) * d], v[:, h * d:(h + 1) * d]
        for r0 in range(0, n_q, row_block):
            S = s * (qh[r0:r0 + row_block] @ kh.T)
            m = S.max(axis=1, keepdims=True)
            E = np.exp(S - m)
            l = E.sum(axis=1, keepdims=True)
            o[r0:r0 + row_block, h * d:(h + 1) * d] = (E / l) @ vh
            lse[h, r0:r0 + row_block] = (m + np.log(l))[:, 0]
    return o, lse


def concat_segments(segments: Sequence[Tuple[np.ndarray, np.ndarray]], D: int):
    ks = [_f64(k) for k, _ in segments if len(k)]
    vs = [_f64(v) for _, v in segments if len(v)]
    if not ks:
        return np.zeros((0, D)), np.zeros((0, D))
    return np.concatenate(ks, 0), np.concatenate(vs, 0)


def dual_stream(q, local: Sequence[Tuple[np.ndarray, np.ndarray]],
                hist: Sequence[Tuple[np.ndarray, np.ndarray]], n_heads: int,
                scale: float | None = None) -> Dict[str, np.ndarray]:
    """Both streams of an F-layer during warm-up [gist §2.1].

    A_full attends to local + history keys, computed in ONE pass over their
    concatenation (not through the merge); A_loc attends to the local keys
    (sink + current) only; the history-only branch (O_hist, LSE_hist) is
    returned for the merge tests.  delta = A_full - A_loc.
    """
    q = _f64(q)
    D = q.shape[1]
    kl, vl = concat_segments(local, D)
    kh, vh = concat_segments(hist, D)
    a_loc, lse_loc = attention(q, kl, vl, n_heads, scale)
    o_hist, lse_hist = attention(q, kh, vh, n_heads, scale)
    a_full, lse_full = attention(q, np.concatenate([kl, kh], 0), np.concatenate([vl, vh], 0),
                                 n_heads, scale)
    return {"a_loc": a_loc, "lse_loc": lse_loc, "o_hist": o_hist, "lse_hist": lse_hist,
            "a_full": a_full, "lse_full": lse_full, "delta": a_full - a_loc}


def lse_merge(o_loc, lse_loc, o_hist, lse_hist, n_heads: int):
    """Post-hoc fusion of two attention branches through their LSE states
    [gist §2.1 "Decomposable Attention", gist §3 item 2].

    With L = log(exp(L_loc) + exp(L_hist)) per (head, row), the full output is
    exp(L_loc - L) * O_loc + exp(L_hist - L) * O_hist.  An empty branch has
    LSE = -inf and weight 0; when both are empty (L = -inf) both weights are 0,
    so A_full = 0 and L = -inf, which is attention over the empty union of the
    two key sets.  Returns (A_full, delta = A_full - O_loc, L).
    """
    o_loc, o_hist = _f64(o_loc), _f64(o_hist)
    lse_loc, lse_hist = _f64(lse_loc), _f64(lse_hist)
    n_q, D = o_loc.shape
    d = D // n_heads
    L = np.logaddexp(lse_loc, lse_hist)                     # [H, n_q]
    empty = np.isneginf(L)
    Ls = np.where(empty, 0.0, L)
    w_loc = np.where(empty, 0.0, np.exp(np.where(empty, 0.0, lse_loc - Ls)))
    w_hist = np.where(empty, 0.0, np.exp(np.where(empty, 0.0, lse_hist - Ls)))
    w_loc_rows = np.repeat(w_loc.T, d, axis=1)              # [n_q, D], head-major columns
    w_hist_rows = np.repeat(w_hist.T, d, axis=1)
    a_full = w_loc_rows * o_loc + w_hist_rows * o_hist
    return a_full, a_full - o_loc, L


# --------------------------------------------------------------------------
# Layer Absorb [gist §2.2]
# --------------------------------------------------------------------------
def gram(a_loc, delta) -> Tuple[np.ndarray, np.ndarray]:
    """Sufficient statistics of the ridge problem over a block of rows:
    G = A_loc^T A_loc and R = A_loc^T (A_full - A_loc)."""
    a_loc, delta = _f64(a_loc), _f64(delta)
    return a_loc.T @ a_loc, a_loc.T @ delta


def ridge_lambda(G, lambda_rel: float = LAMBDA_REL, lambda_abs: float = 0.0) -> float:
    G = _f64(G)
    return float(lambda_abs + lambda_rel * np.trace(G) / G.shape[0])


def absorb(G, R, W, lam: float) -> np.ndarray:
    """Closed-form weight modulation dW = (G + lam I)^-1 R W  [gist §2.2],
    by a dense LU solve of the normal equations."""
    G, R, W = _f64(G), _f64(R), _f64(W)
    M = G + lam * np.eye(G.shape[0])
    return np.linalg.solve(M, R @ W)


def objective(a_loc, a_full, W, dW, lam: float) -> float:
    """The ridge objective of [gist §2.2] with the Frobenius norm:
    ||A_loc (W + dW) - A_full W||^2 + lam ||dW||^2."""
    a_loc, a_full, W, dW = _f64(a_loc), _f64(a_full), _f64(W), _f64(dW)
    r = a_loc @ (W + dW) - a_full @ W
    return float(np.sum(r * r) + lam * np.sum(dW * dW))


def reconstruction_error(a_loc, a_full, W, dW) -> float:
    """Reconstruction error of one layer after the warm-up [gist sel]: the
    relative squared Frobenius error of the absorbed local stream,
    ||A_loc (W + dW) - A_full W||^2 / ||A_full W||^2 (0 when both vanish,
    +inf when only the denominator does)."""
    a_loc, a_full, W, dW = _f64(a_loc), _f64(a_full), _f64(W), _f64(dW)
    target = a_full @ W
    r = a_loc @ (W + dW) - target
    num, den = float(np.sum(r * r)), float(np.sum(target * target))
    if den == 0.0:
        return 0.0 if num == 0.0 else math.inf
    return num / den


def select_layers(eps: Sequence[float], k: int) -> List[int]:
    """The k layers converted to L-layers [gist sel]: the k smallest
    reconstruction errors, ties to the lower layer index, NaN ranked after
    every number; returned in increasing layer order."""
    if not 0 <= k <= len(eps):
        raise ValueError("k must lie in [0, number of layers]")
    order = sorted(range(len(eps)), key=lambda l: (math.isnan(eps[l]), 0.0 if math.isnan(eps[l]) else eps[l], l))
    return sorted(order[:k])


def modulated_weight(W, dW) -> np.ndarray:
    """W_new = W + dW [gist §2.3]."""
    return _f64(W) + _f64(dW)


def project(a, W) -> np.ndarray:
    """Layer output y = A @ W (A [n, D_in], W [D_in, D_out])."""
    return _f64(a) @ _f64(W)


# --------------------------------------------------------------------------
# Streaming bookkeeping [gist §2.1, §2.3; abstract]
# --------------------------------------------------------------------------
def chunk_token_ranges(chunk: int, frame_tokens: int, chunk_frames: int,
                       sink_frames: int = 1) -> Dict[str, Tuple[int, int]]:
    """Half-open token ranges of the sink, history and current segments seen by
    the queries of rollout chunk ``chunk`` (0-based) of a stream that starts at
    token 0.  Chunk 0 holds the sink frame inside its own current chunk, so it
    has no separate sink and no history; chunk c >= 1 sees sink = the first
    ``sink_frames`` frames, history = the frames between the sink and the
    current chunk, current = frames [c*chunk_frames, (c+1)*chunk_frames).  The
    sink precedes the current chunk, so chunk c >= 1 needs
    sink_frames <= c*chunk_frames (ValueError otherwise)."""
    F, cf = frame_tokens, chunk_frames
    if chunk > 0 and sink_frames > chunk * cf:
        raise ValueError("the sink must end before the current chunk starts")
    cur = (chunk * cf * F, (chunk + 1) * cf * F)
    if chunk == 0:
        return {"sink": (0, 0), "hist": (0, 0), "cur": cur}
    return {"sink": (0, sink_frames * F), "hist": (sink_frames * F, chunk * cf * F), "cur": cur}


def layer_mask(n_layers: int, absorbed: Sequence[int]) -> int:
    """Bit l set <=> layer l is an L-layer (history evicted) [gist §2.3]."""
    m = 0
    for l in absorbed:
        m |= 1 << l
    return m


def resident_tokens(chunk: int, is_l_layer: bool, transitioned: bool, frame_tokens: int,
                    chunk_frames: int, sink_frames: int = 1) -> int:
    """KV tokens a layer holds while it runs chunk ``chunk``: an F-layer keeps
    every frame up to the current chunk; an L-layer after the transition keeps
    only the sink and the current chunk [gist §2.3]."""
    r = chunk_token_ranges(chunk, frame_tokens, chunk_frames, sink_frames)
    if is_l_layer and transitioned:
        return (r["sink"][1] - r["sink"][0]) + (r["cur"][1] - r["cur"][0])
    return r["cur"][1]


def kv_bytes(chunk: int, n_layers: int, mask: int, transitioned: bool, frame_tokens: int,
             chunk_frames: int, d_model: int, elem_bytes: int, sink_frames: int = 1) -> int:
    """Total K and V bytes held by all layers at chunk ``chunk``."""
    total = 0
    for l in range(n_layers):
        t = resident_tokens(chunk, bool((mask >> l) & 1), transitioned, frame_tokens,
                            chunk_frames, sink_frames)
        total += t * 2 * d_model * elem_bytes
    return total

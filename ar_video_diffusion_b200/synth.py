"""Seeded synthetic inputs for the ISPA hot path.

This module is the only code shared by the fp64 CPU oracle (``oracle/``) and the
CUDA path.  It draws random tensors and rounds them to the storage dtype; it
holds none of the method's arithmetic (no attention, no statistics, no solve).

Workload shapes follow the streaming setting of "Towards Memory-Efficient
Autoregressive Video Generation via Instance-Specific Parametric Absorption"
(gist.science technical summary, section 2, "Dual-Stream Warmup"): a chunk's
queries attend to a sink frame, the evicted-history frames and the current
chunk.  The latent-frame sizes (1560 tokens per latent frame, 12/40 heads of
dim 128) are those of Wan-1.3B / Wan-14B shaped layers.

Generator recipe (all draws fp32 from numpy PCG64):
  * every tensor has its own stream, ``SeedSequence([seed, layer, key, tensor_id])``
    where ``key`` is a latent-frame index for K/V and a chunk index for Q;
  * Q, V ~ N(0, 1);
  * K = N(0, 1) + 0.5 * sum_{r<4} c[t, r] * B[h, frame(t), r, :], with
    c ~ N(0, 1) per token and B ~ N(0, 1) per (head, latent frame), so that the
    tokens of one latent frame share a rank-4 component and softmax is peaked;
  * W ~ N(0, 1/D), shape [D_in, D_out], used as y = A @ W;
  * bf16 workloads round every fp32 draw to the nearest bf16 (ties to even);
    both sides then consume exactly these representable values.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np

# tensor ids inside a SeedSequence key
_T_Q, _T_K_NOISE, _T_K_COEF, _T_K_BASIS, _T_V, _T_W = 1, 2, 3, 4, 5, 6
RANK = 4            # rank of the per-frame shared key component
RANK_SCALE = 0.5    # its scale


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shapes of one synthetic streaming-attention layer.

    Token counts are multiples of ``frame_tokens``; the sink is one latent frame.
    """
    name: str
    seed: int
    n_heads: int
    head_dim: int
    frame_tokens: int
    sink_frames: int
    chunk_frames: int
    hist_frames: int
    dtype: str                 # "bf16" or "f32"
    warm_chunks: int           # chunks whose rows enter G, R
    n_layers: int = 1
    post_chunks: int = 0       # chunks run after the transition (rollout only)

    @property
    def d_model(self) -> int:
        return self.n_heads * self.head_dim

    @property
    def n_sink(self) -> int:
        return self.sink_frames * self.frame_tokens

    @property
    def n_q(self) -> int:
        return self.chunk_frames * self.frame_tokens

    @property
    def n_hist(self) -> int:
        return self.hist_frames * self.frame_tokens


# The five workloads: tiny fp32; Wan-1.3B shaped; long history; Wan-14B shaped;
# 30-layer streaming rollout with 1.3B shapes.
WORKLOADS: Dict[str, Workload] = {
    "tiny_f32": Workload("tiny_f32", seed=0, n_heads=2, head_dim=64, frame_tokens=16,
                         sink_frames=1, chunk_frames=4, hist_frames=16, dtype="f32",
                         warm_chunks=4),
    "wan1.3b": Workload("wan1.3b", seed=1, n_heads=12, head_dim=128, frame_tokens=1560,
                        sink_frames=1, chunk_frames=3, hist_frames=12, dtype="bf16",
                        warm_chunks=4),
    "long_hist": Workload("long_hist", seed=2, n_heads=12, head_dim=128, frame_tokens=1560,
                          sink_frames=1, chunk_frames=3, hist_frames=60, dtype="bf16",
                          warm_chunks=20),
    # a long-lived F-layer: 129 latent frames (201240 tokens) of history
    "hist_200k": Workload("hist_200k", seed=5, n_heads=12, head_dim=128, frame_tokens=1560,
                          sink_frames=1, chunk_frames=3, hist_frames=129, dtype="bf16",
                          warm_chunks=1),
    "wan14b": Workload("wan14b", seed=3, n_heads=40, head_dim=128, frame_tokens=1560,
                       sink_frames=1, chunk_frames=3, hist_frames=12, dtype="bf16",
                       warm_chunks=4),
    "rollout": Workload("rollout", seed=4, n_heads=12, head_dim=128, frame_tokens=1560,
                        sink_frames=1, chunk_frames=3, hist_frames=0, dtype="bf16",
                        warm_chunks=4, n_layers=30, post_chunks=20),
    # the rollout schedule at a size the CPU oracle follows end to end (every
    # row of every chunk): 2 heads, 120 tokens per frame (360 chunk queries,
    # a ragged third query tile), 4 layers
    "rollout_small": Workload("rollout_small", seed=6, n_heads=2, head_dim=128, frame_tokens=120,
                              sink_frames=1, chunk_frames=3, hist_frames=0, dtype="bf16",
                              warm_chunks=4, n_layers=4, post_chunks=2),
}


def _rng(seed: int, layer: int, key: int, tensor_id: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, layer, key, tensor_id])))


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bfloat16 (ties to even); returns fp32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)
    # NaN/Inf are never drawn; keep them untouched anyway
    special = (u & np.uint32(0x7F800000)) == np.uint32(0x7F800000)
    r = np.where(special, u, r).astype(np.uint32)
    return r.view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Upper 16 bits of fp32 values that are already bf16-representable."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return (u >> np.uint32(16)).astype(np.uint16)


def _store(x: np.ndarray, dtype: str) -> np.ndarray:
    x = x.astype(np.float32, copy=False)
    return round_bf16(x) if dtype == "bf16" else x


def frame_kv(w: Workload, layer: int, frame: int) -> (np.ndarray, np.ndarray):
    """K and V of one latent frame, each ``[frame_tokens, D]`` (token-major, heads interleaved)."""
    F, H, d = w.frame_tokens, w.n_heads, w.head_dim
    noise = _rng(w.seed, layer, frame, _T_K_NOISE).standard_normal((F, H * d), dtype=np.float32)
    coef = _rng(w.seed, layer, frame, _T_K_COEF).standard_normal((F, RANK), dtype=np.float32)
    basis = _rng(w.seed, layer, frame, _T_K_BASIS).standard_normal((H, RANK, d), dtype=np.float32)
    shared = np.einsum("tr,hrd->thd", coef, basis, optimize=True).reshape(F, H * d)
    k = noise + np.float32(RANK_SCALE) * shared
    v = _rng(w.seed, layer, frame, _T_V).standard_normal((F, H * d), dtype=np.float32)
    return _store(k, w.dtype), _store(v, w.dtype)


def frames_kv(w: Workload, layer: int, frames: List[int]) -> (np.ndarray, np.ndarray):
    """Concatenated K, V of the listed latent frames, in list order."""
    D = w.d_model
    if not frames:
        return np.zeros((0, D), np.float32), np.zeros((0, D), np.float32)
    ks, vs = zip(*(frame_kv(w, layer, f) for f in frames))
    return np.concatenate(ks, 0), np.concatenate(vs, 0)


def chunk_q(w: Workload, layer: int, chunk: int, n_rows: Optional[int] = None) -> np.ndarray:
    """Queries of one chunk, ``[n_q, D]``."""
    n = w.n_q if n_rows is None else n_rows
    q = _rng(w.seed, layer, chunk, _T_Q).standard_normal((n, w.d_model), dtype=np.float32)
    return _store(q, w.dtype)


def weight(w: Workload, layer: int) -> np.ndarray:
    """Output projection W ~ N(0, 1/D), ``[D_in, D_out]`` (y = A @ W)."""
    D = w.d_model
    W = _rng(w.seed, layer, 0, _T_W).standard_normal((D, D), dtype=np.float32) / np.float32(np.sqrt(D))
    return _store(W, w.dtype)


def single_layer_frames(w: Workload, warm_chunk: int) -> Dict[str, List[int]]:
    """Frame lists of warm-up chunk ``warm_chunk`` for a single-layer workload.

    Sink = frame 0; history = frames 1..hist_frames (shared by every chunk);
    the current chunk takes fresh frames after the history, so each warm-up
    chunk sees its own current keys and queries.
    """
    first_cur = w.sink_frames + w.hist_frames + warm_chunk * w.chunk_frames
    return {
        "sink": list(range(w.sink_frames)),
        "hist": list(range(w.sink_frames, w.sink_frames + w.hist_frames)),
        "cur": list(range(first_cur, first_cur + w.chunk_frames)),
    }


def single_layer_inputs(w: Workload, warm_chunk: int, layer: int = 0) -> Dict[str, np.ndarray]:
    fr = single_layer_frames(w, warm_chunk)
    ks, vs = frames_kv(w, layer, fr["sink"])
    kh, vh = frames_kv(w, layer, fr["hist"])
    kc, vc = frames_kv(w, layer, fr["cur"])
    return {"q": chunk_q(w, layer, warm_chunk), "k_sink": ks, "v_sink": vs,
            "k_hist": kh, "v_hist": vh, "k_cur": kc, "v_cur": vc}


def random_case(seed: int, n_q: int, n_heads: int, head_dim: int, seg_tokens: List[int],
                dtype: str = "bf16", rank_scale: float = RANK_SCALE) -> Dict[str, object]:
    """Free-form case for edge-case tests: Q plus one (K, V) pair per segment length."""
    D = n_heads * head_dim
    g = _rng(seed, 99, 0, 0)
    q = _store(g.standard_normal((n_q, D), dtype=np.float32), dtype)
    segs = []
    for n in seg_tokens:
        k = g.standard_normal((n, D), dtype=np.float32)
        if n:
            coef = g.standard_normal((n, RANK), dtype=np.float32)
            basis = g.standard_normal((n_heads, RANK, head_dim), dtype=np.float32)
            k = k + np.float32(rank_scale) * np.einsum("tr,hrd->thd", coef, basis).reshape(n, D)
        v = g.standard_normal((n, D), dtype=np.float32)
        segs.append((_store(k, dtype), _store(v, dtype)))
    return {"q": q, "segments": segs}


# ----------------------------------------------------------------------------
# Device-side generator for the streaming rollout: the same recipe (noise plus
# a rank-4 per-frame key component, W ~ N(0, 1/D)) drawn with torch's CUDA RNG
# so that thousands of frames are produced in milliseconds.  Each tensor is
# seeded from the same (seed, layer, key, tensor_id) tuple as the host recipe;
# the values differ from the host generator's but are fixed by the seed.
def _seed_int(seed: int, layer: int, key: int, tensor_id: int) -> int:
    s = np.random.SeedSequence([seed, layer, key, tensor_id]).generate_state(2, dtype=np.uint32)
    return (int(s[0]) << 31) ^ int(s[1])


def _randn_device(shape, seed_int: int, device):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed_int)
    return torch.randn(*shape, generator=g, device=device, dtype=torch.float32)


def frame_kv_device(w: Workload, layer: int, frame: int, device):
    """K and V of one latent frame on `device`, bf16 [frame_tokens, D]."""
    import torch
    F, H, d = w.frame_tokens, w.n_heads, w.head_dim
    noise = _randn_device((F, H * d), _seed_int(w.seed, layer, frame, _T_K_NOISE), device)
    coef = _randn_device((F, RANK), _seed_int(w.seed, layer, frame, _T_K_COEF), device)
    basis = _randn_device((H, RANK, d), _seed_int(w.seed, layer, frame, _T_K_BASIS), device)
    shared = (coef @ basis.reshape(H, RANK, d).permute(1, 0, 2).reshape(RANK, H * d))
    k = noise + RANK_SCALE * shared
    v = _randn_device((F, H * d), _seed_int(w.seed, layer, frame, _T_V), device)
    return k.to(torch.bfloat16), v.to(torch.bfloat16)


def chunk_q_device(w: Workload, layer: int, chunk: int, device):
    import torch
    q = _randn_device((w.n_q, w.d_model), _seed_int(w.seed, layer, chunk, _T_Q), device)
    return q.to(torch.bfloat16)


def weight_device(w: Workload, layer: int, device):
    import torch
    D = w.d_model
    W = _randn_device((D, D), _seed_int(w.seed, layer, 0, _T_W), device) / float(np.sqrt(D))
    return W.to(torch.bfloat16)

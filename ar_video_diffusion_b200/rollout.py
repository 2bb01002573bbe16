"""Streaming rollout of the ISPA hot path over all layers of a model.

The schedule of "Towards Memory-Efficient Autoregressive Video Generation via
Instance-Specific Parametric Absorption" (gist.science technical summary,
section 2):
  * warm-up chunks (stage 1, "Dual-Stream Warmup"): every layer is an F-layer
    running the dual stream -- A_loc over sink + current chunk, A_full over
    sink + history + current chunk -- and projects A_full with its W; the
    layers selected for absorption accumulate G and R from their rows;
  * transition (stage 2, "Layer Absorb"): each selected layer solves
    dW = (G + lambda I)^-1 R W, forms W_new = W + dW and evicts its history
    K/V, keeping only the sink frame;
  * later chunks (stage 3): selected layers (L-layers) attend to sink +
    current only and project with W_new; the others (F-layers) attend to the
    whole growing cache and project with W.
Chunk 0 holds the sink frame inside its own current chunk, so it has no
separate sink and no history.  Every step runs in libispa's kernels; this
module only owns the device buffers (torch tensors), the chunk schedule and the
KV bookkeeping.  Layer inputs (queries and each new frame's K/V) come from the
seeded device generator in ``synth``: no trained model is involved.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, Dict, List, Optional, Sequence

import torch

from . import ispa, synth


@dataclasses.dataclass
class ChunkReport:
    chunk: int
    phase: str              # "warmup", "post"
    gpu_ms: float           # device time of all layers' attention + projection (+ statistics)
    kv_bytes: int           # K/V bytes resident while the chunk runs (bookkeeping)
    kv_bytes_all_f: int     # the same if no layer were absorbed


class Rollout:
    def __init__(self, w: synth.Workload, absorbed: Optional[Sequence[int]] = None, device="cuda",
                 lambda_rel: float = 1e-2,
                 on_layer: Optional[Callable[[int, int, dict], None]] = None):
        self.w = w
        self.device = torch.device(device)
        self.L = w.n_layers
        self.absorbed = sorted(set(range(0, self.L, 2) if absorbed is None else absorbed))
        self.mask = 0
        for l in self.absorbed:
            self.mask |= 1 << l
        self.n_chunks = w.warm_chunks + w.post_chunks
        self.lambda_rel = lambda_rel
        self.on_layer = on_layer
        F, cf, D = w.frame_tokens, w.chunk_frames, w.d_model
        self.F, self.cf, self.D = F, cf, D
        self.chunk_tokens = cf * F
        bf = dict(dtype=torch.bfloat16, device=self.device)
        f32 = dict(dtype=torch.float32, device=self.device)
        self.W = [synth.weight_device(w, l, self.device) for l in range(self.L)]
        self.W_new: List[Optional[torch.Tensor]] = [None] * self.L
        self.dW: List[Optional[torch.Tensor]] = [None] * self.L
        # K/V caches: F-layers hold every frame of the run; absorbed layers hold
        # the warm-up frames until the transition, then only sink + current
        full = self.n_chunks * self.chunk_tokens
        warm = w.warm_chunks * self.chunk_tokens
        self.k: List[torch.Tensor] = []
        self.v: List[torch.Tensor] = []
        for l in range(self.L):
            n = warm if l in self.absorbed else full
            self.k.append(torch.empty(n, D, **bf))
            self.v.append(torch.empty(n, D, **bf))
        self.G = {l: torch.zeros(D, D, **f32) for l in self.absorbed}
        self.R = {l: torch.zeros(D, D, **f32) for l in self.absorbed}
        self.transitioned = False
        n_q = self.chunk_tokens
        self.q = [torch.empty(n_q, D, **bf) for _ in range(self.L)]
        self.out = {"a_loc": torch.empty(n_q, D, **bf), "a_full": torch.empty(n_q, D, **bf),
                    "a_delta": torch.empty(n_q, D, **bf), "lse_loc": torch.empty(w.n_heads, n_q, **f32),
                    "lse_full": torch.empty(w.n_heads, n_q, **f32)}
        self.y = torch.empty(n_q, D, **bf)
        self.status = ispa.new_status(self.device)
        self.workspace = ispa.absorb_workspace(D, self.device)
        self.reports: List[ChunkReport] = []
        self.absorb_ms: List[float] = []

    # ----------------------------------------------------------- bookkeeping
    def ranges(self, c: int) -> Dict[str, tuple]:
        return ispa.ispa_chunk_token_ranges(c, self.F, self.cf, self.w.sink_frames)

    def kv_bytes(self, c: int, all_f: bool = False) -> int:
        mask = 0 if all_f else self.mask
        return ispa.ispa_kv_bytes(c, self.L, mask, self.transitioned, self.F, self.cf, self.D, 2,
                                  self.w.sink_frames)

    def is_l_layer(self, l: int) -> bool:
        return self.transitioned and l in self.absorbed

    # --------------------------------------------------------------- inputs
    def load_chunk_inputs(self, c: int):
        """Queries and the current chunk's K/V of every layer (the generator
        stands in for the model's own Q/K/V projections)."""
        r = self.ranges(c)
        for l in range(self.L):
            self.q[l].copy_(synth.chunk_q_device(self.w, l, c, self.device))
            for j in range(self.cf):
                frame = c * self.cf + j
                k, v = synth.frame_kv_device(self.w, l, frame, self.device)
                if self.is_l_layer(l):
                    pos = self.w.sink_frames * self.F + j * self.F  # after the kept sink frame
                else:
                    pos = r["cur"][0] + j * self.F
                self.k[l][pos:pos + self.F].copy_(k)
                self.v[l][pos:pos + self.F].copy_(v)

    # ------------------------------------------------------------ transition
    def transition(self):
        """Absorb the history of every selected layer and evict its K/V."""
        stream = torch.cuda.current_stream(self.device)
        sink = self.w.sink_frames * self.F
        events = []
        for l in self.absorbed:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            dW, Wn = ispa.absorb_solve(self.G[l], self.R[l], self.W[l], lambda_rel=self.lambda_rel,
                                       workspace=self.workspace, status=self.status)
            e1.record(stream)
            events.append((e0, e1))
            self.dW[l], self.W_new[l] = dW, Wn
            # keep the sink frame, drop the history: a buffer for sink + one chunk
            k_small = torch.empty(sink + self.chunk_tokens, self.D, dtype=torch.bfloat16, device=self.device)
            v_small = torch.empty_like(k_small)
            k_small[:sink].copy_(self.k[l][:sink])
            v_small[:sink].copy_(self.v[l][:sink])
            self.k[l], self.v[l] = k_small, v_small
        torch.cuda.synchronize(self.device)
        self.absorb_ms = [a.elapsed_time(b) for a, b in events]
        self.transitioned = True
        self.G.clear()
        self.R.clear()

    # ----------------------------------------------------------------- chunk
    def run_chunk(self, c: int):
        """All layers' attention + projection for chunk c (plus the statistics
        of the selected layers during warm-up)."""
        r = self.ranges(c)
        warm = c < self.w.warm_chunks
        H = self.w.n_heads
        for l in range(self.L):
            k, v = self.k[l], self.v[l]
            if self.is_l_layer(l):
                n_loc = self.w.sink_frames * self.F + self.chunk_tokens
                local = [(k[:n_loc], v[:n_loc])]
                y, _ = ispa.local_attention_project(self.q[l], local, self.W_new[l], H, y=self.y,
                                                    a_loc=self.out["a_loc"], status=self.status)
                info = {"mode": "L", "local": local, "hist": [], "W": self.W_new[l]}
            else:
                cb, ce = r["cur"]
                local = [(k[cb:ce], v[cb:ce])]
                if r["sink"][1] > r["sink"][0]:
                    local.insert(0, (k[r["sink"][0]:r["sink"][1]], v[r["sink"][0]:r["sink"][1]]))
                hist = [(k[r["hist"][0]:r["hist"][1]], v[r["hist"][0]:r["hist"][1]])] \
                    if r["hist"][1] > r["hist"][0] else []
                if warm:
                    ispa.dual_attention(self.q[l], local, hist, H, out=self.out, status=self.status)
                    if l in self.absorbed:
                        ispa.gram_accumulate(self.out["a_loc"], self.out["a_delta"], self.G[l], self.R[l],
                                             zero_first=(c == 0))
                else:
                    ispa.dual_attention(self.q[l], local, hist, H, dual=False, out=self.out, status=self.status)
                ispa.project(self.out["a_full"], self.W[l], self.y)
                info = {"mode": "F", "local": local, "hist": hist, "W": self.W[l]}
            if self.on_layer is not None:
                info.update(q=self.q[l], y=self.y, out=self.out)
                self.on_layer(l, c, info)

    def run(self, on_chunk_start: Optional[Callable[[int], None]] = None) -> List[ChunkReport]:
        stream = torch.cuda.current_stream(self.device)
        for c in range(self.n_chunks):
            if c == self.w.warm_chunks and not self.transitioned:
                self.transition()
            self.load_chunk_inputs(c)
            torch.cuda.synchronize(self.device)
            if on_chunk_start:
                on_chunk_start(c)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            self.run_chunk(c)
            e1.record(stream)
            torch.cuda.synchronize(self.device)
            code = int(self.status[0].item())
            if code != 0:
                raise ispa.IspaError(code, f"rollout chunk {c}", "device status")
            self.reports.append(ChunkReport(c, "warmup" if c < self.w.warm_chunks else "post",
                                            e0.elapsed_time(e1), self.kv_bytes(c), self.kv_bytes(c, all_f=True)))
        return self.reports

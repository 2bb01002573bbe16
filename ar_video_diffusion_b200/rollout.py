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
    K/V, keeping only the sink frame.  The selected layers are either a fixed
    set (the even layers by default) or, with ``selection="instance"``, the K
    layers of lowest reconstruction error ("Dynamic Layer Selection" of the
    same page): every layer then also accumulates E = dA^T dA, is absorbed at
    the transition and ranked by eps = ||A_loc W_new - A_full W||^2 /
    ||A_full W||^2, evaluated from G, R, E without its activations;
  * later chunks (stage 3): selected layers (L-layers) attend to sink +
    current only and project with W_new; the others (F-layers) attend to the
    whole growing cache and project with W.  With ``precision="w8a8"`` the
    L-layers project with the post-training W8A8 reading of the same page's
    "Speedup" item: W_new quantised to e4m3 once, after the absorb, and each
    chunk's A_loc quantised per token; with ``precision="mx"`` the attention
    epilogue writes A_loc as MX codes (one power-of-two scale per 32
    channels) and the L-layer runs the block-scaled product.
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
                 on_layer: Optional[Callable[[int, int, dict], None]] = None,
                 selection: str = "fixed", rank_all: bool = False, precision: str = "bf16"):
        """``absorbed``: the fixed L-layer set (default: even layers); with
        ``selection="instance"`` only its size K is used and the K layers of
        lowest reconstruction error are chosen at the transition.
        ``rank_all``: rank every layer (eps of each) even for a fixed set."""
        if selection not in ("fixed", "instance"):
            raise ValueError("selection must be 'fixed' or 'instance'")
        if precision not in ("bf16", "w8a8", "mx"):
            raise ValueError("precision must be 'bf16', 'w8a8' or 'mx'")
        self.precision = precision
        self.w8: Dict[int, tuple] = {}  # L-layer -> (e4m3 codes of W_new, transposed; per-channel scales)
        self.w = w
        self.device = torch.device(device)
        self.L = w.n_layers
        self.absorbed = sorted(set(range(0, self.L, 2) if absorbed is None else absorbed))
        self.selection = selection
        self.k_select = len(self.absorbed)
        self.rank = rank_all or selection == "instance"
        if selection == "instance":
            self.absorbed = []  # chosen at the transition
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
        self.stats_layers = list(range(self.L)) if self.rank else list(self.absorbed)
        self.G = {l: torch.zeros(D, D, **f32) for l in self.stats_layers}
        self.R = {l: torch.zeros(D, D, **f32) for l in self.stats_layers}
        self.E = {l: torch.zeros(D, D, **f32) for l in self.stats_layers} if self.rank else {}
        self.eps: List[float] = []      # reconstruction error of every layer (when ranked)
        self.dW_ranked: Dict[int, torch.Tensor] = {}  # every ranked layer's dW (when ranked)
        self.select_ms = 0.0
        self.transitioned = False
        n_q = self.chunk_tokens
        self.q = [torch.empty(n_q, D, **bf) for _ in range(self.L)]
        self.out = {"a_loc": torch.empty(n_q, D, **bf), "a_full": torch.empty(n_q, D, **bf),
                    "a_delta": torch.empty(n_q, D, **bf), "lse_loc": torch.empty(w.n_heads, n_q, **f32),
                    "lse_full": torch.empty(w.n_heads, n_q, **f32)}
        self.y = torch.empty(n_q, D, **bf)
        self.w8_out = None
        if precision == "w8a8":
            self.w8_out = {"y": self.y, "a_loc": self.out["a_loc"],
                           "a_codes": torch.empty(n_q, D, dtype=torch.uint8, device=self.device),
                           "a_scales": torch.empty(n_q, dtype=torch.float32, device=self.device)}
        elif precision == "mx":
            self.w8_out = {"y": self.y, "a_codes": torch.empty(n_q, D, dtype=torch.uint8, device=self.device),
                           "a_exps": torch.empty(n_q, D // 32, dtype=torch.uint8, device=self.device)}
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
    def rank_layers(self):
        """Absorb every layer and evaluate its reconstruction error; with
        instance selection, choose the K layers of lowest error."""
        stream = torch.cuda.current_stream(self.device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ws = torch.empty(ispa.ispa_layer_error_workspace_bytes(self.D), dtype=torch.uint8, device=self.device)
        num_den = torch.empty(self.L, 2, dtype=torch.float64, device=self.device)
        cand, ev = {}, {}
        e0.record(stream)
        for l in range(self.L):
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            dW, Wn = ispa.absorb_solve(self.G[l], self.R[l], self.W[l], lambda_rel=self.lambda_rel,
                                       workspace=self.workspace, status=self.status)
            a1.record(stream)
            ispa.layer_error(self.G[l], self.R[l], self.E[l], self.W[l], dW, workspace=ws, num_den=num_den[l])
            cand[l], ev[l] = (dW, Wn), (a0, a1)
        e1.record(stream)
        torch.cuda.synchronize(self.device)
        self.select_ms = e0.elapsed_time(e1)  # every layer's absorb and error
        nd = num_den.cpu().tolist()
        self.eps = [n / d if d > 0 else float("nan") for n, d in nd]
        if self.selection == "instance":
            self.absorbed = ispa.select_layers(self.eps, self.k_select)
            self.mask = 0
            for l in self.absorbed:
                self.mask |= 1 << l
        self.dW_ranked = {l: cand[l][0] for l in cand}
        for l in self.absorbed:
            self.dW[l], self.W_new[l] = cand[l]
        self.absorb_ms = [ev[l][0].elapsed_time(ev[l][1]) for l in self.absorbed]

    def transition(self):
        """Absorb the history of every selected layer and evict its K/V."""
        stream = torch.cuda.current_stream(self.device)
        sink = self.w.sink_frames * self.F
        events = []
        if self.rank:
            self.rank_layers()
        for l in self.absorbed:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            if not self.rank:
                dW, Wn = ispa.absorb_solve(self.G[l], self.R[l], self.W[l], lambda_rel=self.lambda_rel,
                                           workspace=self.workspace, status=self.status)
                self.dW[l], self.W_new[l] = dW, Wn
            e1.record(stream)
            events.append((e0, e1))
            # keep the sink frame, drop the history: a buffer for sink + one chunk
            k_small = torch.empty(sink + self.chunk_tokens, self.D, dtype=torch.bfloat16, device=self.device)
            v_small = torch.empty_like(k_small)
            k_small[:sink].copy_(self.k[l][:sink])
            v_small[:sink].copy_(self.v[l][:sink])
            self.k[l], self.v[l] = k_small, v_small
        if self.precision in ("w8a8", "mx"):
            for l in self.absorbed:
                self.w8[l] = ispa.quantize_e4m3_weight(self.W_new[l])
        torch.cuda.synchronize(self.device)
        if not self.rank:
            self.absorb_ms = [a.elapsed_time(b) for a, b in events]
        self.transitioned = True
        self.G.clear()
        self.R.clear()
        self.E.clear()

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
                if self.precision == "w8a8":
                    qwt, sw = self.w8[l]
                    ispa.local_attention_project_w8a8(self.q[l], local, qwt, sw, H, out=self.w8_out,
                                                      status=self.status)
                elif self.precision == "mx":
                    qwt, sw = self.w8[l]
                    ispa.local_attention_project_mx(self.q[l], local, qwt, sw, H, out=self.w8_out,
                                                    status=self.status)
                else:
                    ispa.local_attention_project(self.q[l], local, self.W_new[l], H, y=self.y,
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
                    if l in self.G:
                        ispa.gram_accumulate(self.out["a_loc"], self.out["a_delta"], self.G[l], self.R[l],
                                             zero_first=(c == 0))
                        if self.rank:
                            ispa.sym_gram_accumulate(self.out["a_delta"], self.E[l], zero_first=(c == 0))
                else:
                    ispa.dual_attention(self.q[l], local, hist, H, dual=False, out=self.out, status=self.status)
                ispa.project(self.out["a_full"], self.W[l], self.y)
                info = {"mode": "F", "local": local, "hist": hist, "W": self.W[l]}
            if self.on_layer is not None:
                info.update(q=self.q[l], y=self.y, out=self.out)
                self.on_layer(l, c, info)

    def chunk_graph_ms(self, c: int, iters: int = 5) -> float:
        """Device time of chunk c's launches (every layer's attention and
        projection) captured into one CUDA graph and replayed: the chunk
        latency without host launch gaps.  Chunk c's key ranges are used with
        whatever the caches hold, which does not change the work."""
        if self.on_layer is not None:
            raise RuntimeError("chunk graphs need on_layer=None")
        if c < self.w.warm_chunks or not self.transitioned:
            raise ValueError("only post-transition chunks are captured")
        stream = torch.cuda.current_stream(self.device)
        self.run_chunk(c)  # every first-call set-up happens outside the capture
        torch.cuda.synchronize(self.device)
        side = torch.cuda.Stream(self.device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side, capture_error_mode="relaxed"):
            self.run_chunk(c)
        g.replay()
        torch.cuda.synchronize(self.device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(iters):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize(self.device)
        del g
        return e0.elapsed_time(e1) / iters

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
                raise ispa.IspaError(code, f"rollout chunk {c}", f"device status detail {int(self.status[1].item())}")
            self.reports.append(ChunkReport(c, "warmup" if c < self.w.warm_chunks else "post",
                                            e0.elapsed_time(e1), self.kv_bytes(c), self.kv_bytes(c, all_f=True)))
        return self.reports

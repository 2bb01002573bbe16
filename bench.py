#!/usr/bin/env python
"""Benchmark of the ISPA hot path on B200 (one JSON line on rank 0).

One step = one pass of the whole hot path for one Wan-1.3B-shaped layer
(12 heads x 128, 4680 chunk queries, 1560 sink + 18720 history keys, bf16):
  dual-stream attention (local + history branches, fused LSE merge)
  -> warm-up output projection y = A_full W
  -> Gram / cross-covariance accumulation G += A_loc^T A_loc, R += A_loc^T delta
  -> absorb solve dW = (G + lambda I)^-1 R W and W_new = W + dW
  -> L-layer chunk: local-only attention + projection with W_new
  -> F-layer chunk: single-pass attention over all keys + projection with W.
The headline value is the dual-stream attention throughput (algorithmic
FLOPs 4 n_q n_k d H over the kernel's CUDA-event time); absorb ms/layer and
the L-/F-layer chunk latencies are reported beside it.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]

With --gpus N > 1 (launched under torchrun) every rank runs the same layer
(replicas: the single-layer path has no data exchange), value = all ranks'
FLOPs / the slowest rank's time.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from ar_video_diffusion_b200 import synth  # noqa: E402

METRIC = "dual-stream attn TFLOP/s (% BF16 peak); absorb ms/layer; chunk latency"
WORKLOAD = "wan1.3b"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
COMP_REPS = 1  # launches of one component per timing graph


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def attn_flops(w) -> float:
    n_k = w.n_sink + w.n_q + w.n_hist
    return 4.0 * w.n_q * n_k * w.head_dim * w.n_heads


def gram_flops(w, rows) -> float:
    D = w.d_model
    return rows * D * (D + 1) + 2.0 * rows * D * D


def solve_flops(D: int) -> float:
    """Algorithmic FLOPs of one absorb solve: Cholesky D^3/3, S = R W 2 D^3 and
    the two triangular solves with D right-hand sides 2 D^3."""
    return (1.0 / 3.0 + 4.0) * float(D) ** 3


def chunk_roofline_ms(w, peak_tflops: float) -> dict:
    """Lower bound of each chunk's latency: the tensor-core time of its dense
    contractions at the peak (every step of a chunk is tensor-bound)."""
    D = w.d_model
    proj = 2.0 * w.n_q * D * D
    local = 4.0 * w.n_q * (w.n_sink + w.n_q) * w.head_dim * w.n_heads
    full = attn_flops(w)
    to_ms = lambda f: f / (peak_tflops * 1e12) * 1e3
    return {"l_layer": to_ms(local + proj), "f_layer": to_ms(full + proj),
            "warmup_f_layer": to_ms(full + proj + gram_flops(w, w.n_q))}


def max_over_ranks(times_ms, world: int, device) -> list:
    """Elementwise max over the ranks of per-rank device times (ms); every rank
    takes the same collective step, and gets the same list back."""
    t = torch.tensor([float(v) for v in times_ms], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def replica_tflops(flop_per_step: float, steps: int, world: int, t_max_ms: float) -> float:
    """Whole-job throughput of `world` replicas that each ran `steps` steps of
    `flop_per_step` FLOPs, over the slowest rank's time."""
    return world * flop_per_step * steps / (t_max_ms * 1e-3) / 1e12


def absorb_launches(D: int) -> int:
    """Kernel launches of one tensor-core absorb solve (bf16 W, D % 128 == 0):
    split of R, [0 | I] fill, S = R W, trace, shift and the first diagonal
    factorisation; per 64-wide panel its application, and for every panel but
    the last the next diagonal step (side stream) and the update
    product; the split of [L^-1 S | L^-1], dW = (L^-1)^T (L^-1 S), W_new."""
    nb = D // 64
    return 6 + nb + 2 * (nb - 1) + 3


def cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait(timeout=10)
        self.file.flush()
        self.file.seek(0)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.file.read().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.file.name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# --------------------------------------------------------------- our arm
def run_ours(args, rank, world, device):
    from ar_video_diffusion_b200 import ispa

    w = synth.WORKLOADS[WORKLOAD]
    H, d, D = w.n_heads, w.head_dim, w.d_model
    x = synth.single_layer_inputs(w, 1)
    Wh = synth.weight(w, 0)

    def t(a):
        return torch.from_numpy(a).to(torch.bfloat16).to(device)

    q, ks, vs, kc, vc, kh, vh = (t(x[k]) for k in ("q", "k_sink", "v_sink", "k_cur", "v_cur", "k_hist", "v_hist"))
    W = t(Wh)
    local = [(ks, vs), (kc, vc)]
    hist = [(kh, vh)]
    bf = dict(dtype=torch.bfloat16, device=device)
    f32 = dict(dtype=torch.float32, device=device)
    dual_out = {"a_loc": torch.empty(w.n_q, D, **bf), "a_full": torch.empty(w.n_q, D, **bf),
                "a_delta": torch.empty(w.n_q, D, **bf), "lse_loc": torch.empty(H, w.n_q, **f32),
                "lse_full": torch.empty(H, w.n_q, **f32)}
    f_out = {"a_full": torch.empty(w.n_q, D, **bf), "lse_full": torch.empty(H, w.n_q, **f32)}
    y_warm = torch.empty(w.n_q, D, **bf)
    y_l, a_l = torch.empty(w.n_q, D, **bf), torch.empty(w.n_q, D, **bf)
    y_f = torch.empty(w.n_q, D, **bf)
    G, R = torch.empty(D, D, **f32), torch.empty(D, D, **f32)
    dW, Wn = torch.empty(D, D, **f32), torch.empty(D, D, **bf)
    ws = ispa.absorb_workspace(D, device)
    status = ispa.new_status(device)
    stream = torch.cuda.current_stream(device)

    # statistics start from one chunk so the first solve already sees SPD data
    ispa.dual_attention(q, local, hist, H, out=dual_out, status=status)
    ispa.gram_accumulate(dual_out["a_loc"], dual_out["a_delta"], G, R, zero_first=True)

    comps = [
        ("dual_attention", lambda: ispa.dual_attention(q, local, hist, H, out=dual_out, status=status)),
        ("warmup_projection", lambda: ispa.project(dual_out["a_full"], W, y_warm)),
        ("gram_accumulate", lambda: ispa.gram_accumulate(dual_out["a_loc"], dual_out["a_delta"], G, R)),
        ("absorb_solve", lambda: ispa.absorb_solve(G, R, W, lambda_rel=1e-2, workspace=ws, status=status,
                                                   delta_w=dW, w_new=Wn)),
        ("local_attention_project", lambda: ispa.local_attention_project(q, local, Wn, H, y=y_l, a_loc=a_l,
                                                                         status=status)),
        ("full_attention", lambda: ispa.dual_attention(q, local, hist, H, dual=False, out=f_out, status=status)),
        ("f_projection", lambda: ispa.project(f_out["a_full"], W, y_f)),
    ]

    def step():
        for _, fn in comps:
            fn()

    # eager warm-up, then the launches of a step are captured into CUDA graphs
    # (one graph for the whole step, one per component) so that the timings
    # below hold device time only, without host launch gaps
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    side = torch.cuda.Stream(device)
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step, stream=side, capture_error_mode="relaxed"):
        step()
    # each component graph holds COMP_REPS back-to-back launches of the
    # component, so that the gap between graph launches is amortised
    g_comp = []
    for name, fn in comps:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side, capture_error_mode="relaxed"):
            for _ in range(COMP_REPS):
                fn()
        g_comp.append((name, g))
    for _ in range(args.warmup):
        g_step.replay()
    torch.cuda.synchronize(device)

    if world > 1:
        torch.distributed.barrier()
    clocks = ClockSampler(device.index if device.index is not None else 0)
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for _ in range(args.steps):
        g_step.replay()
    t_end.record(stream)
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    # per-component device time: K back-to-back replays of a graph holding
    # only that component's launches
    comp_ms = {}
    for name, g in g_comp:
        g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize(device)
        comp_ms[name] = e0.elapsed_time(e1) / (args.steps * COMP_REPS)
    clk = clocks.stop()
    code = int(status[0].item())
    if code != 0:
        raise RuntimeError(f"device status {ispa.STATUS_NAMES.get(code, code)} during the benchmark")

    total_ms = t_start.elapsed_time(t_end)
    mean = [comp_ms[n] for n, _ in comps]  # ms per component
    t_dual = comp_ms["dual_attention"] * args.steps
    # max over ranks of the time that defines `value`, and of the step time
    t_dual_max, total_max = max_over_ranks([t_dual, total_ms], world, device)
    F = attn_flops(w)
    value = replica_tflops(F, args.steps, world, t_dual_max)

    # e2e through the public API with host buffers: pinned H2D of the chunk's
    # new inputs (queries and the current chunk's K, V; the sink/history cache
    # is device-resident state), the dual attention, D2H of A_full and LSE_full.
    # A streaming caller overlaps the copies with the compute: two sets of
    # device buffers, a copy-in stream, the compute stream and a copy-out
    # stream; set b's inputs are refilled only once its previous attention has
    # consumed them, its outputs overwritten only once they have been copied out.
    hq = torch.from_numpy(x["q"]).to(torch.bfloat16).pin_memory()
    hk = torch.from_numpy(x["k_cur"]).to(torch.bfloat16).pin_memory()
    hv = torch.from_numpy(x["v_cur"]).to(torch.bfloat16).pin_memory()
    out_a = [torch.empty(w.n_q, D, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    out_l = [torch.empty(H, w.n_q, dtype=torch.float32).pin_memory() for _ in range(2)]
    dq = [torch.empty_like(q) for _ in range(2)]
    dk = [torch.empty_like(kc) for _ in range(2)]
    dv = [torch.empty_like(vc) for _ in range(2)]
    douts = [dual_out, {k2: torch.empty_like(v2) for k2, v2 in dual_out.items()}]
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = {name: [torch.cuda.Event() for _ in range(2)] for name in ("in_ready", "consumed", "copied")}
    started = [False, False]

    def e2e_step(k_step):
        b = k_step & 1
        with torch.cuda.stream(s_in):
            if started[b]:
                s_in.wait_event(ev["consumed"][b])
            dq[b].copy_(hq, non_blocking=True)
            dk[b].copy_(hk, non_blocking=True)
            dv[b].copy_(hv, non_blocking=True)
            ev["in_ready"][b].record(s_in)
        stream.wait_event(ev["in_ready"][b])
        if started[b]:
            stream.wait_event(ev["copied"][b])
        ispa.dual_attention(dq[b], [(ks, vs), (dk[b], dv[b])], hist, H, out=douts[b], status=status, stream=stream)
        ev["consumed"][b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["consumed"][b])
            out_a[b].copy_(douts[b]["a_full"], non_blocking=True)
            out_l[b].copy_(douts[b]["lse_full"], non_blocking=True)
            ev["copied"][b].record(s_out)
        started[b] = True

    def e2e_join():
        for b in range(2):
            if started[b]:
                stream.wait_event(ev["copied"][b])

    for i in range(2):
        e2e_step(i)
    e2e_join()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)  # nothing of the timed steps starts before e0
    for i in range(args.steps):
        e2e_step(i)
    e2e_join()
    e1.record(stream)
    torch.cuda.synchronize(device)
    (e2e_ms,) = max_over_ranks([e0.elapsed_time(e1)], world, device)
    e2e_value = replica_tflops(F, args.steps, world, e2e_ms)
    h2d = (hq.numel() + hk.numel() + hv.numel()) * 2
    d2h = out_a[0].numel() * 2 + out_l[0].numel() * 4

    # standalone LSE merge over rotating buffer sets larger than L2
    merge_gbs = merge_bench(ispa, w, device)
    long_hist = long_history_bench(ispa, device)
    pk0, _ = peaks()
    w8a8 = w8a8_bench(ispa, w, device, pk0["bf16_tflops"], pk0["hbm_gbs"])

    configs = configs_bench(ispa, device, pk0["bf16_tflops"], pk0["hbm_gbs"])
    rollout = None if args.no_rollout else _section(run_rollout, device)
    rollout_12warm = None if args.no_rollout else _section(run_rollout_12warm, device)

    pk, src = peaks()
    tc_peak = pk["bf16_tflops"]
    achieved = F / (t_dual / args.steps * 1e-3) / 1e12
    traffic = load_traffic("attention_kernel<128,3>")
    res = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_max / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded PCG64; Wan-1.3B latent shapes; random-init W)",
        "config": {"workload": "wan1.3b single layer: 12 heads x 128, 4680 chunk queries, 1560 sink + 4680 "
                               "current + 18720 history keys; warm-up statistics over one chunk per step; "
                               "absorb D=1536",
                   "l2": "inputs larger than L2 (153 MB of K/V read per attention pass)",
                   "timing": "CUDA-graph replays: a step graph for ms_per_step, one graph per component for the "
                             "breakdown and the value",
                   "parallelism": f"replicas x{world}"},
        "absorb_ms_per_layer": round(float(mean[3]), 4),
        "absorb_tflops": round(solve_flops(D) / (mean[3] * 1e-3) / 1e12, 3),
        "chunk_latency_roofline_frac": {k: round(v / lat, 4) for (k, v), lat in zip(
            chunk_roofline_ms(w, tc_peak).items(), (mean[4], mean[5] + mean[6], mean[0] + mean[1] + mean[2]))},
        "chunk_latency_ms": {"l_layer": round(float(mean[4]), 4),
                             "f_layer": round(float(mean[5] + mean[6]), 4),
                             "warmup_f_layer": round(float(mean[0] + mean[1] + mean[2]), 4)},
        "components_ms": {"dual_attention": round(float(mean[0]), 4), "warmup_projection": round(float(mean[1]), 4),
                          "gram_accumulate": round(float(mean[2]), 4), "absorb_solve": round(float(mean[3]), 4),
                          "local_attention_project": round(float(mean[4]), 4),
                          "full_attention": round(float(mean[5]), 4), "f_projection": round(float(mean[6]), 4)},
        "components_rate": {
            "dual_attention_tflops": round(achieved, 2),
            "full_attention_tflops": round(F / (mean[5] * 1e-3) / 1e12, 2),
            "gram_tflops": round(gram_flops(w, w.n_q) / (mean[2] * 1e-3) / 1e12, 2),
            "projection_tflops": round(2.0 * w.n_q * D * D / (mean[1] * 1e-3) / 1e12, 2),
            "lse_merge_gbs": round(merge_gbs, 1)},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": tc_peak, "unit": "TFLOP/s",
                     "frac": round(achieved / tc_peak, 4), "traffic": traffic,
                     "kernel": "attn2::attention_kernel<128,3>", "peak_source": f"{src} bf16 burst",
                     "frac_of_spec_2250": round(achieved / 2250.0, 4)},
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "clocks": clk,
        "gpu_launches": args.steps * (7 + absorb_launches(D)) * (1 + COMP_REPS),
        "long_history": long_hist,
        "configs": configs,
        "w8a8": w8a8,
        "rollout": rollout,
        "rollout_12warm": rollout_12warm,
    }
    return res


def run_profile_case(op: str, reps: int, device):
    """One op of the hot path on the wan1.3b shapes, `reps` times back to back."""
    from ar_video_diffusion_b200 import ispa
    w = synth.WORKLOADS[WORKLOAD]
    H, D, n = w.n_heads, w.d_model, w.n_q
    x = synth.single_layer_inputs(w, 1)

    def t(a):
        return torch.from_numpy(a).to(torch.bfloat16).to(device)

    q, ks, vs, kc, vc, kh, vh = (t(x[k]) for k in ("q", "k_sink", "v_sink", "k_cur", "v_cur", "k_hist", "v_hist"))
    W = t(synth.weight(w, 0))
    local, hist = [(ks, vs), (kc, vc)], [(kh, vh)]
    status = ispa.new_status(device)
    # set-up launches are issued only for the ops that need them, so that an
    # ncu capture with "-s 1" skips exactly the first launch of the loop below
    out = G = R = o_hist = None
    if op in ("gram", "absorb", "project", "merge"):
        out = ispa.dual_attention(q, local, hist, H, status=status)
    if op in ("gram", "absorb"):
        G, R = torch.empty(D, D, device=device), torch.empty(D, D, device=device)
        ispa.gram_accumulate(out["a_loc"], out["a_delta"], G, R, zero_first=True)
    if op == "merge":
        o_hist = ispa.dual_attention(q, [], hist, H, dual=False, status=status)
    if op in ("project_w8a8", "quantize_rows", "project_mx", "local_mx"):
        a16 = ispa.dual_attention(q, local, hist, H, status=status)["a_loc"]
        qwt, sw = ispa.quantize_e4m3_weight(W)
        qa, sa = ispa.quantize_e4m3_rows(a16)
        mq, me = ispa.mx_quantize_e4m3_rows(a16)
    if op == "layer_error":
        out = ispa.dual_attention(q, local, hist, H, status=status)
        G, R, E = (torch.empty(D, D, device=device) for _ in range(3))
        ispa.gram_accumulate(out["a_loc"], out["a_delta"], G, R, zero_first=True)
        ispa.sym_gram_accumulate(out["a_delta"], E, zero_first=True)
        dW, _ = ispa.absorb_solve(G, R, W, status=status)
        ws = torch.empty(ispa.ispa_layer_error_workspace_bytes(D), dtype=torch.uint8, device=device)
    if op == "dual":
        out = {"a_loc": torch.empty(n, D, dtype=torch.bfloat16, device=device),
               "a_full": torch.empty(n, D, dtype=torch.bfloat16, device=device),
               "a_delta": torch.empty(n, D, dtype=torch.bfloat16, device=device),
               "lse_loc": torch.empty(H, n, device=device), "lse_full": torch.empty(H, n, device=device)}
    torch.cuda.synchronize(device)
    for _ in range(reps):
        if op == "dual":
            ispa.dual_attention(q, local, hist, H, out=out, status=status)
        elif op == "full":
            ispa.dual_attention(q, local, hist, H, dual=False, status=status)
        elif op == "local":
            ispa.local_attention_project(q, local, W, H, status=status)
        elif op == "gram":
            ispa.gram_accumulate(out["a_loc"], out["a_delta"], G, R)
        elif op == "project":
            ispa.project(out["a_full"], W)
        elif op == "merge":
            ispa.lse_merge(out["a_loc"], out["lse_loc"], o_hist["a_full"], o_hist["lse_full"], H)
        elif op == "absorb":
            ispa.absorb_solve(G, R, W, status=status)
        elif op == "project_w8a8":
            ispa.project_w8a8(qa, sa, qwt, sw)
        elif op == "quantize_rows":
            ispa.quantize_e4m3_rows(a16, qa, sa)
        elif op == "project_mx":
            ispa.project_mx(mq, me, qwt, sw)
        elif op == "local_mx":
            ispa.local_attention_project_mx(q, local, qwt, sw, H, status=status)
        elif op == "layer_error":
            ispa.layer_error(G, R, E, W, dW, workspace=ws)
    torch.cuda.synchronize(device)
    if int(status[0].item()) != 0:
        raise RuntimeError(f"device status {int(status[0].item())}")
    print(f"profile case {op} x{reps} done")


def _section(fn, *args) -> dict:
    """A supplementary section of the JSON line (the rollouts): a device
    error inside it (a bounded wait that gave up, reported through the status
    word) is recorded in the line instead of ending the run, since the
    headline measurement does not depend on it."""
    from ar_video_diffusion_b200 import ispa
    try:
        return fn(*args)
    except ispa.IspaError as e:
        torch.cuda.synchronize()
        return {"error": str(e)}


def run_rollout(device) -> dict:
    """30-layer streaming rollout, 1.3B shapes: 4 warm-up chunks with every
    layer dual-stream (the even layers accumulating statistics), absorb +
    eviction of the 15 even layers, then 20 chunks with L-/F-layers."""
    from ar_video_diffusion_b200.rollout import Rollout
    w = synth.WORKLOADS["rollout"]
    ro = Rollout(w, device=device)
    reps = ro.run()
    post = [r for r in reps if r.phase == "post"]
    warm = [r for r in reps if r.phase == "warmup"]
    last = reps[-1]
    flops_last = 0.0
    F_tok = w.frame_tokens
    n_k_f = (last.chunk + 1) * w.n_q
    for l in range(w.n_layers):
        n_k = (w.sink_frames * F_tok + w.n_q) if l in ro.absorbed else n_k_f
        flops_last += 4.0 * w.n_q * n_k * w.head_dim * w.n_heads + 2.0 * w.n_q * w.d_model ** 2
    # the first and the last post-transition chunk again, each as one CUDA graph
    g_first = ro.chunk_graph_ms(w.warm_chunks)
    g_last = ro.chunk_graph_ms(last.chunk)
    if int(ro.status[0].item()) != 0:
        raise RuntimeError("device status during the chunk graphs")
    res = {
        "workload": "rollout: 30 layers, 1.3B shapes, 4 warm-up + 20 post-transition chunks, even layers absorbed",
        "chunk_ms": [round(r.gpu_ms, 3) for r in reps],
        "warmup_chunk_ms_mean": round(sum(r.gpu_ms for r in warm) / len(warm), 3),
        "post_chunk_ms_first": round(post[0].gpu_ms, 3),
        "post_chunk_ms_last": round(post[-1].gpu_ms, 3),
        "post_chunk_graph_ms_first": round(g_first, 3),
        "post_chunk_graph_ms_last": round(g_last, 3),
        "post_chunk_graph_tflops_last": round(flops_last / (g_last * 1e-3) / 1e12, 1),
        "post_chunk_graph_roofline_frac_last": round(flops_last / (peaks()[0]["bf16_tflops"] * 1e12) * 1e3 / g_last, 4),
        "last_chunk_tflops": round(flops_last / (last.gpu_ms * 1e-3) / 1e12, 1),
        "absorb_ms_per_layer": round(sum(ro.absorb_ms) / len(ro.absorb_ms), 4),
        "kv_bytes_last": last.kv_bytes,
        "kv_bytes_all_f_last": last.kv_bytes_all_f,
        "kv_removed_frac": round(1 - last.kv_bytes / last.kv_bytes_all_f, 4),
    }
    del ro
    torch.cuda.empty_cache()
    res["w8a8"] = _section(run_rollout_w8a8, device, res, "w8a8")
    res["mx"] = _section(run_rollout_w8a8, device, res, "mx")
    res["layer_selection"] = _section(run_layer_selection, device)
    return res


def run_rollout_w8a8(device, bf16_res: dict, precision: str) -> dict:
    """The same rollout with W8A8 L-layers (W_new quantised to e4m3 once after
    the absorb; A_loc per token every chunk, or with precision "mx" as MX
    codes from the attention epilogue), post-transition chunks timed the same
    way as the bf16 rollout's."""
    from ar_video_diffusion_b200.rollout import Rollout
    w = synth.WORKLOADS["rollout"]
    ro = Rollout(w, device=device, precision=precision)
    reps = ro.run()
    post = [r for r in reps if r.phase == "post"]
    g_first = ro.chunk_graph_ms(w.warm_chunks)
    g_last = ro.chunk_graph_ms(reps[-1].chunk)
    if int(ro.status[0].item()) != 0:
        raise RuntimeError("device status during the W8A8 rollout")
    del ro
    torch.cuda.empty_cache()
    form = "A_loc per token" if precision == "w8a8" else "A_loc as MX codes written by the attention epilogue"
    return {"workload": f"the rollout above with W8A8 L-layers (e4m3 W_new per output channel, {form})",
            "post_chunk_ms_first": round(post[0].gpu_ms, 3), "post_chunk_ms_last": round(post[-1].gpu_ms, 3),
            "post_chunk_graph_ms_first": round(g_first, 3), "post_chunk_graph_ms_last": round(g_last, 3),
            "speedup_vs_bf16_graph_first": round(bf16_res["post_chunk_graph_ms_first"] / g_first, 4),
            "speedup_vs_bf16_graph_last": round(bf16_res["post_chunk_graph_ms_last"] / g_last, 4)}


def run_layer_selection(device) -> dict:
    """The same 30 layers through the warm-up with every layer accumulating
    G, R and E, then the instance-specific choice of K = 15 layers by
    reconstruction error (all 30 absorbed and ranked), against the fixed
    even-layer set on the same errors."""
    import dataclasses
    from ar_video_diffusion_b200 import ispa
    from ar_video_diffusion_b200.rollout import Rollout
    w = dataclasses.replace(synth.WORKLOADS["rollout"], post_chunks=0)
    ro = Rollout(w, device=device, selection="instance")
    ro.run()
    ro.transition()
    even = list(range(0, w.n_layers, 2))
    eps = ro.eps
    res = {
        "workload": "30 layers, 1.3B shapes, 4 warm-up chunks; K = 15 of 30 chosen by reconstruction error",
        "selected": ro.absorbed,
        "eps": [round(e, 6) for e in eps],
        "eps_sum_selected": round(sum(eps[l] for l in ro.absorbed), 6),
        "eps_sum_even_layers": round(sum(eps[l] for l in even), 6),
        "rank_ms_all_layers": round(ro.select_ms, 3),
        "rank_ms_per_layer": round(ro.select_ms / w.n_layers, 4),
    }
    assert ro.absorbed == ispa.select_layers(eps, len(even))
    del ro
    torch.cuda.empty_cache()
    return res


def _frames_device(w, layer: int, frames, device):
    """K, V of the listed latent frames from the seeded device generator."""
    F, D = w.frame_tokens, w.d_model
    k = torch.empty(len(frames) * F, D, dtype=torch.bfloat16, device=device)
    v = torch.empty_like(k)
    for i, f in enumerate(frames):
        kf, vf = synth.frame_kv_device(w, 0, f, device)
        k[i * F:(i + 1) * F].copy_(kf)
        v[i * F:(i + 1) * F].copy_(vf)
    return k, v


def _single_layer_device(w, device):
    """One warm-up chunk of a single-layer workload on the device: Q and the
    sink / history / current K, V (device generator, the host recipe's shapes)."""
    fr = synth.single_layer_frames(w, 1)
    ks, vs = _frames_device(w, 0, fr["sink"], device)
    kh, vh = _frames_device(w, 0, fr["hist"], device)
    kc, vc = _frames_device(w, 0, fr["cur"], device)
    q = synth.chunk_q_device(w, 0, 1, device)
    return q, [(ks, vs), (kc, vc)], [(kh, vh)]


def _rows_like(src: torch.Tensor, n_rows: int) -> torch.Tensor:
    """n_rows rows made of repeats of src's rows (statistics inputs of the
    workload's size; the values do not change the work)."""
    reps = (n_rows + src.shape[0] - 1) // src.shape[0]
    return src.repeat(reps, 1)[:n_rows].contiguous()


def configs_bench(ispa, device, peak_bf16: float, peak_hbm: float, iters=10) -> dict:
    """The other benchmark configurations, each timed as CUDA-graph replays:
    tiny fp32 (latency of every step), long history (93600 history tokens:
    dual attention, LSE merge and a 93600-row statistics accumulation) and
    Wan-14B shapes (dual attention, 18720-row statistics, 5120 x 5120 absorb)."""
    res = {}
    status = ispa.new_status(device)

    # ---- tiny fp32: 2 heads x 64, 64 queries, 16 sink + 64 current + 256 history keys, D = 128
    w = synth.WORKLOADS["tiny_f32"]
    H, D = w.n_heads, w.d_model
    x = synth.single_layer_inputs(w, 1)
    t32 = {k: torch.from_numpy(v).to(device) for k, v in x.items()}
    loc = [(t32["k_sink"], t32["v_sink"]), (t32["k_cur"], t32["v_cur"])]
    his = [(t32["k_hist"], t32["v_hist"])]
    out = ispa.dual_attention(t32["q"], loc, his, H, status=status)
    oh = ispa.dual_attention(t32["q"], [], his, H, dual=False, status=status)
    a_rows = _rows_like(out["a_loc"], w.warm_chunks * w.n_q)
    d_rows = _rows_like(out["a_delta"], w.warm_chunks * w.n_q)
    G, R = torch.empty(D, D, device=device), torch.empty(D, D, device=device)
    ispa.gram_accumulate(a_rows, d_rows, G, R, zero_first=True)
    W = torch.from_numpy(synth.weight(w, 0)).to(device)
    ws = ispa.absorb_workspace(D, device)
    dW, Wn = torch.empty(D, D, device=device), torch.empty_like(W)
    mo = {"a_full": torch.empty_like(out["a_loc"]), "a_delta": torch.empty_like(out["a_loc"]),
          "lse_full": torch.empty_like(out["lse_loc"])}
    ms = {
        "dual_attention": _graph_ms(lambda: ispa.dual_attention(t32["q"], loc, his, H, out=out, status=status),
                                    device, iters),
        "lse_merge": _graph_ms(lambda: ispa.lse_merge(out["a_loc"], out["lse_loc"], oh["a_full"], oh["lse_full"], H,
                                                      out=mo), device, iters),
        "gram_256_rows": _graph_ms(lambda: ispa.gram_accumulate(a_rows, d_rows, G, R, zero_first=True), device, iters),
        "absorb_solve": _graph_ms(lambda: ispa.absorb_solve(G, R, W, workspace=ws, status=status, delta_w=dW,
                                                            w_new=Wn), device, iters),
    }
    res["tiny_f32"] = {"workload": "tiny fp32: 2 heads x 64, 64 queries, 16 sink + 64 current + 256 history keys, "
                                   "256 statistics rows, D = 128 (latency only; fp32 on the CUDA cores)",
                       "ms": {k: round(v, 4) for k, v in ms.items()},
                       "step_ms": round(sum(ms.values()), 4)}

    # ---- long history: wan1.3b shapes, 93600 history tokens, 93600-row statistics
    w = synth.WORKLOADS["long_hist"]
    H, D = w.n_heads, w.d_model
    q, loc, his = _single_layer_device(w, device)
    out = ispa.dual_attention(q, loc, his, H, status=status)
    oh = ispa.dual_attention(q, [], his, H, dual=False, status=status)
    n_rows = w.warm_chunks * w.n_q
    a_rows, d_rows = _rows_like(out["a_loc"], n_rows), _rows_like(out["a_delta"], n_rows)
    G, R = torch.empty(D, D, device=device), torch.empty(D, D, device=device)
    t_dual = _graph_ms(lambda: ispa.dual_attention(q, loc, his, H, out=out, status=status), device, iters)
    mo = {"a_full": torch.empty_like(out["a_loc"]), "a_delta": torch.empty_like(out["a_loc"]),
          "lse_full": torch.empty_like(out["lse_loc"])}
    t_merge = _graph_ms(lambda: ispa.lse_merge(out["a_loc"], out["lse_loc"], oh["a_full"], oh["lse_full"], H, out=mo),
                        device, iters)
    t_gram = _graph_ms(lambda: ispa.gram_accumulate(a_rows, d_rows, G, R, zero_first=True), device, iters)
    F_attn = attn_flops(w)
    merge_bytes = w.n_q * D * 2 * 4 + H * w.n_q * 4 * 3
    res["long_hist"] = {
        "workload": "long history: wan1.3b shapes, 1560 sink + 4680 current + 93600 history keys; statistics over "
                    "93600 rows",
        "dual_attention_ms": round(t_dual, 4),
        "dual_attention_tflops": round(F_attn / (t_dual * 1e-3) / 1e12, 1),
        "dual_attention_frac": round(F_attn / (t_dual * 1e-3) / 1e12 / peak_bf16, 4),
        "lse_merge_ms": round(t_merge, 4),
        "lse_merge_gbs": round(merge_bytes / (t_merge * 1e-3) / 1e9, 1),
        "lse_merge_frac": round(merge_bytes / (t_merge * 1e-3) / 1e9 / peak_hbm, 4),
        "lse_merge_note": "one launch, inputs partly L2-resident (58.2 MB < 126 MB L2)",
        "gram_93600_rows_ms": round(t_gram, 4),
        "gram_tflops": round(gram_flops(w, n_rows) / (t_gram * 1e-3) / 1e12, 1),
        "gram_frac": round(gram_flops(w, n_rows) / (t_gram * 1e-3) / 1e12 / peak_bf16, 4),
    }
    del q, loc, his, out, oh, mo, a_rows, d_rows, G, R
    torch.cuda.empty_cache()

    # ---- Wan-14B shapes: 40 heads x 128 (D = 5120), 18720 history keys, 18720-row statistics, 5120^2 absorb
    w = synth.WORKLOADS["wan14b"]
    H, D = w.n_heads, w.d_model
    q, loc, his = _single_layer_device(w, device)
    out = ispa.dual_attention(q, loc, his, H, status=status)
    n_rows = w.warm_chunks * w.n_q
    a_rows, d_rows = _rows_like(out["a_loc"], n_rows), _rows_like(out["a_delta"], n_rows)
    G, R = torch.empty(D, D, device=device), torch.empty(D, D, device=device)
    ispa.gram_accumulate(a_rows, d_rows, G, R, zero_first=True)
    W = synth.weight_device(w, 0, device)
    ws = ispa.absorb_workspace(D, device)
    dW, Wn = torch.empty(D, D, device=device), torch.empty_like(W)
    t_dual = _graph_ms(lambda: ispa.dual_attention(q, loc, his, H, out=out, status=status), device, iters)
    t_gram = _graph_ms(lambda: ispa.gram_accumulate(a_rows, d_rows, G, R, zero_first=True), device, iters)
    t_abs = _graph_ms(lambda: ispa.absorb_solve(G, R, W, workspace=ws, status=status, delta_w=dW, w_new=Wn),
                      device, 3)
    F_attn = attn_flops(w)
    res["wan14b"] = {
        "workload": "wan14b: 40 heads x 128 (D = 5120), 4680 queries, 1560 sink + 4680 current + 18720 history "
                    "keys; statistics over 18720 rows; absorb on 5120 x 5120",
        "dual_attention_ms": round(t_dual, 4),
        "dual_attention_tflops": round(F_attn / (t_dual * 1e-3) / 1e12, 1),
        "dual_attention_frac": round(F_attn / (t_dual * 1e-3) / 1e12 / peak_bf16, 4),
        "gram_18720_rows_ms": round(t_gram, 4),
        "gram_tflops": round(gram_flops(w, n_rows) / (t_gram * 1e-3) / 1e12, 1),
        "gram_frac": round(gram_flops(w, n_rows) / (t_gram * 1e-3) / 1e12 / peak_bf16, 4),
        "absorb_ms_per_layer": round(t_abs, 3),
        "absorb_tflops": round(solve_flops(D) / (t_abs * 1e-3) / 1e12, 2),
        "absorb_frac": round(solve_flops(D) / (t_abs * 1e-3) / 1e12 / peak_bf16, 4),
    }
    torch.cuda.synchronize(device)
    if int(status[0].item()) != 0:
        raise RuntimeError("device status during the configuration benchmarks")
    del q, loc, his, out, a_rows, d_rows, G, R, W, ws, dW, Wn
    torch.cuda.empty_cache()
    return res


def run_rollout_12warm(device) -> dict:
    """The secondary reading of the rollout's warm-up: 12 warm-up chunks
    (36 latent frames, 56160 statistics rows per absorbed layer) instead of
    T_warm = 12 latent frames, then the same 20 chunks."""
    from ar_video_diffusion_b200.rollout import Rollout
    import dataclasses
    w = dataclasses.replace(synth.WORKLOADS["rollout"], warm_chunks=12)
    ro = Rollout(w, device=device)
    reps = ro.run()
    post = [r for r in reps if r.phase == "post"]
    warm = [r for r in reps if r.phase == "warmup"]
    last = reps[-1]
    res = {
        "workload": "rollout, secondary warm-up reading: 30 layers, 1.3B shapes, 12 warm-up chunks (56160 rows) + "
                    "20 post-transition chunks, even layers absorbed",
        "chunk_ms": [round(r.gpu_ms, 3) for r in reps],
        "warmup_chunk_ms_mean": round(sum(r.gpu_ms for r in warm) / len(warm), 3),
        "post_chunk_ms_first": round(post[0].gpu_ms, 3),
        "post_chunk_ms_last": round(post[-1].gpu_ms, 3),
        "absorb_ms_per_layer": round(sum(ro.absorb_ms) / len(ro.absorb_ms), 4),
        "kv_bytes_last": last.kv_bytes,
        "kv_bytes_all_f_last": last.kv_bytes_all_f,
        "kv_removed_frac": round(1 - last.kv_bytes / last.kv_bytes_all_f, 4),
    }
    del ro
    torch.cuda.empty_cache()
    return res


def long_history_bench(ispa, device, iters=5) -> dict:
    """A long-lived F-layer: the dual-stream and the single-pass attention of
    one 4680-query chunk over 129 latent frames (201240 tokens) of history,
    K/V drawn by the device generator, timed as CUDA-graph replays."""
    w = synth.WORKLOADS["hist_200k"]
    F, D, H = w.frame_tokens, w.d_model, w.n_heads
    n_frames = w.sink_frames + w.hist_frames + w.chunk_frames
    k = torch.empty(n_frames * F, D, dtype=torch.bfloat16, device=device)
    v = torch.empty_like(k)
    for f in range(n_frames):
        kf, vf = synth.frame_kv_device(w, 0, f, device)
        k[f * F:(f + 1) * F].copy_(kf)
        v[f * F:(f + 1) * F].copy_(vf)
    q = synth.chunk_q_device(w, 0, 1, device)
    s, h = w.n_sink, w.n_sink + w.n_hist
    local = [(k[:s], v[:s]), (k[h:], v[h:])]
    hist = [(k[s:h], v[s:h])]
    status = ispa.new_status(device)
    out = ispa.dual_attention(q, local, hist, H, status=status)
    fout = ispa.dual_attention(q, local, hist, H, dual=False, status=status)
    res = {"n_hist": w.n_hist, "n_keys": w.n_sink + w.n_hist + w.n_q}
    side = torch.cuda.Stream(device)
    stream = torch.cuda.current_stream(device)
    for name, fn in (("dual", lambda: ispa.dual_attention(q, local, hist, H, out=out, status=status)),
                     ("full", lambda: ispa.dual_attention(q, local, hist, H, dual=False, out=fout, status=status))):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side, capture_error_mode="relaxed"):
            fn()
        g.replay()
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(iters):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize(device)
        ms = e0.elapsed_time(e1) / iters
        res[name + "_ms"] = round(ms, 4)
        res[name + "_tflops"] = round(attn_flops(w) / (ms * 1e-3) / 1e12, 1)
    if int(status[0].item()) != 0:
        raise RuntimeError("device status during the long-history benchmark")
    del k, v
    torch.cuda.empty_cache()
    return res


def _graph_ms(fn, device, iters) -> float:
    """Device time of fn's launches: captured COMP_REPS times back to back
    into one graph, replayed iters times, per call of fn."""
    side = torch.cuda.Stream(device)
    stream = torch.cuda.current_stream(device)
    fn()
    torch.cuda.synchronize(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side, capture_error_mode="relaxed"):
        for _ in range(COMP_REPS):
            fn()
    g.replay()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(iters):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize(device)
    return e0.elapsed_time(e1) / (iters * COMP_REPS)


def _graph_ms_flushed(fn, device, iters) -> float:
    """Device time of one call of fn, captured once into a graph; before each
    of the iters replays a 256 MB buffer is written, so no operand is left in
    the 126 MB L2 by the previous replay.  Mean over the replays."""
    side = torch.cuda.Stream(device)
    stream = torch.cuda.current_stream(device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    fn()
    torch.cuda.synchronize(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side, capture_error_mode="relaxed"):
        fn()
    g.replay()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
    for e0, e1 in ev:
        flush.zero_()
        e0.record(stream)
        g.replay()
        e1.record(stream)
    torch.cuda.synchronize(device)
    return sum(e0.elapsed_time(e1) for e0, e1 in ev) / iters


def w8a8_bench(ispa, w, device, peak_bf16: float, peak_hbm: float, iters=20) -> dict:
    """The W8A8 variants of the post-transition L-layer against the bf16
    L-layer on the same inputs: per-token (attention -> bf16 A_loc -> e4m3
    codes -> e4m3 product) and MX (the attention epilogue writes e4m3 codes
    with a power-of-two scale per 32 channels -> block-scaled product).  The
    L-layers are timed with L2 flushed before every replay (their inputs,
    52.8 MB, fit in L2); the single kernels as back-to-back graph replays.
    The fp8 peak is the measured bf16 peak times the nominal fp8 / bf16 ratio
    of 2."""
    H, D, n = w.n_heads, w.d_model, w.n_q
    x = synth.single_layer_inputs(w, 1)

    def t(a):
        return torch.from_numpy(a).to(torch.bfloat16).to(device)

    q = t(x["q"])
    local = [(t(x["k_sink"]), t(x["v_sink"])), (t(x["k_cur"]), t(x["v_cur"]))]
    W = t(synth.weight(w, 0))
    status = ispa.new_status(device)
    y16, a16 = torch.empty(n, D, dtype=torch.bfloat16, device=device), torch.empty(n, D, dtype=torch.bfloat16,
                                                                                  device=device)
    qwt, sw = ispa.quantize_e4m3_weight(W)
    out8 = ispa.local_attention_project_w8a8(q, local, qwt, sw, H, status=status)
    ispa.local_attention_project(q, local, W, H, y=y16, a_loc=a16, status=status)
    qa, sa = ispa.quantize_e4m3_rows(a16)
    outmx = ispa.local_attention_project_mx(q, local, qwt, sw, H, status=status)
    mq, me = ispa.mx_quantize_e4m3_rows(a16)
    yp = torch.empty(n, D, dtype=torch.bfloat16, device=device)
    ms = {
        "l_layer_w8a8": _graph_ms_flushed(lambda: ispa.local_attention_project_w8a8(q, local, qwt, sw, H, out=out8,
                                                                                    status=status), device, iters),
        "l_layer_mx": _graph_ms_flushed(lambda: ispa.local_attention_project_mx(q, local, qwt, sw, H, out=outmx,
                                                                                status=status), device, iters),
        "l_layer_bf16": _graph_ms_flushed(lambda: ispa.local_attention_project(q, local, W, H, y=y16, a_loc=a16,
                                                                               status=status), device, iters),
        "project_mx": _graph_ms(lambda: ispa.project_mx(mq, me, qwt, sw, yp), device, iters),
        "mx_quantize_rows": _graph_ms(lambda: ispa.mx_quantize_e4m3_rows(a16, mq, me), device, iters),
        "project_w8a8": _graph_ms(lambda: ispa.project_w8a8(qa, sa, qwt, sw, yp), device, iters),
        "project_bf16": _graph_ms(lambda: ispa.project(a16, W, yp), device, iters),
        "quantize_rows": _graph_ms(lambda: ispa.quantize_e4m3_rows(a16, qa, sa), device, iters),
        "quantize_weight": _graph_ms(lambda: ispa.quantize_e4m3_weight(W, qwt, sw), device, iters),
    }
    torch.cuda.synchronize(device)
    if int(status[0].item()) != 0:
        raise RuntimeError("device status during the W8A8 benchmark")
    flops = 2.0 * n * D * D
    pk8 = 2.0 * peak_bf16
    q_bytes = n * D * 2 + n * D + n * 4
    diff = (out8["y"].float() - y16.float()).norm() / y16.float().norm()
    diff_mx = (outmx["y"].float() - y16.float()).norm() / y16.float().norm()
    return {
        "workload": "wan1.3b L-layer: local attention (4680 queries, 6240 keys) + y = A_loc W_new, "
                    "W8A8 = e4m3 codes; W_new per output channel, A_loc per token or (MX) per 32 channels",
        "timing": "l_layer_*: L2 flushed before each replay; single kernels: back-to-back graph replays",
        "ms": {k: round(v, 4) for k, v in ms.items()},
        "project_w8a8_tflops": round(flops / (ms["project_w8a8"] * 1e-3) / 1e12, 1),
        "project_w8a8_frac_of_fp8_peak": round(flops / (ms["project_w8a8"] * 1e-3) / 1e12 / pk8, 4),
        "project_mx_tflops": round(flops / (ms["project_mx"] * 1e-3) / 1e12, 1),
        "project_mx_frac_of_fp8_peak": round(flops / (ms["project_mx"] * 1e-3) / 1e12 / pk8, 4),
        "l_layer_mx_speedup_vs_bf16": round(ms["l_layer_bf16"] / ms["l_layer_mx"], 4),
        "y_rel_diff_mx_vs_bf16": round(float(diff_mx), 5),
        "fp8_peak_tflops": round(pk8, 1),
        "quantize_rows_gbs": round(q_bytes / (ms["quantize_rows"] * 1e-3) / 1e9, 1),
        "quantize_rows_frac_of_hbm": round(q_bytes / (ms["quantize_rows"] * 1e-3) / 1e9 / peak_hbm, 4),
        "l_layer_speedup_vs_bf16": round(ms["l_layer_bf16"] / ms["l_layer_w8a8"], 4),
        "y_rel_diff_vs_bf16": round(float(diff), 5),
    }


def merge_bench(ispa, w, device, sets=4, iters=20) -> float:
    H, D, n = w.n_heads, w.d_model, w.n_q
    g = torch.Generator(device=device).manual_seed(0)
    bufs = []
    for _ in range(sets):
        bufs.append({"o_loc": torch.randn(n, D, device=device, generator=g).to(torch.bfloat16),
                     "o_hist": torch.randn(n, D, device=device, generator=g).to(torch.bfloat16),
                     "l_loc": torch.randn(H, n, device=device, generator=g),
                     "l_hist": torch.randn(H, n, device=device, generator=g),
                     "out": {"a_full": torch.empty(n, D, dtype=torch.bfloat16, device=device),
                             "a_delta": torch.empty(n, D, dtype=torch.bfloat16, device=device),
                             "lse_full": torch.empty(H, n, device=device)}})
    for b in bufs:
        ispa.lse_merge(b["o_loc"], b["l_loc"], b["o_hist"], b["l_hist"], H, out=b["out"])
    torch.cuda.synchronize(device)
    # back-to-back launches over rotating buffer sets (232 MB > L2), replayed
    # from a CUDA graph so that the timing holds device time only
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=torch.cuda.Stream(device), capture_error_mode="relaxed"):
        for i in range(iters):
            b = bufs[i % sets]
            ispa.lse_merge(b["o_loc"], b["l_loc"], b["o_hist"], b["l_hist"], H, out=b["out"])
    g.replay()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize(device)
    nbytes = n * D * 2 * 4 + H * n * 4 * 3
    return nbytes * iters / (e0.elapsed_time(e1) * 1e-3) / 1e9


def load_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from profiles/traffic.md, or None when
    the kernel's source has changed since that capture."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.md")
    if not os.path.exists(p):
        return None
    for line in open(p):
        cells = [c.strip() for c in line.strip().strip("|").split("|")]
        if len(cells) != 4 or cells[0] != kernel:
            continue
        src = os.path.join(ROOT, cells[1])
        if not os.path.exists(src):
            return None
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        return int(cells[3]) if digest == cells[2] else None
    return None


# --------------------------------------------------------- CPU baseline
def oracle_sample(rows: int):
    """fp64 oracle dual-stream pass over `rows` query rows of the workload."""
    from oracle import ispa_oracle as orc
    w = synth.WORKLOADS[WORKLOAD]
    x = synth.single_layer_inputs(w, 1)
    loc = [(x["k_sink"], x["v_sink"]), (x["k_cur"], x["v_cur"])]
    his = [(x["k_hist"], x["v_hist"])]
    flops = attn_flops(w) * rows / w.n_q

    def run():
        orc.dual_stream(x["q"][:rows], loc, his, w.n_heads)
    return run, flops


def blas_info() -> dict:
    """BLAS library numpy uses and its thread count."""
    try:
        import threadpoolctl
        info = [i for i in threadpoolctl.threadpool_info() if i.get("user_api") == "blas"]
        if info:
            return {"vendor": f"{info[0].get('internal_api')} {info[0].get('version')}",
                    "threads": info[0].get("num_threads")}
    except Exception:  # noqa: BLE001 - reporting only
        pass
    return {"vendor": "unknown", "threads": None}


def oracle_tiny_step():
    """The oracle's whole hot path on the tiny fp32 workload: four warm-up
    chunks of the dual stream, their statistics, the absorb and an L-layer."""
    from oracle import ispa_oracle as orc
    w = synth.WORKLOADS["tiny_f32"]
    xs = [synth.single_layer_inputs(w, c) for c in range(w.warm_chunks)]
    W = synth.weight(w, 0)

    def run():
        a, d = [], []
        for x in xs:
            r = orc.dual_stream(x["q"], [(x["k_sink"], x["v_sink"]), (x["k_cur"], x["v_cur"])],
                                [(x["k_hist"], x["v_hist"])], w.n_heads)
            a.append(r["a_loc"])
            d.append(r["delta"])
        G, R = orc.gram(np.concatenate(a), np.concatenate(d))
        dW = orc.absorb(G, R, W, orc.ridge_lambda(G))
        orc.project(a[-1], orc.modulated_weight(W, dW))
    return run


def cpu_baseline(rows=256, rows_1t=32):
    from threadpoolctl import threadpool_limits
    run, flops = oracle_sample(rows)
    t0 = time.perf_counter()
    run()
    dt = time.perf_counter() - t0
    run1, flops1 = oracle_sample(rows_1t)
    tiny = oracle_tiny_step()
    with threadpool_limits(limits=1, user_api="blas"):
        t0 = time.perf_counter()
        run1()
        dt1 = time.perf_counter() - t0
        t0 = time.perf_counter()
        tiny()
        dt_tiny1 = time.perf_counter() - t0
    t0 = time.perf_counter()
    tiny()
    dt_tiny = time.perf_counter() - t0
    blas = blas_info()
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": cores(), "kind": "oracle",
            "blas": blas["vendor"], "blas_threads": blas["threads"],
            "sample": f"fp64 numpy oracle, {rows} of 4680 query rows of the wan1.3b chunk (local, history and "
                      f"single-pass full attention), {dt:.2f} s",
            "one_thread": {"wan1.3b_tflops": round(flops1 / dt1 / 1e12, 6),
                           "wan1.3b_sample": f"{rows_1t} query rows, {dt1:.2f} s",
                           "tiny_f32_step_ms": round(dt_tiny1 * 1e3, 2)},
            "tiny_f32_step_ms": round(dt_tiny * 1e3, 2),
            "tiny_f32_step": "4 warm-up chunks of the dual stream, statistics, absorb, one L-layer projection"}


def run_reference(args):
    rows = 64
    run, flops = oracle_sample(rows)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = time.perf_counter() - t0
    v = flops * args.steps / dt / 1e12
    return {"impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded PCG64; Wan-1.3B latent shapes)",
            "config": {"workload": "wan1.3b single layer dual-stream attention; each step a bounded sample of "
                                   f"{rows} query rows", "parallelism": "none (host cores)"},
            "cpu_baseline": {"value": round(v, 6), "unit": "TFLOP/s", "cores": cores(), "kind": "oracle",
                             "blas": blas_info()["vendor"], "blas_threads": blas_info()["threads"],
                             "sample": f"{rows} of 4680 query rows per step"},
            "e2e": {"value": round(v, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-rollout", action="store_true", help="skip the 30-layer streaming rollout")
    ap.add_argument("--profile", choices=["dual", "full", "local", "gram", "project", "merge", "absorb",
                                          "project_w8a8", "quantize_rows", "project_mx", "local_mx",
                                          "layer_error"],
                    help="run only this op --steps times on the wan1.3b shapes (for ncu captures), no timing")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    from ar_video_diffusion_b200 import build as ispa_build
    if rank == 0:
        ispa_build.build()
    if world > 1:
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        torch.distributed.barrier()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device for the GPU arm")
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if args.profile:
        run_profile_case(args.profile, args.steps, device)
        return
    res = run_ours(args, rank, world, device)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline()
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

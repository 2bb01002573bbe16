"""Shared helpers of the GPU parity tests: moving seeded numpy inputs to the
device and the error measures the tolerances are stated in."""
import numpy as np
import torch

from oracle import ispa_oracle as orc

# Tolerances (bf16 operands, fp32 accumulation):
ATTN_MAX_REL = 2e-2      # attention outputs: max|x - ref| / max|ref| per tensor
LSE_ABS = 1e-3           # log-sum-exp: absolute
DW_REL_BF16 = 1e-2       # dW: relative Frobenius, statistics fed from bf16 activations
DW_REL_F32 = 1e-3        # dW: relative Frobenius, fp32 workloads
# G, R: fp32 sums of exact bf16 products over n rows; the only error is the
# fp32 summation, ~sqrt(n) * 2^-24 relative, far below this bound.
GRAM_REL = 1e-4
# y = A W: bf16 operands, fp32 accumulation over D terms, bf16 output rounding
PROJ_MAX_REL = 1e-2


def dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    t = t.to(torch.bfloat16) if dtype == "bf16" else t
    return t.cuda()


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def max_rel(x, ref) -> float:
    ref = np.asarray(ref, np.float64)
    return float(np.max(np.abs(np.asarray(x, np.float64) - ref)) / max(np.max(np.abs(ref)), 1e-30))


def max_abs(x, ref) -> float:
    return float(np.max(np.abs(np.asarray(x, np.float64) - np.asarray(ref, np.float64))))


def fro_rel(x, ref) -> float:
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(np.asarray(x, np.float64) - ref) / np.linalg.norm(ref))


# ------------------------------------------------ streaming rollout helpers
def cat_segments(segs, i, D):
    return np.concatenate([host(s[i]) for s in segs]) if segs else np.zeros((0, D))


def oracle_rollout_statistics(w, inputs, layer):
    """The oracle's A_loc and A_full over every warm-up row of one layer, from
    the captured seeded inputs of that layer's warm-up chunks."""
    a_loc, a_full = [], []
    for c in range(w.warm_chunks):
        x = inputs[(layer, c)]
        ref = orc.dual_stream(x["q"], [(x["k_loc"], x["v_loc"])], [(x["k_hist"], x["v_hist"])], w.n_heads)
        a_loc.append(ref["a_loc"])
        a_full.append(ref["a_full"])
    return np.concatenate(a_loc), np.concatenate(a_full)


def capture_inputs(w, store, with_y=True):
    """on_layer hook: host copies of each layer's seeded inputs (queries and
    the K/V segments it attends to; one local segment list concatenated) and
    of its output."""
    def on_layer(l, c, info):
        torch.cuda.synchronize()
        D = w.d_model
        rec = {"mode": info["mode"], "q": host(info["q"]),
               "k_loc": cat_segments(info["local"], 0, D), "v_loc": cat_segments(info["local"], 1, D),
               "k_hist": cat_segments(info["hist"], 0, D), "v_hist": cat_segments(info["hist"], 1, D)}
        if with_y:
            rec["y"] = host(info["y"])
        store[(l, c)] = rec
    return on_layer

"""Multi-GPU sharding of the ISPA hot path: one process per GPU, torch.distributed.

The method ("Instance-Specific Parametric Absorption", gist.science technical
summary, section 2) shards without changing its arithmetic:

* Decomposable attention (stage 1): every query row is independent, so the
  chunk's queries are split across ranks in whole 128-row query tiles.  Each
  rank holds the layer's K/V and runs the dual-stream kernel on its rows: no
  exchange.
* Statistics (stage 2): G = sum over rows of A_loc^T A_loc and R likewise are
  sums over rows.  Each rank accumulates its rows and one all-reduce (sum) of
  the packed [G | R] buffer gives every rank the full statistics, 2 D^2 fp32
  (18.9 MB at D = 1536).
* Absorb (stage 2) and modulation (stage 3): layers are independent
  ("Dynamic Layer Selection": the selected layers are absorbed one by one).
  The i-th absorbed layer in increasing layer order is solved by rank
  i mod world, so the ranks' shares differ by at most one layer whatever the
  selected set (the even layers, or an instance-specific choice).  Every rank
  first solves all of its layers back to back, then the owners broadcast
  W_new (D^2 in the weight dtype) to the others, which need it for their rows
  of the L-layer; the broadcasts are issued together and awaited at the end,
  so no rank's solve waits for another rank's.

Every step on a device runs in libispa's kernels through ``ispa``; this module
only partitions rows and layers and issues the collectives.  The collectives
are NCCL's over NVLink (the transfers are small and not fused with compute).
"""
from __future__ import annotations

from typing import Optional, Sequence, Tuple

import torch
import torch.distributed as dist

from . import ispa

Q_TILE = 128  # query rows per attention CTA: shards never split a query tile


def query_shard(n_q: int, world: int, rank: int, tile: int = Q_TILE) -> Tuple[int, int]:
    """Half-open row range [begin, end) of rank `rank`.  Ranges are made of
    whole query tiles (only the last range may end in a partial tile), cover
    [0, n_q) without overlap, and differ by at most one tile."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    n_tiles = (n_q + tile - 1) // tile
    base, extra = divmod(n_tiles, world)
    t0 = rank * base + min(rank, extra)
    t1 = t0 + base + (1 if rank < extra else 0)
    return min(t0 * tile, n_q), min(t1 * tile, n_q)


def absorb_owners(layers: Sequence[int], world: int) -> dict:
    """layer -> the rank that solves its absorb: the i-th layer of the sorted
    set goes to rank i mod world (balanced to within one layer)."""
    if world <= 0:
        raise ValueError("world must be positive")
    return {l: i % world for i, l in enumerate(sorted(set(layers)))}


def new_statistics(d_model: int, device) -> torch.Tensor:
    """The packed statistics buffer [2, D, D] fp32: [0] is G, [1] is R.  One
    buffer makes the all-reduce a single collective."""
    return torch.zeros(2, d_model, d_model, dtype=torch.float32, device=device)


def accumulate_statistics(a_loc: torch.Tensor, a_delta: torch.Tensor, stats: torch.Tensor,
                          zero_first: bool = False, stream=None):
    """This rank's rows into its partial G, R (the tensor-core statistics
    kernel; G's lower triangle)."""
    ispa.gram_accumulate(a_loc, a_delta, stats[0], stats[1], zero_first=zero_first, stream=stream)


def allreduce_statistics(stats: torch.Tensor, group=None):
    """Sum the ranks' partial [G | R] in place: afterwards every rank holds the
    statistics of all rows."""
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(stats, op=dist.ReduceOp.SUM, group=group)


def dual_attention_rows(q: torch.Tensor, local: Sequence[Tuple[torch.Tensor, torch.Tensor]],
                        hist: Sequence[Tuple[torch.Tensor, torch.Tensor]], n_heads: int, world: int, rank: int,
                        status: Optional[torch.Tensor] = None, stream=None):
    """Dual-stream attention of this rank's query rows (a view of q with q's
    row stride).  Returns (begin, end, outputs); `outputs` holds the rows
    [begin, end) of A_loc, A_full, delta and the LSEs."""
    b, e = query_shard(q.shape[0], world, rank)
    if e == b:
        return b, e, None
    out = ispa.dual_attention(q[b:e], local, hist, n_heads, status=status, stream=stream)
    return b, e, out


def absorb_layers(stats_by_layer, W_by_layer, world: int, rank: int, lambda_rel: float = 1e-2,
                  workspace: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                  group=None):
    """Solve the absorbs of the layers this rank owns and share every W_new.

    stats_by_layer / W_by_layer: dicts layer -> all-reduced [2, D, D] stats /
    weight [D, D].  Returns a dict layer -> W_new, identical on every rank.
    This rank's solves run back to back first; then every rank takes the same
    broadcasts in the same (sorted layer) order, issued asynchronously and
    awaited together."""
    owners = absorb_owners(stats_by_layer.keys(), world)
    w_new = {}
    for l in sorted(stats_by_layer):
        if owners[l] == rank:
            _, w_new[l] = ispa.absorb_solve(stats_by_layer[l][0], stats_by_layer[l][1], W_by_layer[l],
                                            lambda_rel=lambda_rel, workspace=workspace, status=status)
        else:
            w_new[l] = torch.empty_like(W_by_layer[l])
    if dist.is_initialized() and world > 1:
        works = [dist.broadcast(w_new[l], src=owners[l], group=group, async_op=True) for l in sorted(w_new)]
        for wk in works:
            wk.wait()
    return w_new

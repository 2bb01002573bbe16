"""Host side of the N > 1 benchmark path, on CPU with two gloo ranks.

The hot path is replicated, not sharded: with N processes every rank runs the
same layer, and the only collectives are the barriers and the max over ranks
of the device times that define the throughput.  These tests run that
reduction and the reference arm's rank handling as real separate processes.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

RANK_CODE = r"""
import datetime, json, os, sys
sys.path.insert(0, os.environ["ISPA_ROOT"])
import torch
import torch.distributed as dist
import bench
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
rank, world = dist.get_rank(), dist.get_world_size()
times = json.loads(os.environ["RANK_TIMES"])[rank]
got = bench.max_over_ranks(times, world, torch.device("cpu"))
value = bench.replica_tflops(2.0e12, 4, world, got[0])
dist.barrier()
dist.destroy_process_group()
print(json.dumps({"rank": rank, "world": world, "max": got, "value": value}))
"""


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run_ranks(code, world, extra_env, args=(), timeout=120):
    port = _free_port()
    procs = []
    for r in range(world):
        env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(r),
                   LOCAL_RANK=str(r), WORLD_SIZE=str(world), ISPA_ROOT=ROOT, **extra_env)
        cmd = [sys.executable, "-c", code] if code else [sys.executable, os.path.join(ROOT, "bench.py"), *args]
        procs.append(subprocess.Popen(cmd, env=env, cwd=ROOT, stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                                      text=True))
    outs = []
    try:
        for p in procs:
            out, err = p.communicate(timeout=timeout)
            outs.append((p.returncode, out, err))
    finally:
        for p in procs:
            if p.poll() is None:
                p.kill()
    return outs


def test_max_over_ranks_two_gloo_ranks():
    # rank 0 is slower on the first timing, rank 1 on the second
    times = [[30.0, 7.5, 1.0], [20.0, 9.25, 1.0]]
    outs = _run_ranks(RANK_CODE, 2, {"RANK_TIMES": json.dumps(times)})
    results = []
    for rc, out, err in outs:
        assert rc == 0, err[-2000:]
        results.append(json.loads(out.strip().splitlines()[-1]))
    assert sorted(r["rank"] for r in results) == [0, 1]
    for r in results:
        assert r["world"] == 2
        assert r["max"] == [30.0, 9.25, 1.0]
        # 2 replicas x 4 steps x 2 TFLOP over the slowest rank's 30 ms
        assert r["value"] == pytest.approx(2 * 4 * 2.0 / 30e-3)


def test_replica_tflops_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    import torch
    assert bench.max_over_ranks([1.5, 2.5], 1, torch.device("cpu")) == [1.5, 2.5]
    assert bench.replica_tflops(1.0e12, 10, 1, 1000.0) == pytest.approx(10.0)
    # weak scaling: N replicas over the same slowest time give N times the value
    assert bench.replica_tflops(1.0e12, 10, 8, 1000.0) == pytest.approx(80.0)


def test_reference_arm_other_ranks_do_no_work():
    # under torchrun only rank 0 runs the oracle arm; rank 1 exits at once
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2", MASTER_ADDR="127.0.0.1",
               MASTER_PORT=str(_free_port()))
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, cwd=ROOT, capture_output=True, text=True,
                       timeout=120)
    assert p.returncode == 0, p.stderr[-2000:]
    assert p.stdout.strip() == ""


def test_reference_arm_rank0_line():
    env = dict(os.environ, RANK="0", LOCAL_RANK="0", WORLD_SIZE="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr[-2000:]
    line = json.loads(p.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["value"] > 0


# ------------------------------------------------------ sharded hot path (host side)
def test_query_shard_partitions_whole_tiles():
    sys.path.insert(0, ROOT)
    from ar_video_diffusion_b200 import sharded
    for n in (1, 127, 128, 129, 300, 4680, 18720):
        for world in (1, 2, 3, 4, 8):
            ranges = [sharded.query_shard(n, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == n
            for (b0, e0), (b1, e1) in zip(ranges, ranges[1:]):
                assert e0 == b1  # contiguous, no overlap
            sizes_in_tiles = [-(-(e - b) // 128) for b, e in ranges]
            assert max(sizes_in_tiles) - min(sizes_in_tiles) <= 1
            for b, e in ranges:
                # a range starts on a tile boundary (an empty one sits at n) and ends on one or at n
                assert (b % 128 == 0 or b == e == n) and (e % 128 == 0 or e == n)
    with pytest.raises(ValueError):
        sharded.query_shard(10, 2, 2)


STATS_CODE = r"""
import datetime, json, os, sys
sys.path.insert(0, os.environ["ISPA_ROOT"])
import numpy as np
import torch
import torch.distributed as dist
from ar_video_diffusion_b200 import sharded
from oracle import ispa_oracle as orc
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
rank, world = dist.get_rank(), dist.get_world_size()
rng = np.random.default_rng(5)                      # the same seeded rows on every rank
n, D = 700, 48
A = rng.standard_normal((n, D))
Dl = 0.1 * rng.standard_normal((n, D))
b, e = sharded.query_shard(n, world, rank)
# stand-in for the statistics kernel on this rank's rows (CPU, fp64)
stats = torch.zeros(2, D, D, dtype=torch.float64)
stats[0] = torch.from_numpy(A[b:e].T @ A[b:e])
stats[1] = torch.from_numpy(A[b:e].T @ Dl[b:e])
sharded.allreduce_statistics(stats)
G, R = orc.gram(A, Dl)
err = max(float(np.abs(stats[0].numpy() - G).max() / np.abs(G).max()),
          float(np.abs(stats[1].numpy() - R).max() / np.abs(R).max()))
dist.barrier()
dist.destroy_process_group()
print(json.dumps({"rank": rank, "rows": [b, e], "err": err}))
"""


def test_statistics_allreduce_two_gloo_ranks():
    outs = _run_ranks(STATS_CODE, 2, {})
    res = []
    for rc, out, err in outs:
        assert rc == 0, err[-2000:]
        res.append(json.loads(out.strip().splitlines()[-1]))
    rows = sorted(tuple(r["rows"]) for r in res)
    assert rows[0][0] == 0 and rows[0][1] == rows[1][0] and rows[1][1] == 700
    for r in res:
        assert r["err"] < 1e-12  # the sum of the partial Gram matrices is the oracle's Gram


ABSORB_CODE = r"""
import datetime, json, os, sys
sys.path.insert(0, os.environ["ISPA_ROOT"])
import numpy as np
import torch
import torch.distributed as dist
from ar_video_diffusion_b200 import sharded
from oracle import ispa_oracle as orc
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
rank, world = dist.get_rank(), dist.get_world_size()
solved = []

def absorb_solve(G, R, W, lambda_rel=1e-2, workspace=None, status=None):
    # stand-in for the device solve: the oracle's, on this rank
    Gn, Rn, Wn = (t.numpy().astype(np.float64) for t in (G, R, W))
    Gs = np.tril(Gn) + np.tril(Gn, -1).T
    dW = orc.absorb(Gs, Rn, Wn, orc.ridge_lambda(Gs, lambda_rel))
    solved.append(len(solved))
    return torch.from_numpy(dW), torch.from_numpy(Wn + dW)

sharded.ispa.absorb_solve = absorb_solve
D, layers = 16, [0, 2, 4, 6, 8]
rng = np.random.default_rng(9)
stats, W = {}, {}
for l in layers:
    A = rng.standard_normal((40, D))
    Dl = 0.1 * rng.standard_normal((40, D))
    s = torch.zeros(2, D, D, dtype=torch.float64)
    s[0] = torch.from_numpy(A.T @ A)
    s[1] = torch.from_numpy(A.T @ Dl)
    stats[l] = s
    W[l] = torch.from_numpy(rng.standard_normal((D, D)) / 4)
w_new = sharded.absorb_layers(stats, W, world, rank)
mine = [l for l, r in sharded.absorb_owners(layers, world).items() if r == rank]
out = {"rank": rank, "n_solved": len(solved), "mine": mine,
       "w_new": {str(l): float(w_new[l].sum()) for l in layers}}
dist.barrier()
dist.destroy_process_group()
print(json.dumps(out))
"""


def test_absorb_layers_owned_once_and_broadcast_two_gloo_ranks():
    outs = _run_ranks(ABSORB_CODE, 2, {})
    res = []
    for rc, out, err in outs:
        assert rc == 0, err[-2000:]
        res.append(json.loads(out.strip().splitlines()[-1]))
    # every layer solved exactly once, by its owner; every rank ends with the same W_new
    owned = sorted(l for r in res for l in r["mine"])
    assert owned == [0, 2, 4, 6, 8]
    for r in res:
        assert r["n_solved"] == len(r["mine"])
    # both ranks solve: the even layers are split 3 / 2, not all to rank 0
    assert sorted(len(r["mine"]) for r in res) == [2, 3]
    assert res[0]["w_new"] == res[1]["w_new"]


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_absorb_owners_balanced_for_any_layer_set(world):
    from ar_video_diffusion_b200 import sharded
    rng = np.random.default_rng(world)
    sets = [list(range(0, 30, 2)), list(range(1, 30, 2)), list(range(30)),
            sorted(rng.choice(30, 15, replace=False).tolist()), [4], []]
    for layers in sets:
        owners = sharded.absorb_owners(layers, world)
        assert sorted(owners) == sorted(layers)
        counts = [sum(1 for r in owners.values() if r == k) for k in range(world)]
        assert sum(counts) == len(layers)
        assert max(counts) - min(counts) <= 1, (layers, counts)
        assert all(0 <= r < world for r in owners.values())

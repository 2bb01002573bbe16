"""GPU parity: every entry point of libispa against the fp64 oracle, through
the C ABI, on seeded inputs -- small cases that span several 128-row/128-key
tiles with ragged tails, edge cases (no history, one key, one query row, many
segments, short and long history), and the full Wan-1.3B-shaped layer on
sampled query rows (attention is row-independent, so a row subset is exact).
Tolerances: see tests/helpers.py."""
import numpy as np
import pytest
import torch

from ar_video_diffusion_b200 import build as ispa_build
from ar_video_diffusion_b200 import ispa, synth
from oracle import ispa_oracle as orc
from helpers import (ATTN_MAX_REL, DW_REL_BF16, DW_REL_F32, GRAM_REL, LSE_ABS, PROJ_MAX_REL, dev, fro_rel, host,
                     max_abs, max_rel)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    ispa_build.build()
    ispa.lib()


def _run_dual(case, n_local_segs, H, dtype, dual=True, rows=None):
    q = case["q"]
    segs = case["segments"]
    loc = [(dev(k, dtype), dev(v, dtype)) for k, v in segs[:n_local_segs]]
    his = [(dev(k, dtype), dev(v, dtype)) for k, v in segs[n_local_segs:]]
    status = ispa.new_status()
    out = ispa.dual_attention(dev(q, dtype), loc, his, H, dual=dual, status=status)
    torch.cuda.synchronize()
    ispa.raise_on_status(status, "dual_attention")
    return {k: host(v) for k, v in out.items()}


def _oracle_dual(case, n_local_segs, H, rows=None):
    q = case["q"] if rows is None else case["q"][rows]
    segs = case["segments"]
    return orc.dual_stream(q, segs[:n_local_segs], segs[n_local_segs:], H)


def _check_dual(got, ref, rows=None, dual=True):
    sl = slice(None) if rows is None else rows
    if dual:
        assert max_rel(got["a_loc"][sl], ref["a_loc"]) <= ATTN_MAX_REL
        assert max_rel(got["a_delta"][sl], ref["delta"]) <= ATTN_MAX_REL
        assert max_abs(got["lse_loc"][:, sl], ref["lse_loc"]) <= LSE_ABS
    assert max_rel(got["a_full"][sl], ref["a_full"]) <= ATTN_MAX_REL
    assert max_abs(got["lse_full"][:, sl], ref["lse_full"]) <= LSE_ABS


# (seed, n_q, H, d, local segment lengths, history segment lengths)
DUAL_CASES = [
    (1, 300, 2, 128, [100, 300], [700]),        # ragged everywhere; even number of local tiles
    (2, 130, 3, 64, [16, 64], [256]),           # head_dim 64
    (3, 257, 2, 128, [128, 256], [128]),        # odd local tiles, one history tile: warpgroup 0 has no
                                                # history tile and takes its checkpoint after its loop
    (4, 200, 1, 128, [1560 // 8, 4680 // 8], []),  # no history at all
    (5, 1, 2, 128, [1], [5]),                  # one query row, one local key
    (6, 129, 2, 128, [3, 200, 17], [64, 1, 300, 129]),  # many segments, tiny ones
    (7, 64, 2, 64, [16, 64], [0, 256]),         # an empty history segment is ignored
    (8, 390, 4, 128, [200, 390], [2500]),       # long history
    (9, 77, 2, 128, [50], []),                  # a single key tile: warpgroup 1 owns no tile
    (10, 140, 2, 128, [10, 130, 30, 40], [50, 129, 70, 1]),  # the maximum of 8 segments
]


@pytest.mark.parametrize("seed,n_q,H,d,loc,his", DUAL_CASES)
def test_dual_attention_bf16_matches_oracle(seed, n_q, H, d, loc, his):
    case = synth.random_case(seed, n_q, H, d, loc + his, dtype="bf16")
    got = _run_dual(case, len(loc), H, "bf16")
    ref = _oracle_dual(case, len(loc), H)
    _check_dual(got, ref)


@pytest.mark.parametrize("seed,n_q,H,d,loc,his", DUAL_CASES[:3] + DUAL_CASES[5:6] + DUAL_CASES[8:9])
def test_single_pass_attention_bf16_matches_oracle(seed, n_q, H, d, loc, his):
    case = synth.random_case(seed, n_q, H, d, loc + his, dtype="bf16")
    got = _run_dual(case, len(loc), H, "bf16", dual=False)
    ref = _oracle_dual(case, len(loc), H)
    _check_dual(got, ref, dual=False)


@pytest.mark.parametrize("seed,n_q,H,d,loc,his", DUAL_CASES[:3])
def test_dual_attention_f32_matches_oracle(seed, n_q, H, d, loc, his):
    case = synth.random_case(seed, n_q, H, d, loc + his, dtype="f32")
    got = _run_dual(case, len(loc), H, "f32")
    ref = _oracle_dual(case, len(loc), H)
    _check_dual(got, ref)


def test_tiny_f32_workload_end_to_end():
    """Tiny fp32 layer: 4 warm-up chunks of dual attention, statistics over
    256 rows, absorb solve.  dW is checked against the oracle chain: the
    oracle's own dual stream, its G, R and its solve, from the same seeded
    inputs.  The fp32 attention path is accurate to about 1e-6 relative, so
    the chained dW stays within the fp32 bound."""
    w = synth.WORKLOADS["tiny_f32"]
    D = w.d_model
    G = torch.zeros(D, D, device="cuda")
    R = torch.zeros(D, D, device="cuda")
    A_rows, D_rows = [], []
    for c in range(w.warm_chunks):
        x = synth.single_layer_inputs(w, c)
        status = ispa.new_status()
        out = ispa.dual_attention(dev(x["q"], "f32"), [(dev(x["k_sink"], "f32"), dev(x["v_sink"], "f32")),
                                                      (dev(x["k_cur"], "f32"), dev(x["v_cur"], "f32"))],
                                  [(dev(x["k_hist"], "f32"), dev(x["v_hist"], "f32"))], w.n_heads, status=status)
        ispa.gram_accumulate(out["a_loc"], out["a_delta"], G, R, zero_first=(c == 0))
        torch.cuda.synchronize()
        ispa.raise_on_status(status, "dual_attention")
        ref = orc.dual_stream(x["q"], [(x["k_sink"], x["v_sink"]), (x["k_cur"], x["v_cur"])],
                              [(x["k_hist"], x["v_hist"])], w.n_heads)
        _check_dual({k: host(v) for k, v in out.items()}, ref)
        A_rows.append(ref["a_loc"])
        D_rows.append(ref["a_full"] - ref["a_loc"])
    A, Dl = np.concatenate(A_rows), np.concatenate(D_rows)
    Gr, Rr = orc.gram(A, Dl)
    assert fro_rel(host(G), Gr) <= GRAM_REL and fro_rel(host(R), Rr) <= GRAM_REL
    W = synth.weight(w, 0)
    status = ispa.new_status()
    dW, Wn = ispa.absorb_solve(G, R, dev(W, "f32"), lambda_rel=orc.LAMBDA_REL, status=status)
    torch.cuda.synchronize()
    ispa.raise_on_status(status, "absorb_solve")
    dW_ref = orc.absorb(Gr, Rr, W, orc.ridge_lambda(Gr))
    assert fro_rel(host(dW), dW_ref) <= DW_REL_F32
    assert max_abs(host(Wn), W + dW_ref) <= 1e-4 * np.max(np.abs(W))


def test_wan13b_layer_sampled_rows():
    """Full Wan-1.3B-shaped warm-up chunk (4680 queries, 1560 sink, 18720
    history, 12 heads of 128) in the launch configuration the benchmark
    times; 256 seeded query rows are checked against the oracle."""
    w = synth.WORKLOADS["wan1.3b"]
    x = synth.single_layer_inputs(w, 1)
    status = ispa.new_status()
    out = ispa.dual_attention(dev(x["q"], "bf16"), [(dev(x["k_sink"], "bf16"), dev(x["v_sink"], "bf16")),
                                                   (dev(x["k_cur"], "bf16"), dev(x["v_cur"], "bf16"))],
                              [(dev(x["k_hist"], "bf16"), dev(x["v_hist"], "bf16"))], w.n_heads, status=status)
    torch.cuda.synchronize()
    ispa.raise_on_status(status, "dual_attention")
    got = {k: host(v) for k, v in out.items()}
    rows = np.sort(np.random.default_rng(11).choice(w.n_q, 256, replace=False))
    rows[-1] = w.n_q - 1  # always include the ragged last tile
    ref = orc.dual_stream(x["q"][rows], [(x["k_sink"], x["v_sink"]), (x["k_cur"], x["v_cur"])],
                          [(x["k_hist"], x["v_hist"])], w.n_heads)
    _check_dual(got, ref, rows=rows)
    # every output is finite over the whole chunk
    for k, v in got.items():
        assert np.all(np.isfinite(v)), k


def test_lse_merge_matches_oracle():
    g = np.random.default_rng(5)
    H, d, n = 3, 128, 517
    o_loc = synth.round_bf16(g.standard_normal((n, H * d)).astype(np.float32))
    o_hist = synth.round_bf16(g.standard_normal((n, H * d)).astype(np.float32))
    l_loc = (g.standard_normal((H, n)) * 3).astype(np.float32)
    l_hist = (g.standard_normal((H, n)) * 3).astype(np.float32)
    l_hist[1, :50] = -np.inf  # empty history rows
    out = ispa.lse_merge(dev(o_loc, "bf16"), torch.from_numpy(l_loc).cuda(), dev(o_hist, "bf16"),
                         torch.from_numpy(l_hist).cuda(), H)
    torch.cuda.synchronize()
    a_full, delta, L = orc.lse_merge(o_loc, l_loc, o_hist, l_hist, H)
    assert max_rel(host(out["a_full"]), a_full) <= ATTN_MAX_REL
    assert max_rel(host(out["a_delta"]), delta) <= ATTN_MAX_REL
    assert max_abs(host(out["lse_full"]), L) <= LSE_ABS
    # rows with an empty history reproduce the local branch exactly
    assert np.array_equal(host(out["a_full"])[:50, d:2 * d], o_loc[:50, d:2 * d])


def test_lse_merge_rows_with_both_branches_empty():
    """(row, head) pairs whose local and historical branches are both empty
    (both LSEs -inf; the outputs of those branches are 0, as attention over no
    keys gives): A_full = 0 and LSE = -inf, as for attention over the empty
    union, and no NaN anywhere; every other pair as the oracle."""
    g = np.random.default_rng(6)
    H, d, n = 2, 64, 131
    o_loc = synth.round_bf16(g.standard_normal((n, H * d)).astype(np.float32))
    o_hist = synth.round_bf16(g.standard_normal((n, H * d)).astype(np.float32))
    l_loc = (g.standard_normal((H, n)) * 3).astype(np.float32)
    l_hist = (g.standard_normal((H, n)) * 3).astype(np.float32)
    empty = np.zeros((H, n), bool)
    empty[0, 10:40] = True
    empty[1, 100:] = True
    for h in range(H):
        r = np.nonzero(empty[h])[0]
        l_loc[h, r] = l_hist[h, r] = -np.inf
        o_loc[np.ix_(r, range(h * d, (h + 1) * d))] = 0.0
        o_hist[np.ix_(r, range(h * d, (h + 1) * d))] = 0.0
    out = ispa.lse_merge(dev(o_loc, "bf16"), torch.from_numpy(l_loc).cuda(), dev(o_hist, "bf16"),
                         torch.from_numpy(l_hist).cuda(), H)
    torch.cuda.synchronize()
    got = {k: host(v) for k, v in out.items()}
    a_full, delta, L = orc.lse_merge(o_loc, l_loc, o_hist, l_hist, H)
    for v in got.values():
        assert not np.any(np.isnan(v))
    assert np.array_equal(np.isneginf(got["lse_full"]), empty) and np.array_equal(np.isneginf(L), empty)
    assert max_abs(got["lse_full"][~empty], L[~empty]) <= LSE_ABS
    assert max_rel(got["a_full"], a_full) <= ATTN_MAX_REL
    assert max_rel(got["a_delta"], delta) <= ATTN_MAX_REL
    for h in range(H):
        r = np.nonzero(empty[h])[0]
        assert np.all(got["a_full"][np.ix_(r, range(h * d, (h + 1) * d))] == 0.0)


# (1, 256): one row; (130, 512): ragged rows over several 224-wide tiles
# (the last overhangs D); (1000, 640): a width the 256-wide tile cannot take
@pytest.mark.parametrize("n_rows,D", [(4680, 1536), (300, 256), (1, 256), (130, 512), (5000, 768), (1000, 640),
                                      (1, 128), (129, 384)])
def test_gram_bf16_matches_oracle(n_rows, D):
    g = np.random.default_rng(n_rows + D)
    A = synth.round_bf16((g.standard_normal((n_rows, D)) * 0.3).astype(np.float32))
    Dl = synth.round_bf16((g.standard_normal((n_rows, D)) * 0.1).astype(np.float32))
    G = torch.full((D, D), 7.0, device="cuda")
    R = torch.full((D, D), -3.0, device="cuda")
    ispa.gram_accumulate(dev(A, "bf16"), dev(Dl, "bf16"), G, R, zero_first=True)
    ispa.gram_accumulate(dev(A, "bf16"), dev(Dl, "bf16"), G, R, zero_first=False)  # accumulate a second time
    torch.cuda.synchronize()
    Gr, Rr = orc.gram(A, Dl)
    # G is symmetric and only its lower triangle is produced
    assert fro_rel(np.tril(host(G)), np.tril(2 * Gr)) <= GRAM_REL
    assert fro_rel(host(R), 2 * Rr) <= GRAM_REL


def _absorb_case(seed, n, D, dtype):
    g = np.random.default_rng(seed)
    A = synth.round_bf16((g.standard_normal((n, D)) * 0.2).astype(np.float32))
    Dl = synth.round_bf16((g.standard_normal((n, D)) * 0.05).astype(np.float32))
    W = (g.standard_normal((D, D)) / np.sqrt(D)).astype(np.float32)
    if dtype == "bf16":
        W = synth.round_bf16(W)
    return A, Dl, W


@pytest.mark.parametrize("n,D,dtype", [(18720, 1536, "bf16"), (600, 128, "f32"), (900, 320, "bf16")])
def test_absorb_solve_matches_oracle(n, D, dtype):
    A, Dl, W = _absorb_case(D, n, D, dtype)
    G = torch.empty(D, D, device="cuda")
    R = torch.empty(D, D, device="cuda")
    if dtype == "bf16" and D % 128 == 0:
        ispa.gram_accumulate(dev(A, "bf16"), dev(Dl, "bf16"), G, R, zero_first=True)
    else:
        ispa.gram_accumulate(dev(A, "f32"), dev(Dl, "f32"), G, R, zero_first=True)
    status = ispa.new_status()
    dW, Wn = ispa.absorb_solve(G, R, dev(W, dtype), lambda_rel=orc.LAMBDA_REL, status=status)
    torch.cuda.synchronize()
    ispa.raise_on_status(status, "absorb_solve")
    Gr, Rr = orc.gram(A, Dl)
    dW_ref = orc.absorb(Gr, Rr, W, orc.ridge_lambda(Gr))
    tol = DW_REL_BF16 if dtype == "bf16" else DW_REL_F32
    assert fro_rel(host(dW), dW_ref) <= tol
    # the normal-equation residual of the GPU answer, relative to R W
    lam = orc.ridge_lambda(Gr)
    res = (Gr + lam * np.eye(D)) @ host(dW) - Rr @ W
    assert np.linalg.norm(res) <= tol * np.linalg.norm(Rr @ W)
    assert max_rel(host(Wn), W + dW_ref) <= 1e-2


def test_absorb_zero_statistics_gives_zero_update():
    D = 256
    g = np.random.default_rng(3)
    A = synth.round_bf16(g.standard_normal((500, D)).astype(np.float32))
    G = torch.empty(D, D, device="cuda")
    R = torch.empty(D, D, device="cuda")
    zeros = np.zeros_like(A)
    ispa.gram_accumulate(dev(A, "bf16"), dev(zeros, "bf16"), G, R, zero_first=True)
    W = synth.round_bf16((g.standard_normal((D, D)) / 16).astype(np.float32))
    dW, Wn = ispa.absorb_solve(G, R, dev(W, "bf16"))
    torch.cuda.synchronize()
    assert torch.count_nonzero(R).item() == 0
    assert torch.count_nonzero(dW).item() == 0
    assert np.array_equal(host(Wn), W)


def test_absorb_reports_not_spd():
    D = 128
    G = torch.zeros(D, D, device="cuda")
    G[:64, :64] = torch.eye(64, device="cuda")  # rank-deficient, lambda = 0
    R = torch.zeros(D, D, device="cuda")
    W = torch.zeros(D, D, device="cuda")
    status = ispa.new_status()
    ispa.absorb_solve(G, R, W, lambda_rel=0.0, status=status)
    torch.cuda.synchronize()
    code, pivot = status.cpu().tolist()
    assert code == 4 and pivot == 64


def test_bounded_wait_times_out_and_gpu_stays_usable():
    status = ispa.new_status()
    ispa.ispa_selftest_wait_timeout(2000, status.data_ptr(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert status[0].item() == 5
    x = torch.ones(1000, device="cuda")
    assert x.sum().item() == 1000


# (4680, *, 1536) and (4680, *, 1280) take the 128 x 384 tile (the second
# overhangs the last columns), (4680, *, 5120) the 256 x 256 tile and
# (77, *, 256) the 256 x 128 tile on a 148-SM B200
@pytest.mark.parametrize("n,din,dout", [(4680, 1536, 1536), (4680, 256, 1280), (4680, 64, 5120), (77, 128, 256)])
def test_project_bf16_matches_oracle(n, din, dout):
    g = np.random.default_rng(n)
    A = synth.round_bf16(g.standard_normal((n, din)).astype(np.float32))
    W = synth.round_bf16((g.standard_normal((din, dout)) / np.sqrt(din)).astype(np.float32))
    y = ispa.project(dev(A, "bf16"), dev(W, "bf16"))
    torch.cuda.synchronize()
    assert max_rel(host(y), orc.project(A, W)) <= PROJ_MAX_REL


def test_local_attention_project_matches_oracle():
    case = synth.random_case(9, 333, 2, 128, [156, 333], dtype="bf16")
    (ks, vs), (kc, vc) = case["segments"]
    g = np.random.default_rng(9)
    Wn = synth.round_bf16((g.standard_normal((256, 256)) / 16).astype(np.float32))
    status = ispa.new_status()
    y, a_loc = ispa.local_attention_project(dev(case["q"], "bf16"),
                                            [(dev(ks, "bf16"), dev(vs, "bf16")), (dev(kc, "bf16"), dev(vc, "bf16"))],
                                            dev(Wn, "bf16"), 2, status=status)
    torch.cuda.synchronize()
    ispa.raise_on_status(status, "local_attention_project")
    a_ref, _ = orc.attention(case["q"], np.concatenate([ks, kc]), np.concatenate([vs, vc]), 2)
    assert max_rel(host(a_loc), a_ref) <= ATTN_MAX_REL
    assert max_rel(host(y), orc.project(a_ref, Wn)) <= ATTN_MAX_REL


def test_local_attention_project_wan13b_sampled_rows():
    """Post-transition L-layer at the Wan-1.3B shapes: 4680 chunk queries
    over sink + current keys (6240), projected with a seeded weight standing
    in for W_new; 48 sampled rows (the last included) against the oracle."""
    w = synth.WORKLOADS["wan1.3b"]
    x = synth.single_layer_inputs(w, 1)
    W = synth.weight(w, 1)
    status = ispa.new_status()
    y, a_loc = ispa.local_attention_project(dev(x["q"], "bf16"),
                                            [(dev(x["k_sink"], "bf16"), dev(x["v_sink"], "bf16")),
                                             (dev(x["k_cur"], "bf16"), dev(x["v_cur"], "bf16"))],
                                            dev(W, "bf16"), w.n_heads, status=status)
    torch.cuda.synchronize()
    ispa.raise_on_status(status, "local_attention_project")
    rows = np.sort(np.random.default_rng(6).choice(w.n_q, 48, replace=False))
    rows[-1] = w.n_q - 1
    a_ref, _ = orc.attention(x["q"][rows], np.concatenate([x["k_sink"], x["k_cur"]]),
                             np.concatenate([x["v_sink"], x["v_cur"]]), w.n_heads)
    assert max_rel(host(a_loc)[rows], a_ref) <= ATTN_MAX_REL
    assert max_rel(host(y)[rows], orc.project(a_ref, W)) <= ATTN_MAX_REL


def _layer_outputs(w, chunk=1):
    x = synth.single_layer_inputs(w, chunk)
    status = ispa.new_status()
    out = ispa.dual_attention(dev(x["q"], "bf16"), [(dev(x["k_sink"], "bf16"), dev(x["v_sink"], "bf16")),
                                                   (dev(x["k_cur"], "bf16"), dev(x["v_cur"], "bf16"))],
                              [(dev(x["k_hist"], "bf16"), dev(x["v_hist"], "bf16"))], w.n_heads, status=status)
    torch.cuda.synchronize()
    ispa.raise_on_status(status, "dual_attention")
    return x, out


def _check_sampled_rows(w, x, out, n_rows, seed):
    rows = np.sort(np.random.default_rng(seed).choice(w.n_q, n_rows, replace=False))
    rows[-1] = w.n_q - 1
    got = {k: host(v) for k, v in out.items()}
    ref = orc.dual_stream(x["q"][rows], [(x["k_sink"], x["v_sink"]), (x["k_cur"], x["v_cur"])],
                          [(x["k_hist"], x["v_hist"])], w.n_heads)
    _check_dual(got, ref, rows=rows)


def _check_gram_entries(A, Dl, G, R, n_pairs, seed):
    """G[i, j] and R[i, j] at seeded (i, j), each an fp64 dot product over all
    rows.  The products of bf16 values are exact in fp32, so the only error is
    the fp32 summation: bounded here by GRAM_REL times the sum of |products|."""
    g = np.random.default_rng(seed)
    D = A.shape[1]
    ii, jj = g.integers(0, D, n_pairs), g.integers(0, D, n_pairs)
    ii, jj = np.maximum(ii, jj), np.minimum(ii, jj)  # G: lower triangle; R: any entry
    Ah = A.float().cpu().numpy().astype(np.float64)
    Dh = Dl.float().cpu().numpy().astype(np.float64)
    Gh, Rh = G.cpu().numpy(), R.cpu().numpy()
    for i, j in zip(ii, jj):
        pg, pr = Ah[:, i] * Ah[:, j], Ah[:, i] * Dh[:, j]
        assert abs(Gh[i, j] - pg.sum()) <= GRAM_REL * np.abs(pg).sum() + 1e-30
        assert abs(Rh[i, j] - pr.sum()) <= GRAM_REL * np.abs(pr).sum() + 1e-30


def test_long_history_layer_sampled_rows_and_gram():
    """Long-history stress: 93600 history tokens (60 latent frames); 128 query
    rows against the oracle, and the statistics accumulated over 93600 rows
    checked entry by entry."""
    w = synth.WORKLOADS["long_hist"]
    x, out = _layer_outputs(w)
    _check_sampled_rows(w, x, out, 128, 21)
    # statistics over 93600 rows: 20 chunks' worth of (A_loc, delta) rows
    g = np.random.default_rng(22)
    n = 93600
    A = dev(synth.round_bf16((g.standard_normal((n, w.d_model)) * 0.2).astype(np.float32)), "bf16")
    Dl = dev(synth.round_bf16((g.standard_normal((n, w.d_model)) * 0.05).astype(np.float32)), "bf16")
    G = torch.empty(w.d_model, w.d_model, device="cuda")
    R = torch.empty(w.d_model, w.d_model, device="cuda")
    ispa.gram_accumulate(A, Dl, G, R, zero_first=True)
    torch.cuda.synchronize()
    _check_gram_entries(A, Dl, G, R, 64, 23)


def test_history_200k_dual_and_single_pass_sampled_rows():
    """A long-lived F-layer: 201240 history tokens (129 latent frames), 1572
    key tiles per query tile.  64 query rows of the dual-stream outputs and of
    the single-pass (F-layer) outputs against the oracle."""
    w = synth.WORKLOADS["hist_200k"]
    x, out = _layer_outputs(w)
    _check_sampled_rows(w, x, out, 64, 41)
    status = ispa.new_status()
    full = ispa.dual_attention(dev(x["q"], "bf16"), [(dev(x["k_sink"], "bf16"), dev(x["v_sink"], "bf16")),
                                                    (dev(x["k_cur"], "bf16"), dev(x["v_cur"], "bf16"))],
                               [(dev(x["k_hist"], "bf16"), dev(x["v_hist"], "bf16"))], w.n_heads, dual=False,
                               status=status)
    torch.cuda.synchronize()
    ispa.raise_on_status(status, "dual_attention")
    # the single pass computes exactly the dual stream's fused A_full
    rows = np.sort(np.random.default_rng(42).choice(w.n_q, 64, replace=False))
    ref = orc.dual_stream(x["q"][rows], [(x["k_sink"], x["v_sink"]), (x["k_cur"], x["v_cur"])],
                          [(x["k_hist"], x["v_hist"])], w.n_heads)
    assert max_rel(host(full["a_full"])[rows], ref["a_full"]) <= ATTN_MAX_REL
    assert max_abs(host(full["lse_full"])[:, rows], ref["lse_full"]) <= LSE_ABS


def test_wan14b_layer_sampled_rows_statistics_and_absorb():
    """Wan-14B-shaped layer (40 heads, D = 5120):
    - sampled attention rows against the oracle;
    - the statistics of 18720 seeded bf16 rows, entry by entry;
    - the 5120 x 5120 absorb solve against the oracle's solve of the oracle's
      G, R of the same rows."""
    w = synth.WORKLOADS["wan14b"]
    x, out = _layer_outputs(w)
    _check_sampled_rows(w, x, out, 48, 31)
    del out
    D = w.d_model
    n = w.warm_chunks * w.n_q  # 18720 warm-up rows
    A, Dl, W = _absorb_case(31, n, D, "bf16")
    G = torch.empty(D, D, device="cuda")
    R = torch.empty(D, D, device="cuda")
    Ad, Dd = dev(A, "bf16"), dev(Dl, "bf16")
    for c in range(w.warm_chunks):  # accumulated chunk by chunk, as in the warm-up
        rows = slice(c * w.n_q, (c + 1) * w.n_q)
        ispa.gram_accumulate(Ad[rows], Dd[rows], G, R, zero_first=(c == 0))
    torch.cuda.synchronize()
    _check_gram_entries(Ad, Dd, G, R, 32, 32)
    status = ispa.new_status()
    dW, Wn = ispa.absorb_solve(G, R, dev(W, "bf16"), lambda_rel=orc.LAMBDA_REL, status=status)
    torch.cuda.synchronize()
    ispa.raise_on_status(status, "absorb_solve")
    Gr, Rr = orc.gram(A, Dl)
    dW_ref = orc.absorb(Gr, Rr, W, orc.ridge_lambda(Gr))
    assert fro_rel(host(dW), dW_ref) <= DW_REL_BF16

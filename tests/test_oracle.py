"""Pins for the fp64 oracle: checks against what the ISPA pages and the
mathematics fix, never against the oracle's own formulas retyped.

Attention / LSE [gist §2.1]: a library attention routine (torch SDPA, fp64),
scipy's logsumexp, closed forms (two keys, one key, uniform scores, constant
values) and key-permutation invariance; the local + history merge must equal
single-pass attention over the concatenated keys.

Absorb [gist §2.2]: brute-force minimisation of the stated objective (an
augmented least-squares problem solved by SVD, gradient descent, random
perturbations), the scalar closed form, dW = 0 when A_full = A_loc, dW -> 0 as
lambda grows, ordinary least squares at lambda = 0, scipy's Cholesky solve.

Bookkeeping [gist §2.3, abstract]: closed-form token ranges and KV bytes.
"""
import math

import numpy as np
import pytest
import scipy.linalg
import scipy.special
import torch

from oracle import ispa_oracle as orc
from ar_video_diffusion_b200 import synth


def _rand(seed, *shape, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# ------------------------------------------------------------------ attention
@pytest.mark.parametrize("H,d,nq,nk", [(2, 64, 37, 81), (3, 16, 5, 1), (1, 128, 9, 300)])
def test_attention_matches_torch_sdpa(H, d, nq, nk):
    q, k, v = _rand(1, nq, H * d), _rand(2, nk, H * d, scale=1.5), _rand(3, nk, H * d)
    o, lse = orc.attention(q, k, v, H, row_block=7)
    tq = torch.from_numpy(q).view(nq, H, d).transpose(0, 1)[None]
    tk = torch.from_numpy(k).view(nk, H, d).transpose(0, 1)[None]
    tv = torch.from_numpy(v).view(nk, H, d).transpose(0, 1)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)[0]  # [H, nq, d]
    ref = ref.transpose(0, 1).reshape(nq, H * d).numpy()
    assert np.max(np.abs(o - ref)) <= 1e-12
    # LSE through scipy's logsumexp of the scaled scores (natural log)
    for h in range(H):
        S = (q[:, h * d:(h + 1) * d] @ k[:, h * d:(h + 1) * d].T) / math.sqrt(d)
        assert np.max(np.abs(lse[h] - scipy.special.logsumexp(S, axis=1))) <= 1e-12


def test_attention_two_keys_closed_form():
    # d = 4, scale = 1/2: s1 = <q,k1>/2 = 1, s2 = 0
    q = np.array([[1.0, 0, 0, 0]])
    k = np.array([[2.0, 0, 0, 0], [0, 0, 0, 0]])
    v = np.array([[1.0, 0, 0, 0], [0, 1.0, 0, 0]])
    o, lse = orc.attention(q, k, v, 1)
    e = math.e
    assert np.allclose(o[0], [e / (e + 1), 1 / (e + 1), 0, 0], rtol=0, atol=1e-15)
    assert abs(lse[0, 0] - math.log(e + 1)) < 1e-15


def test_attention_single_key_and_uniform_and_constant():
    H, d = 2, 8
    q, k1, v1 = _rand(4, 6, H * d), _rand(5, 1, H * d), _rand(6, 1, H * d)
    o, lse = orc.attention(q, k1, v1, H)
    assert np.allclose(o, np.repeat(v1, 6, 0), atol=1e-15)
    for h in range(H):
        s = (q[:, h * d:(h + 1) * d] @ k1[0, h * d:(h + 1) * d]) / math.sqrt(d)
        assert np.allclose(lse[h], s, atol=1e-14)
    # all scores equal (K = 0): mean of V, LSE = log n_k
    n_k = 13
    v = _rand(7, n_k, H * d)
    o, lse = orc.attention(q, np.zeros((n_k, H * d)), v, H)
    assert np.allclose(o, np.repeat(v.mean(0, keepdims=True), 6, 0), atol=1e-14)
    assert np.allclose(lse, math.log(n_k), atol=1e-14)
    # constant value rows: output is that constant whatever the scores
    c = _rand(8, 1, H * d)
    o, _ = orc.attention(q, _rand(9, n_k, H * d, scale=3.0), np.repeat(c, n_k, 0), H)
    assert np.allclose(o, np.repeat(c, 6, 0), atol=1e-13)


def test_attention_key_permutation_invariance():
    H, d = 2, 16
    q, k, v = _rand(10, 11, H * d), _rand(11, 40, H * d), _rand(12, 40, H * d)
    p = np.random.default_rng(13).permutation(40)
    o1, l1 = orc.attention(q, k, v, H)
    o2, l2 = orc.attention(q, k[p], v[p], H)
    assert np.max(np.abs(o1 - o2)) < 1e-13 and np.max(np.abs(l1 - l2)) < 1e-13


def test_attention_empty_keys():
    o, lse = orc.attention(_rand(1, 3, 8), np.zeros((0, 8)), np.zeros((0, 8)), 2)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


def test_merge_equals_single_pass_full_attention():
    """[gist §2.1]: the local and historical branches fused through their LSE
    states reproduce attention over the whole context."""
    c = synth.random_case(21, n_q=29, n_heads=3, head_dim=32, seg_tokens=[16, 50, 120], dtype="f32")
    (ks, vs), (kc, vc), (kh, vh) = c["segments"]
    r = orc.dual_stream(c["q"], [(ks, vs), (kc, vc)], [(kh, vh)], 3)
    a_full, delta, L = orc.lse_merge(r["a_loc"], r["lse_loc"], r["o_hist"], r["lse_hist"], 3)
    assert np.max(np.abs(a_full - r["a_full"])) < 1e-12
    assert np.max(np.abs(L - r["lse_full"])) < 1e-12
    assert np.max(np.abs(delta - r["delta"])) < 1e-12


def test_merge_with_empty_history_is_identity():
    c = synth.random_case(22, n_q=7, n_heads=2, head_dim=16, seg_tokens=[10, 20], dtype="f32")
    (ks, vs), (kc, vc) = c["segments"]
    r = orc.dual_stream(c["q"], [(ks, vs), (kc, vc)], [], 2)
    assert np.all(np.isneginf(r["lse_hist"]))
    a_full, delta, L = orc.lse_merge(r["a_loc"], r["lse_loc"], r["o_hist"], r["lse_hist"], 2)
    assert np.array_equal(a_full, r["a_loc"]) and np.all(delta == 0)
    assert np.array_equal(L, r["lse_loc"])
    assert np.max(np.abs(r["a_full"] - r["a_loc"])) == 0


def test_merge_of_two_empty_branches_is_attention_over_no_keys():
    """A row whose local and historical branches are both empty: the merge
    must give what attention over the (empty) union gives -- o = 0 and
    LSE = -inf -- with no NaN; rows with a non-empty branch are unaffected."""
    H, d, n = 2, 8, 5
    c = synth.random_case(23, n_q=n, n_heads=H, head_dim=d, seg_tokens=[9, 14], dtype="f32")
    (kl, vl), (kh, vh) = c["segments"]
    o_l, l_l = orc.attention(c["q"], kl, vl, H)
    o_h, l_h = orc.attention(c["q"], kh, vh, H)
    o_e, l_e = orc.attention(c["q"], np.zeros((0, H * d)), np.zeros((0, H * d)), H)
    # rows 1 and 3 lose both branches for head 0; row 4 keeps only its history for head 1
    for r in (1, 3):
        o_l[r, :d], l_l[0, r] = o_e[r, :d], l_e[0, r]
        o_h[r, :d], l_h[0, r] = o_e[r, :d], l_e[0, r]
    o_l[4, d:], l_l[1, 4] = 0.0, -np.inf
    a_full, delta, L = orc.lse_merge(o_l, l_l, o_h, l_h, H)
    assert not np.any(np.isnan(a_full)) and not np.any(np.isnan(delta)) and not np.any(np.isnan(L))
    for r in (1, 3):
        assert np.all(a_full[r, :d] == o_e[r, :d]) and np.isneginf(L[0, r]) and np.isneginf(l_e[0, r])
    assert np.array_equal(a_full[4, d:], o_h[4, d:]) and L[1, 4] == l_h[1, 4]
    ref, _, Lref = orc.lse_merge(orc.attention(c["q"], kl, vl, H)[0], orc.attention(c["q"], kl, vl, H)[1],
                                 orc.attention(c["q"], kh, vh, H)[0], orc.attention(c["q"], kh, vh, H)[1], H)
    keep = [0, 2]
    assert np.array_equal(a_full[keep], ref[keep]) and np.array_equal(L[:, keep], Lref[:, keep])


# ---------------------------------------------------------------------- absorb
def _ridge_case(seed, N, D, Dout=None):
    Dout = D if Dout is None else Dout
    a_loc = _rand(seed, N, D)
    a_full = a_loc + 0.3 * _rand(seed + 1, N, D)
    W = _rand(seed + 2, D, Dout) / math.sqrt(D)
    return a_loc, a_full, W


def test_gram_bruteforce_loops():
    a_loc, a_full, _ = _ridge_case(30, 6, 4)
    G, R = orc.gram(a_loc, a_full - a_loc)
    for i in range(4):
        for j in range(4):
            g = sum(a_loc[n, i] * a_loc[n, j] for n in range(6))
            r = sum(a_loc[n, i] * (a_full[n, j] - a_loc[n, j]) for n in range(6))
            assert abs(G[i, j] - g) < 1e-13 and abs(R[i, j] - r) < 1e-13


def test_gram_is_additive_over_chunks():
    a_loc, a_full, _ = _ridge_case(31, 40, 5)
    G, R = orc.gram(a_loc, a_full - a_loc)
    G1, R1 = orc.gram(a_loc[:17], (a_full - a_loc)[:17])
    G2, R2 = orc.gram(a_loc[17:], (a_full - a_loc)[17:])
    assert np.allclose(G, G1 + G2, atol=1e-12) and np.allclose(R, R1 + R2, atol=1e-12)


@pytest.mark.parametrize("N,D", [(32, 8), (5, 8), (64, 3)])
def test_absorb_matches_bruteforce_lstsq(N, D):
    """Stacking [A_loc; sqrt(lam) I] dW = [(A_full - A_loc) W; 0] turns the
    objective of [gist §2.2] into one least-squares problem, solved here by
    SVD -- a route that never forms the normal equations."""
    a_loc, a_full, W = _ridge_case(40 + N, N, D, Dout=D + 2)
    G, R = orc.gram(a_loc, a_full - a_loc)
    lam = orc.ridge_lambda(G)
    dW = orc.absorb(G, R, W, lam)
    A = np.vstack([a_loc, math.sqrt(lam) * np.eye(D)])
    B = np.vstack([(a_full - a_loc) @ W, np.zeros((D, W.shape[1]))])
    ref = np.linalg.lstsq(A, B, rcond=None)[0]
    assert np.linalg.norm(dW - ref) <= 1e-10 * np.linalg.norm(ref)


def test_absorb_minimises_objective_gradient_descent_and_perturbation():
    a_loc, a_full, W = _ridge_case(50, 32, 8)
    G, R = orc.gram(a_loc, a_full - a_loc)
    lam = orc.ridge_lambda(G)
    dW = orc.absorb(G, R, W, lam)
    # gradient descent on the objective itself (step from its Lipschitz bound)
    X = np.zeros_like(W)
    step = 1.0 / (2 * (np.linalg.norm(a_loc, 2) ** 2 + lam))
    for _ in range(4000):
        grad = 2 * a_loc.T @ (a_loc @ (W + X) - a_full @ W) + 2 * lam * X
        X -= step * grad
    assert np.linalg.norm(X - dW) <= 1e-8 * np.linalg.norm(dW)
    f0 = orc.objective(a_loc, a_full, W, dW, lam)
    g = np.random.default_rng(51)
    for _ in range(20):
        E = g.standard_normal(W.shape)
        assert orc.objective(a_loc, a_full, W, dW + 1e-3 * E, lam) > f0


def test_absorb_scalar_closed_form():
    # D = 1: dW = w * sum a_l (a_f - a_l) / (sum a_l^2 + lam)
    a_l = np.array([[1.0], [2.0], [-1.0]])
    a_f = np.array([[1.5], [1.0], [0.0]])
    w, lam = 0.7, 0.25
    dW = orc.absorb(*orc.gram(a_l, a_f - a_l), np.array([[w]]), lam)
    num = 1 * 0.5 + 2 * (-1.0) + (-1) * 1.0
    den = 1 + 4 + 1 + lam
    assert abs(dW[0, 0] - w * num / den) < 1e-15


def test_absorb_zero_when_streams_agree():
    a_loc, _, W = _ridge_case(60, 20, 6)
    G, R = orc.gram(a_loc, a_loc - a_loc)
    assert np.all(R == 0)
    assert np.all(orc.absorb(G, R, W, orc.ridge_lambda(G)) == 0)


def test_absorb_vanishes_as_lambda_grows():
    a_loc, a_full, W = _ridge_case(61, 40, 6)
    G, R = orc.gram(a_loc, a_full - a_loc)
    base = np.trace(G) / 6
    RW = R @ W
    norms = []
    for t in [1e3, 1e5, 1e7, 1e9]:
        lam = t * base
        dW = orc.absorb(G, R, W, lam)
        norms.append(np.linalg.norm(dW))
        # lam * dW -> R W with error O(||G|| / lam)
        assert np.linalg.norm(lam * dW - RW) <= 10 * np.linalg.norm(G, 2) / lam * np.linalg.norm(RW)
    assert all(n2 < n1 for n1, n2 in zip(norms, norms[1:]))
    # ||dW|| falls like 1/lambda: six decades of lambda, six decades of norm
    assert 0.5e-6 * norms[0] <= norms[-1] <= 2e-6 * norms[0]


def test_absorb_normal_equation_residual_and_cholesky():
    a_loc, a_full, W = _ridge_case(62, 200, 24)
    G, R = orc.gram(a_loc, a_full - a_loc)
    lam = orc.ridge_lambda(G)
    dW = orc.absorb(G, R, W, lam)
    res = (G + lam * np.eye(24)) @ dW - R @ W
    assert np.linalg.norm(res) <= 1e-12 * np.linalg.norm(R @ W)
    ref = scipy.linalg.cho_solve(scipy.linalg.cho_factor(G + lam * np.eye(24)), R @ W)
    assert np.linalg.norm(dW - ref) <= 1e-12 * np.linalg.norm(ref)


def test_absorb_ols_at_lambda_zero():
    a_loc, a_full, W = _ridge_case(63, 50, 7)
    G, R = orc.gram(a_loc, a_full - a_loc)
    dW = orc.absorb(G, R, W, 0.0)
    ref = np.linalg.lstsq(a_loc, (a_full - a_loc) @ W, rcond=None)[0]
    assert np.linalg.norm(dW - ref) <= 1e-10 * np.linalg.norm(ref)


def test_ridge_lambda_hand_values():
    """lambda = 1e-2 * trace(G) / D, the value every benchmark configuration
    states ("lambda = 1e-2 * trace(G) / D"; the pages give none), on values
    worked out by hand.  A wrong divisor (the row count N instead of D), a
    wrong constant or a missing lambda_abs term fails one of them."""
    # G = diag(1, 2, 3, 4): trace 10, D = 4 -> 1e-2 * 10 / 4
    assert orc.ridge_lambda(np.diag([1.0, 2.0, 3.0, 4.0])) == pytest.approx(0.025, rel=1e-15)
    # G = A^T A with A 7 x 4 (N = 7 rows != D = 4): trace(G) = sum of A's
    # squares = 1 + 4 + 9 + 4 + 0 + 16 + 1 = 35 -> 1e-2 * 35 / 4 = 0.0875 (N in
    # the divisor would give 0.05)
    A = np.array([[1.0, 0, 0, 0], [0, 2, 0, 0], [0, 0, 0, 3], [1, 1, 1, 1], [0, 0, 0, 0], [0, 0, 4, 0],
                  [0, 0, 0, 1]])
    assert np.sum(A * A) == 35
    assert orc.ridge_lambda(A.T @ A) == pytest.approx(0.0875, rel=1e-15)
    # off-diagonal entries do not enter; lambda_abs adds, lambda_rel scales
    G = np.array([[2.0, -7.0], [-7.0, 6.0]])  # trace 8, D = 2
    assert orc.ridge_lambda(G) == pytest.approx(0.04, rel=1e-15)
    assert orc.ridge_lambda(G, lambda_rel=0.5, lambda_abs=0.25) == pytest.approx(0.25 + 0.5 * 8 / 2, rel=1e-15)
    assert orc.LAMBDA_REL == 1e-2


def test_lambda_reading_is_normalisation_invariant():
    a_loc, a_full, W = _ridge_case(64, 30, 5)
    G, R = orc.gram(a_loc, a_full - a_loc)
    dW1 = orc.absorb(G, R, W, orc.ridge_lambda(G))
    dW2 = orc.absorb(G / 30, R / 30, W, orc.ridge_lambda(G / 30))
    assert np.linalg.norm(dW1 - dW2) <= 1e-12 * np.linalg.norm(dW1)


def test_modulated_weight_reconstructs_full_stream_exactly_when_possible():
    # If A_full = A_loc M for some M, lam -> 0 gives A_loc (W + dW) = A_full W.
    a_loc = _rand(70, 60, 6)
    M = np.eye(6) + 0.2 * _rand(71, 6, 6)
    a_full = a_loc @ M
    W = _rand(72, 6, 6)
    G, R = orc.gram(a_loc, a_full - a_loc)
    W_new = orc.modulated_weight(W, orc.absorb(G, R, W, 0.0))
    assert np.max(np.abs(orc.project(a_loc, W_new) - orc.project(a_full, W))) < 1e-10


# ------------------------------------------------------- layer selection
def test_reconstruction_error_zero_when_streams_agree():
    a_loc, _, W = _ridge_case(80, 30, 5)
    G, R = orc.gram(a_loc, a_loc - a_loc)
    dW = orc.absorb(G, R, W, orc.ridge_lambda(G))
    assert orc.reconstruction_error(a_loc, a_loc, W, dW) == 0.0


def test_reconstruction_error_vanishes_for_exact_linear_history():
    # A_full = A_loc M: lam -> 0 absorbs the history exactly
    a_loc = _rand(81, 80, 6)
    a_full = a_loc @ (np.eye(6) + 0.3 * _rand(82, 6, 6))
    W = _rand(83, 6, 6)
    G, R = orc.gram(a_loc, a_full - a_loc)
    assert orc.reconstruction_error(a_loc, a_full, W, orc.absorb(G, R, W, 0.0)) < 1e-20


def test_reconstruction_error_scalar_closed_form():
    # D = 1, hand-evaluated: dW from the scalar ridge formula, then the ratio
    a_l = np.array([[1.0], [2.0], [-1.0]])
    a_f = np.array([[1.5], [1.0], [0.0]])
    w, lam = 0.7, 0.25
    dw = w * (1 * 0.5 + 2 * (-1.0) + (-1) * 1.0) / (1 + 4 + 1 + lam)
    num = sum((al * (w + dw) - af * w) ** 2 for al, af in [(1.0, 1.5), (2.0, 1.0), (-1.0, 0.0)])
    den = sum((af * w) ** 2 for af in (1.5, 1.0, 0.0))
    got = orc.reconstruction_error(a_l, a_f, np.array([[w]]), np.array([[dw]]))
    assert abs(got - num / den) < 1e-14


def test_reconstruction_error_limits_and_invariance():
    a_loc, a_full, W = _ridge_case(84, 50, 6)
    G, R = orc.gram(a_loc, a_full - a_loc)
    # lam -> inf: dW -> 0, the error tends to ||dA W||^2 / ||A_full W||^2
    e_inf = orc.reconstruction_error(a_loc, a_full, W, orc.absorb(G, R, W, 1e12 * np.trace(G)))
    d = (a_full - a_loc) @ W
    t = a_full @ W
    assert abs(e_inf - np.sum(d * d) / np.sum(t * t)) < 1e-9
    # the ridge minimiser can only lower the error term against dW = 0 as lam -> 0
    e0 = orc.reconstruction_error(a_loc, a_full, W, orc.absorb(G, R, W, 0.0))
    assert e0 <= e_inf
    # scaling W scales dW and both norms alike
    lam = orc.ridge_lambda(G)
    e1 = orc.reconstruction_error(a_loc, a_full, W, orc.absorb(G, R, W, lam))
    e3 = orc.reconstruction_error(a_loc, a_full, 3.0 * W, orc.absorb(G, R, 3.0 * W, lam))
    assert abs(e1 - e3) < 1e-12 * max(1.0, e1)


def test_reconstruction_error_from_statistics():
    # the closed form the GPU evaluates: with E = dA^T dA,
    # num = <dW, G dW> - 2 <dW, R W> + <W, E W>, den = <W, (G + R + R^T + E) W>
    a_loc, a_full, W = _ridge_case(85, 64, 7, 5)
    dA = a_full - a_loc
    G, R = orc.gram(a_loc, dA)
    E = dA.T @ dA
    dW = orc.absorb(G, R, W, orc.ridge_lambda(G))
    num = np.sum(dW * (G @ dW)) - 2 * np.sum(dW * (R @ W)) + np.sum(W * (E @ W))
    den = np.sum(W * ((G + R + R.T + E) @ W))
    assert abs(orc.reconstruction_error(a_loc, a_full, W, dW) - num / den) < 1e-12


def test_select_layers_bruteforce_with_ties():
    import itertools
    rng = np.random.default_rng(86)
    for trial in range(40):
        n = int(rng.integers(1, 8))
        eps = list(rng.choice([0.1, 0.2, 0.3, 0.5], size=n))  # many ties
        if trial % 5 == 0 and n > 1:
            eps[int(rng.integers(n))] = float("nan")
        for k in range(n + 1):
            def key(sub):
                vals = [math.inf if math.isnan(eps[l]) else eps[l] for l in sub]
                return (sum(math.isnan(eps[l]) for l in sub), sorted(vals), list(sub))
            best = min(itertools.combinations(range(n), k), key=key)
            assert orc.select_layers(eps, k) == list(best), (eps, k)
    with pytest.raises(ValueError):
        orc.select_layers([0.1, 0.2], 3)


# ---------------------------------------------------------------- bookkeeping
def test_chunk_token_ranges_closed_form():
    F, cf = 1560, 3
    assert orc.chunk_token_ranges(0, F, cf) == {"sink": (0, 0), "hist": (0, 0), "cur": (0, 4680)}
    assert orc.chunk_token_ranges(1, F, cf) == {"sink": (0, 1560), "hist": (1560, 4680),
                                                "cur": (4680, 9360)}
    r = orc.chunk_token_ranges(23, F, cf)
    assert r == {"sink": (0, 1560), "hist": (1560, 23 * 4680), "cur": (23 * 4680, 24 * 4680)}


def test_kv_bytes_rollout_closed_form():
    """30 layers, 1.3B shapes, even layers absorbed; at the last of 24 chunks
    every F-layer holds 72 latent frames, every L-layer sink + current."""
    mask = orc.layer_mask(30, range(0, 30, 2))
    assert mask == 0x15555555
    per_tok = 2 * 1536 * 2
    all_f = orc.kv_bytes(23, 30, 0, True, 1560, 3, 1536, 2)
    ispa = orc.kv_bytes(23, 30, mask, True, 1560, 3, 1536, 2)
    assert all_f == 30 * 112320 * per_tok == 20_702_822_400
    assert ispa == 15 * 112320 * per_tok + 15 * 6240 * per_tok
    assert abs(1 - ispa / all_f - 0.4722222) < 1e-6
    # before the transition the mask does not evict anything
    assert orc.kv_bytes(3, 30, mask, False, 1560, 3, 1536, 2) == orc.kv_bytes(3, 30, 0, False, 1560, 3, 1536, 2)


def test_synth_bf16_rounding_is_rne():
    x = np.array([1.0, 1.00390625, 1.005859375, 1.0078125, -2.5e-3, 3.0e38], np.float32)
    r = synth.round_bf16(x)
    t = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(r, t)
    y = np.random.default_rng(3).standard_normal(10000).astype(np.float32) * 7
    assert np.array_equal(synth.round_bf16(y), torch.from_numpy(y).to(torch.bfloat16).float().numpy())


def _pages_claims():
    """tests/golden/pages_claims.txt: key = value lines (the comments cite the pages)."""
    import os
    vals = {}
    with open(os.path.join(os.path.dirname(__file__), "golden", "pages_claims.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = (x.strip() for x in line.split("="))
                vals[k] = float(v)
    return vals


def test_kv_removal_approaches_but_never_exceeds_the_pages_bound():
    """Half the layers absorbed: the KV fraction removed grows with the video
    and tends to the pages' "up to 50%" without reaching it (an L-layer keeps
    the sink and the current chunk)."""
    claims = _pages_claims()
    L = 30
    K = int(claims["l_layers_fraction"] * L)
    mask = orc.layer_mask(L, range(0, L, 2))
    assert bin(mask).count("1") == K
    prev = 0.0
    for c in (4, 8, 23, 100, 1000, 10000):
        all_f = orc.kv_bytes(c, L, 0, True, 1560, 3, 1536, 2)
        removed = 1 - orc.kv_bytes(c, L, mask, True, 1560, 3, 1536, 2) / all_f
        assert prev < removed < claims["kv_removed_upper_bound"]
        prev = removed
    # closed form: 1/2 * (1 - (sink + chunk) / (frames up to chunk c))
    c = 10000
    frames = 3 * (c + 1)
    assert abs(prev - 0.5 * (1 - (1 + 3) / frames)) < 1e-12
    assert claims["kv_removed_upper_bound"] - prev < 1e-3


def test_warm_up_reading_meets_the_pages_minimum():
    """The primary reading's warm-up is 4 chunks of 3 latent frames = 12
    frames, the pages' sufficient minimum, giving 18720 statistics rows per
    layer at 1560 tokens per frame."""
    claims = _pages_claims()
    from ar_video_diffusion_b200 import synth
    w = synth.WORKLOADS["wan1.3b"]
    assert w.warm_chunks * w.chunk_frames == claims["t_warm_frames_min"]
    assert w.warm_chunks * w.n_q == 18720

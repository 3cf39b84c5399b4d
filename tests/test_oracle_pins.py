"""Pins of the CPU oracle to things other than itself.

Each test checks an oracle function against a closed form, an invariant of the
mathematics, an independent formulation built from library routines, brute
force on tiny inputs, or central finite differences.  The mutation tests at the
end plant plausible mistakes in the oracle (on the CPU) and confirm that these
pins catch them.
"""
import itertools
import math
import json
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import slora_oracle as O
from contextual_sparsity_lora_svd_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def tsilu(x):
    """torch's SiLU on a float64 numpy array (an independent implementation)."""
    return torch.nn.functional.silu(torch.from_numpy(x)).numpy()


def colnorm(x):
    return torch.linalg.vector_norm(torch.from_numpy(x), dim=0).numpy()


# --------------------------------------------------------------------------- SVD
@pytest.mark.parametrize("n,k,r", [(40, 24, 5), (24, 40, 8), (30, 30, 1)])
def test_svd_prepare_closed_form(n, k, r):
    sw = synth.decaying_weight(n, k, seed=7)
    L, U = O.svd_prepare(sw.W, r)
    # rank-r product equals the construction's leading triplets exactly
    Wr = (sw.U[:, :r] * sw.s[None, :r]) @ sw.V[:, :r].T
    np.testing.assert_allclose(U @ L.T, Wr, atol=1e-12 * np.abs(sw.W).max())
    # L = V_r Sigma_r: column norms are the singular values
    np.testing.assert_allclose(np.linalg.norm(L, axis=0), sw.s[:r], rtol=1e-12)
    # U has orthonormal columns
    np.testing.assert_allclose(U.T @ U, np.eye(r), atol=1e-12)
    # Eckart-Young: residual energy is the tail of the spectrum
    res = np.sum((sw.W - U @ L.T) ** 2)
    np.testing.assert_allclose(res, np.sum(sw.s[r:] ** 2), rtol=1e-10)


def test_decaying_weight_rms_and_spectrum():
    sw = synth.decaying_weight(64, 48, seed=3)
    assert abs(np.sqrt(np.mean(sw.W ** 2)) - 0.02) < 1e-12
    sv = np.linalg.svd(sw.W, compute_uv=False)
    np.testing.assert_allclose(sv, sw.c * np.arange(1, 49) ** -0.7, rtol=1e-10)


# ---------------------------------------------------------------------- scores
def _full_rank_factors(W):
    m = min(W.shape)
    return O.svd_prepare(W, m)


def test_ffn_score_full_rank_equals_exact_activation_norm():
    """With r = min(n, k) the estimate is exact, so the score is the true
    SwiGLU activation norm over context tokens (computed with torch here)."""
    tok = synth.Tokens(batch=3, seq=7, ctx_len=np.array([5, 7, 2], np.int32))
    d, d_ff = 12, 18
    X = synth.gaussian((tok.T, d), 1.0, 11)
    Wg = synth.decaying_weight(d_ff, d, 12).W * 20
    Wu = synth.decaying_weight(d_ff, d, 13).W * 20
    Lg, Ug = _full_rank_factors(Wg)
    Lu, Uu = _full_rank_factors(Wu)
    C, _ = O.context_rows(tok.batch, tok.seq, tok.ctx_len)
    got = O.ffn_scores(O.project(X[C], Lg), O.project(X[C], Lu), Ug, Uu)
    exact = colnorm(tsilu(X[C] @ Wg.T) * (X[C] @ Wu.T))
    np.testing.assert_allclose(got, exact, rtol=1e-11)


def test_ffn_score_rank_r_matches_factor_estimate():
    """At rank r the score is the activation norm of the rank-r weights."""
    tok = synth.Tokens.uniform(2, 8)
    d, d_ff, r = 16, 20, 3
    X = synth.gaussian((tok.T, d), 1.0, 21)
    swg = synth.decaying_weight(d_ff, d, 22)
    swu = synth.decaying_weight(d_ff, d, 23)
    Lg, Ug = O.svd_prepare(swg.W, r)
    Lu, Uu = O.svd_prepare(swu.W, r)
    C, _ = O.context_rows(tok.batch, tok.seq, tok.ctx_len)
    Wg_r = (swg.U[:, :r] * swg.s[:r]) @ swg.V[:, :r].T
    Wu_r = (swu.U[:, :r] * swu.s[:r]) @ swu.V[:, :r].T
    exact = colnorm(tsilu(X[C] @ Wg_r.T) * (X[C] @ Wu_r.T))
    got = O.ffn_scores(O.project(X[C], Lg), O.project(X[C], Lu), Ug, Uu)
    np.testing.assert_allclose(got, exact, rtol=1e-10)


def test_qk_score_full_rank_equals_exact_norm_product():
    tok = synth.Tokens(batch=2, seq=6, ctx_len=np.array([4, 3], np.int32))
    d, H, hd = 10, 2, 4
    X = synth.gaussian((tok.T, d), 1.0, 31)
    Wq = synth.decaying_weight(H * hd, d, 32).W
    Wk = synth.decaying_weight(H * hd, d, 33).W
    Lq, Uq = _full_rank_factors(Wq)
    Lk, Uk = _full_rank_factors(Wk)
    C, _ = O.context_rows(tok.batch, tok.seq, tok.ctx_len)
    got = O.qk_scores(O.project(X[C], Lq), O.project(X[C], Lk), Uq, Uk, H, H, hd)
    exact = (colnorm(X[C] @ Wq.T) * colnorm(X[C] @ Wk.T)).reshape(H, hd)
    np.testing.assert_allclose(got, exact, rtol=1e-11)


def test_qk_score_gram_identity():
    """||P U^T e_c||^2 = u_c^T (P^T P) u_c: the Gram form of the same score."""
    rg = synth.rng(5)
    P_q, P_k = rg.standard_normal((9, 3)), rg.standard_normal((9, 3))
    U_q, U_k = rg.standard_normal((8, 3)), rg.standard_normal((8, 3))
    Gq, Gk = P_q.T @ P_q, P_k.T @ P_k
    nq = np.sqrt(np.einsum("cr,rs,cs->c", U_q, Gq, U_q))
    nk = np.sqrt(np.einsum("cr,rs,cs->c", U_k, Gk, U_k))
    got = O.qk_scores(P_q, P_k, U_q, U_k, 2, 2, 4)
    np.testing.assert_allclose(got.ravel(), nq * nk, rtol=1e-12)


def test_ffn_gram_score_full_rank_exact_and_gram_form():
    """The Gram-computable FFN variant: at full rank it is the product of the
    exact column norms of X W_g^T and X W_u^T; each norm equals its r x r Gram
    quadratic form; and it is the one-head QK-norm of the gate/up factors (the
    GPU path runs this variant through the QK criterion with one head)."""
    tok = synth.Tokens(batch=2, seq=9, ctx_len=np.array([6, 8], np.int32))
    d, d_ff = 10, 14
    X = synth.gaussian((tok.T, d), 1.0, 41)
    Wg = synth.decaying_weight(d_ff, d, 42).W * 10
    Wu = synth.decaying_weight(d_ff, d, 43).W * 10
    Lg, Ug = _full_rank_factors(Wg)
    Lu, Uu = _full_rank_factors(Wu)
    C, _ = O.context_rows(tok.batch, tok.seq, tok.ctx_len)
    Pg, Pu = O.project(X[C], Lg), O.project(X[C], Lu)
    got = O.ffn_gram_scores(Pg, Pu, Ug, Uu)
    exact = colnorm(X[C] @ Wg.T) * colnorm(X[C] @ Wu.T)
    np.testing.assert_allclose(got, exact, rtol=1e-11)
    ng = np.sqrt(np.einsum("cr,rs,cs->c", Ug, Pg.T @ Pg, Ug))
    nu = np.sqrt(np.einsum("cr,rs,cs->c", Uu, Pu.T @ Pu, Uu))
    np.testing.assert_allclose(got, ng * nu, rtol=1e-11)
    np.testing.assert_allclose(got, O.qk_scores(Pg, Pu, Ug, Uu, 1, 1, d_ff)[0], rtol=1e-12)


def test_ffn_gram_score_bounds_activation_norm():
    """|silu(x)| <= |x| and ||a * b|| <= ||a|| ||b||: the Gram variant is an
    upper bound of the activation-norm score, channel by channel."""
    rg = synth.rng(44)
    for t, r, n in ((5, 3, 7), (40, 8, 33)):
        Pg, Pu = rg.standard_normal((t, r)), rg.standard_normal((t, r))
        Ug, Uu = rg.standard_normal((n, r)), rg.standard_normal((n, r))
        act = O.ffn_scores(Pg, Pu, Ug, Uu)
        gram = O.ffn_gram_scores(Pg, Pu, Ug, Uu)
        assert np.all(act <= gram * (1 + 1e-12))


def test_qk_gqa_equals_mha_on_replicated_keys():
    """A GQA group score equals the sum of MHA scores of its query heads when
    the shared key head is replicated once per query head."""
    rg = synth.rng(6)
    H, KV, hd, r, t = 4, 2, 3, 2, 7
    P_q, P_k = rg.standard_normal((t, r)), rg.standard_normal((t, r))
    U_q, U_k = rg.standard_normal((H * hd, r)), rg.standard_normal((KV * hd, r))
    gqa = O.qk_scores(P_q, P_k, U_q, U_k, H, KV, hd)
    U_k_rep = np.concatenate([U_k[(h // 2) * hd:(h // 2 + 1) * hd] for h in range(H)])
    mha = O.qk_scores(P_q, P_k, U_q, U_k_rep, H, H, hd)
    np.testing.assert_allclose(gqa, mha.reshape(KV, 2, hd).sum(axis=1), rtol=1e-12)


def test_hand_worked_scores_closed_form():
    """Two context tokens, rank 2, identity-like factors worked by hand:
    P = [[1,0],[0,2]], U = [[1,0],[0,1],[1,1]] for gate and up alike, so
    g_hat = u_hat = [[1,0,1],[0,2,2]] and act = g * sigmoid(g) * g.
    score_0 = sigma(1), score_1 = 4 sigma(2), score_2 = sqrt(sigma(1)^2 + 16 sigma(2)^2)."""
    P = np.array([[1.0, 0.0], [0.0, 2.0]])
    U = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]])
    s1 = 1.0 / (1.0 + math.exp(-1.0))
    s2 = 1.0 / (1.0 + math.exp(-2.0))
    want = [s1, 4 * s2, math.sqrt(s1 * s1 + 16 * s2 * s2)]
    got = O.ffn_scores(P, P, U, U)
    np.testing.assert_allclose(got, want, rtol=1e-15)
    assert O.topk_select(got, 2).tolist() == [1, 2]


def test_golden_regression_fixture():
    """Oracle outputs on a reduced workload-0 case, written by
    tests/golden/make_golden.py (which calls only the oracle): guards against
    unintended changes to the oracle's arithmetic."""
    from tests.golden.make_golden import compute
    with open(os.path.join(GOLDEN, "ffn_reduced_w0.json")) as f:
        g = json.load(f)
    cur = compute()
    assert cur["idx"] == g["idx"]
    for key in ("scores", "out_sum", "dX_sum", "grad_norms"):
        np.testing.assert_allclose(cur[key], g[key], rtol=1e-12)


# ------------------------------------------------------------------- selection
def _brute_force_topk(score, k):
    best = None
    for sub in itertools.combinations(range(len(score)), k):
        key = (sum(score[j] for j in sub), tuple(-j for j in sub))
        if best is None or key > best[0]:
            best = (key, sub)
    return list(best[1])


@pytest.mark.parametrize("seed", range(12))
def test_topk_brute_force_with_ties(seed):
    rg = synth.rng(100 + seed)
    N = int(rg.integers(1, 10))
    k = int(rg.integers(0, N + 1))
    score = rg.integers(0, 4, size=N).astype(float)   # integer scores: many exact ties
    got = O.topk_select(score, k).tolist()
    assert got == sorted(got)
    assert got == _brute_force_topk(score.tolist(), k)


def test_topk_separation_large():
    rg = synth.rng(9)
    score = rg.random(1000)
    idx = O.topk_select(score, 137)
    mask = np.zeros(1000, bool)
    mask[idx] = True
    assert mask.sum() == 137 and score[mask].min() >= score[~mask].max()


@pytest.mark.parametrize("N,s,k", [(688, 0.5, 344), (11008, 0.5, 5504), (128, 0.5, 64),
                                   (14336, 0.0, 14336), (14336, 0.3, 10036), (14336, 0.5, 7168),
                                   (14336, 0.7, 4301), (14336, 0.9, 1434), (7, 0.99, 1)])
def test_keep_count(N, s, k):
    assert O.keep_count(N, s) == k


def test_select_sparsity_zero_keeps_all():
    score = synth.rng(2).random(33)
    assert O.topk_select(score, O.keep_count(33, 0.0)).tolist() == list(range(33))


# ------------------------------------------------------ QK per-group selection
# A hand-built grouped-query case (4 query heads, 2 key heads, head_dim 4, one
# context token, d = rank = 1).  With X_C = [[1]] and L = [[1]] the estimate is
# Q_hat[0, c] = U_q[c, 0], so every channel norm is |U_q[c, 0]| and the scores
# below follow by hand:
#   group 0 (query heads 0, 1):  |K| = [1, 1, 1, 2],  sum|Q| = [4, 4, 3, 1.5]
#                                score = [4, 4, 3, 3]
#   group 1 (query heads 2, 3):  |K| = [2, 1, .5, 1], sum|Q| = [1, 3, 6, 2]
#                                score = [2, 3, 3, 2]
_QK_UQ = [[1, 4, 2, 0.5], [3, 0, 1, 1], [1, 1, 1, 1], [0, 2, 5, 1]]
_QK_UK = [[1, 1, 1, 2], [2, 1, 0.5, 1]]
# The second row is an output token with a huge value: it must not count.
_QK_X = np.array([[1.0], [1000.0]])
# (sparsity, expected idx_q, expected idx_k) written out literally:
#   s = 0.5 keeps 2 per group: group 0 {0, 1}; group 1 {1, 2}.
#   s = 0.25 keeps 3: group 0 {0, 1, 2} (the 3-3 tie goes to channel 2);
#   group 1 {0, 1, 2} (the 2-2 tie goes to channel 0).
#   s = 0 keeps all four channels of every head.
_QK_EXPECT = [
    (0.5, [0, 1, 4, 5, 9, 10, 13, 14], [0, 1, 5, 6]),
    (0.25, [0, 1, 2, 4, 5, 6, 8, 9, 10, 12, 13, 14], [0, 1, 2, 4, 5, 6]),
    (0.0, list(range(16)), list(range(8))),
]


def _qk_hand_case(estimator, s):
    U_q = np.array(_QK_UQ, dtype=float).reshape(16, 1)
    U_k = np.array(_QK_UK, dtype=float).reshape(8, 1)
    one = np.ones((1, 1))
    return estimator(_QK_X, 1, 2, [1], one, U_q, one, U_k, 4, 2, 4, s)


def _check_qk_hand_case(estimator):
    for s, want_q, want_k in _QK_EXPECT:
        idx_q, idx_k, k, scores = _qk_hand_case(estimator, s)
        assert k == len(want_k) // 2, (s, k)
        assert np.asarray(idx_q).tolist() == want_q, (s, np.asarray(idx_q).tolist())
        assert np.asarray(idx_k).tolist() == want_k, (s, np.asarray(idx_k).tolist())
    np.testing.assert_allclose(scores, [[4, 4, 3, 3], [2, 3, 3, 2]], rtol=1e-15)


def test_estimate_select_qk_hand_built_gqa_layout():
    """Literal idx_q / idx_k of the hand-built 4-query / 2-key-head case: each
    query head h takes its group's set (group h // 2) as h*4 + c, each key head
    g its own set as g*4 + c; ties go to the lower channel; the output token is
    ignored."""
    _check_qk_hand_case(O.estimate_select_qk)


def _brute_force_group_topk(row, k):
    return _brute_force_topk(list(row), k)


@pytest.mark.parametrize("seed", range(8))
def test_select_per_group_brute_force_with_ties(seed):
    """Every row of select_per_group is the brute-force best k-subset of that
    row (largest sum, then lowest indices), ascending."""
    rg = synth.rng(300 + seed)
    groups, N = int(rg.integers(1, 5)), int(rg.integers(1, 9))
    k = int(rg.integers(0, N + 1))
    scores = rg.integers(0, 3, size=(groups, N)).astype(float)
    got = O.select_per_group(scores, k)
    assert got.shape == (groups, k)
    for g in range(groups):
        assert got[g].tolist() == _brute_force_group_topk(scores[g], k)


def test_estimate_select_qk_matches_exact_norms_and_brute_force():
    """Full-rank factors on a random GQA case (3 groups of 2 query heads,
    head_dim 6): the scores equal the exact norm products of X_C W^T (torch
    column norms), and each group's set is the brute-force top-k of them."""
    rg = synth.rng(77)
    H, KV, hd, d = 6, 3, 6, 5
    tok = synth.Tokens(batch=2, seq=4, ctx_len=np.array([3, 2], np.int32))
    X = rg.standard_normal((tok.T, d))
    Wq, Wk = rg.standard_normal((H * hd, d)), rg.standard_normal((KV * hd, d))
    Lq, Uq = _full_rank_factors(Wq)
    Lk, Uk = _full_rank_factors(Wk)
    idx_q, idx_k, k, scores = O.estimate_select_qk(X, tok.batch, tok.seq, tok.ctx_len, Lq, Uq,
                                                   Lk, Uk, H, KV, hd, 0.5)
    Xc = X[[0, 1, 2, 4, 5]]
    nq = colnorm(Xc @ Wq.T).reshape(H, hd)
    nk = colnorm(Xc @ Wk.T).reshape(KV, hd)
    want = np.stack([nk[g] * (nq[2 * g] + nq[2 * g + 1]) for g in range(KV)])
    np.testing.assert_allclose(scores, want, rtol=1e-10)
    assert k == 3
    for g in range(KV):
        sel = _brute_force_group_topk(want[g], k)
        assert np.asarray(idx_k[g * k:(g + 1) * k]).tolist() == [g * hd + c for c in sel]
        for h in (2 * g, 2 * g + 1):
            assert np.asarray(idx_q[h * k:(h + 1) * k]).tolist() == [h * hd + c for c in sel]


# ------------------------------------------------- estimator variants (pins)
def _rope_rotate(Y, head_dim, seed):
    """Rotate every (c, c + head_dim/2) pair of every head of Y (tokens x
    heads*head_dim) by a token- and pair-dependent angle (rotary embedding's
    rotate-half form), with torch: an implementation independent of the oracle."""
    T, n = Y.shape
    half = head_dim // 2
    ang = torch.from_numpy(synth.rng(seed).uniform(-np.pi, np.pi, size=(T, half)))
    t = torch.from_numpy(Y).reshape(T, n // head_dim, head_dim)
    x1, x2 = t[..., :half], t[..., half:]
    c, s = torch.cos(ang)[:, None, :], torch.sin(ang)[:, None, :]
    out = torch.cat([x1 * c - x2 * s, x1 * s + x2 * c], dim=-1)
    return out.reshape(T, n).numpy()


def _pair_norms_torch(Y, heads, head_dim):
    half = head_dim // 2
    t = torch.from_numpy(Y).reshape(Y.shape[0], heads, 2, half)
    return torch.sqrt((t * t).sum(dim=(0, 2))).numpy()  # (heads, half)


@pytest.mark.parametrize("H,KV", [(3, 3), (4, 2)])
def test_qk_pair_scores_equal_post_rotary_pair_norms(H, KV):
    """Pair scores computed from the estimate before rotary embedding equal the
    norm products of the rotated estimates, pair by pair: the rotate-half
    partner of channel c is c + head_dim/2 (an adjacent pairing fails this)."""
    rg = synth.rng(501)
    hd, r, t = 6, 4, 9
    P_q, P_k = rg.standard_normal((t, r)), rg.standard_normal((t, r))
    U_q, U_k = rg.standard_normal((H * hd, r)), rg.standard_normal((KV * hd, r))
    got = O.qk_pair_scores(P_q, P_k, U_q, U_k, H, KV, hd)
    Qr = _rope_rotate(P_q @ U_q.T, hd, 502)
    Kr = _rope_rotate(P_k @ U_k.T, hd, 503)
    nq, nk = _pair_norms_torch(Qr, H, hd), _pair_norms_torch(Kr, KV, hd)
    grp = H // KV
    want = np.stack([nk[g] * nq[g * grp:(g + 1) * grp].sum(axis=0) for g in range(KV)])
    np.testing.assert_allclose(got, want, rtol=1e-12)


def test_qk_pair_scores_reduce_to_qk_when_partners_vanish():
    """With the second half of every head zeroed, a pair's score is the plain
    QK-norm score of its first channel."""
    rg = synth.rng(504)
    H, KV, hd, r, t = 4, 2, 8, 3, 7
    P_q, P_k = rg.standard_normal((t, r)), rg.standard_normal((t, r))
    U_q, U_k = rg.standard_normal((H * hd, r)), rg.standard_normal((KV * hd, r))
    for U in (U_q, U_k):
        U.reshape(-1, hd, r)[:, hd // 2:, :] = 0.0
    pair = O.qk_pair_scores(P_q, P_k, U_q, U_k, H, KV, hd)
    plain = O.qk_scores(P_q, P_k, U_q, U_k, H, KV, hd)
    np.testing.assert_allclose(pair, plain[:, :hd // 2], rtol=1e-12)


def test_qk_pair_score_bounds_rotated_products():
    """Cauchy-Schwarz: whatever the rotation angles, a pair's summed share of
    the query-key products |sum_t <q_t,p, k_t,p>| stays within its score (MHA)."""
    rg = synth.rng(505)
    H, hd, r, t = 2, 4, 3, 11
    P_q, P_k = rg.standard_normal((t, r)), rg.standard_normal((t, r))
    U_q, U_k = rg.standard_normal((H * hd, r)), rg.standard_normal((H * hd, r))
    sc = O.qk_pair_scores(P_q, P_k, U_q, U_k, H, H, hd)
    for seed in range(5):
        Qr = _rope_rotate(P_q @ U_q.T, hd, 600 + seed).reshape(t, H, 2, hd // 2)
        Kr = _rope_rotate(P_k @ U_k.T, hd, 700 + seed).reshape(t, H, 2, hd // 2)
        share = np.abs(np.einsum("thap,thap->hp", Qr, Kr))
        assert np.all(share <= sc * (1 + 1e-12))


def test_estimate_select_qk_pairs_hand_built_layout():
    """Two query heads sharing one key head, head_dim 4 (pairs (0, 2), (1, 3)),
    one context token, d = rank = 1, so the norms are the factor entries:
      query head 0 [1, 2, 3, 0] -> pair norms [sqrt(10), 2]
      query head 1 [0, 1, 0, 1] -> pair norms [0, sqrt(2)]
      key head     [1, 1, 1, 1] -> pair norms [sqrt(2), sqrt(2)]
    scores: pair 0 = sqrt(2) sqrt(10) = 4.47, pair 1 = sqrt(2) (2 + sqrt(2)) = 4.83.
    At s = 0.5 one pair (pair 1) is kept: channels 1 and 3 of every head."""
    U_q = np.array([1, 2, 3, 0, 0, 1, 0, 1], dtype=float).reshape(8, 1)
    U_k = np.ones((4, 1))
    one = np.ones((1, 1))
    X = np.array([[1.0], [50.0]])
    iq, ik, k, sc = O.estimate_select_qk_pairs(X, 1, 2, [1], one, U_q, one, U_k, 2, 1, 4, 0.5)
    np.testing.assert_allclose(sc, [[math.sqrt(20), 2 * math.sqrt(2) + 2]], rtol=1e-14)
    assert k == 2
    assert iq.tolist() == [1, 3, 5, 7] and ik.tolist() == [1, 3]
    iq, ik, k, _ = O.estimate_select_qk_pairs(X, 1, 2, [1], one, U_q, one, U_k, 2, 1, 4, 0.0)
    assert k == 4 and iq.tolist() == list(range(8)) and ik.tolist() == [0, 1, 2, 3]


@pytest.mark.parametrize("H,KV", [(3, 3), (4, 2)])
def test_l2_scores_full_rank_exact_and_per_head_selection(H, KV):
    """Full-rank factors: the scores are the exact column norms of X_C W^T per
    value head (torch); each value head keeps the brute-force top-k of its own
    norms, listed as g*head_dim + c, and every query head h repeats the set of
    its group h // (H / KV) as h*head_dim + c."""
    rg = synth.rng(510)
    hd, d = 5, 4
    tok = synth.Tokens(batch=2, seq=3, ctx_len=np.array([2, 3], np.int32))
    X = rg.standard_normal((tok.T, d))
    W = rg.standard_normal((KV * hd, d))
    Lw, Uw = _full_rank_factors(W)
    io, iv, k, sc = O.estimate_select_l2(X, tok.batch, tok.seq, tok.ctx_len, Lw, Uw, H, KV, hd,
                                         0.4)
    want = colnorm(X[[0, 1, 3, 4, 5]] @ W.T).reshape(KV, hd)
    np.testing.assert_allclose(sc, want, rtol=1e-10)
    assert k == 3
    for g in range(KV):
        sel = _brute_force_topk(list(want[g]), k)
        assert iv[g * k:(g + 1) * k].tolist() == [g * hd + c for c in sel]
        for h in range(g * (H // KV), (g + 1) * (H // KV)):
            assert io[h * k:(h + 1) * k].tolist() == [h * hd + c for c in sel]


def test_estimate_select_ffn_gram_full_rank_brute_force():
    """Full-rank gate/up factors: the Gram score is the product of the exact
    column norms of X_C Wg^T and X_C Wu^T, and the kept set is the brute-force
    best subset."""
    rg = synth.rng(511)
    d, d_ff = 4, 9
    tok = synth.Tokens(batch=1, seq=6, ctx_len=np.array([5], np.int32))
    X = rg.standard_normal((tok.T, d))
    Wg, Wu = rg.standard_normal((d_ff, d)), rg.standard_normal((d_ff, d))
    Lg, Ug = _full_rank_factors(Wg)
    Lu, Uu = _full_rank_factors(Wu)
    idx, k, sc = O.estimate_select_ffn_gram(X, tok.batch, tok.seq, tok.ctx_len, Lg, Ug, Lu, Uu,
                                            0.5)
    Xc = X[:5]
    want = colnorm(Xc @ Wg.T) * colnorm(Xc @ Wu.T)
    np.testing.assert_allclose(sc, want, rtol=1e-10)
    assert k == 5 and idx.tolist() == _brute_force_topk(list(want), k)


# ---------------------------------------------------------------- LoRA linear
def _lin_case(seed, n=9, k=7, r=3, tok=None):
    tok = tok or synth.Tokens(batch=2, seq=5, ctx_len=np.array([3, 4], np.int32))
    X = synth.gaussian((tok.T, k), 1.0, seed)
    W0 = synth.gaussian((n, k), 0.3, seed + 1)
    A = synth.gaussian((r, k), 0.3, seed + 2)
    B = synth.gaussian((n, r), 0.3, seed + 3)
    return tok, X, W0, A, B


def _merged(W0, A, B, s):
    return W0 + s * (B @ A)


def test_linear_dense_equals_merged_weight():
    tok, X, W0, A, B = _lin_case(40)
    Y, _, _ = O.linear_fwd("none", X, None, tok.batch, tok.seq, tok.ctx_len, W0, A, B, 0.7, None)
    np.testing.assert_allclose(Y, X @ _merged(W0, A, B, 0.7).T, rtol=1e-12)


def test_linear_out_rows_all_channels_is_dense():
    tok, X, W0, A, B = _lin_case(41)
    C, Oo = O.context_rows(tok.batch, tok.seq, tok.ctx_len)
    idx = np.arange(W0.shape[0])
    Yc, Yo, _ = O.linear_fwd("out_rows", X, None, tok.batch, tok.seq, tok.ctx_len, W0, A, B, 0.5, idx)
    dense = X @ _merged(W0, A, B, 0.5).T
    np.testing.assert_allclose(Yc, dense[C], rtol=1e-12)
    np.testing.assert_allclose(Yo, dense[Oo], rtol=1e-12)


def test_linear_out_rows_slice_equals_masked_dense():
    tok, X, W0, A, B = _lin_case(42)
    C, Oo = O.context_rows(tok.batch, tok.seq, tok.ctx_len)
    idx = np.array([1, 4, 5, 8])
    Yc, Yo, _ = O.linear_fwd("out_rows", X, None, tok.batch, tok.seq, tok.ctx_len, W0, A, B, 0.5, idx)
    dense = X @ _merged(W0, A, B, 0.5).T
    np.testing.assert_allclose(Yc, dense[C][:, idx], rtol=1e-12)
    np.testing.assert_allclose(Yo, dense[Oo], rtol=1e-12)


def test_linear_in_cols_slice_equals_masked_dense():
    tok, X, W0, A, B = _lin_case(43)
    C, Oo = O.context_rows(tok.batch, tok.seq, tok.ctx_len)
    idx = np.array([0, 2, 3, 6])
    Xc = X[C][:, idx]
    Y, _, _ = O.linear_fwd("in_cols", Xc, X[Oo], tok.batch, tok.seq, tok.ctx_len, W0, A, B, 0.5, idx)
    Xmask = np.zeros_like(X)
    Xmask[np.ix_(C, idx)] = Xc
    Xmask[Oo] = X[Oo]
    np.testing.assert_allclose(Y, Xmask @ _merged(W0, A, B, 0.5).T, rtol=1e-12)


def _fd(f, x, eps=1e-6):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = x[i]
        x[i] = old + eps
        fp = f()
        x[i] = old - eps
        fm = f()
        x[i] = old
        g[i] = (fp - fm) / (2 * eps)
    return g


@pytest.mark.parametrize("side", ["none", "out_rows", "in_cols"])
def test_linear_bwd_finite_differences(side):
    tok, X, W0, A, B = _lin_case(50 + len(side))
    C, Oo = O.context_rows(tok.batch, tok.seq, tok.ctx_len)
    s = 0.8
    idx = np.array([0, 3, 4]) if side == "in_cols" else np.array([1, 2, 6, 7])
    if side == "in_cols":
        Xin, Xout = X[C][:, idx].copy(), X[Oo].copy()
    else:
        Xin, Xout = X.copy(), None
    rg = synth.rng(77)

    def fwd():
        return O.linear_fwd(side, Xin, Xout, tok.batch, tok.seq, tok.ctx_len, W0, A, B, s, idx)

    Y1, Y2, XA = fwd()
    dY1 = rg.standard_normal(Y1.shape)
    dY2 = rg.standard_normal(Y2.shape) if Y2 is not None else None

    def loss():
        a, b, _ = fwd()
        v = np.sum(a * dY1)
        return v + (np.sum(b * dY2) if b is not None else 0.0)

    dXc, dXo, dA, dB = O.linear_bwd(side, Xin, Xout, XA, dY1, dY2, tok.batch, tok.seq,
                                    tok.ctx_len, W0, A, B, s, idx)
    np.testing.assert_allclose(dA, _fd(loss, A), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dB, _fd(loss, B), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dXc, _fd(loss, Xin), rtol=1e-6, atol=1e-8)
    if Xout is not None:
        np.testing.assert_allclose(dXo, _fd(loss, Xout), rtol=1e-6, atol=1e-8)


# ----------------------------------------------------------------------- FFN
def _ffn_layer(seed, d=6, d_ff=10, r=2, scale=0.9, wscale=0.6):
    g = lambda shape, k: synth.gaussian(shape, wscale, seed + k)
    return dict(Wg=g((d_ff, d), 1), Wu=g((d_ff, d), 2), Wd=g((d, d_ff), 3),
                Ag=g((r, d), 4), Bg=g((d_ff, r), 5), Au=g((r, d), 6), Bu=g((d_ff, r), 7),
                Ad=g((r, d_ff), 8), Bd=g((d, r), 9), scale=scale)


def _dense_swiglu(X, lay, mask=None):
    """Textbook SwiGLU with merged LoRA weights, torch SiLU; ``mask`` zeroes
    the gate/up rows (weight and LoRA-B) of skipped channels."""
    s = lay["scale"]
    Wg = _merged(lay["Wg"], lay["Ag"], lay["Bg"], s)
    Wu = _merged(lay["Wu"], lay["Au"], lay["Bu"], s)
    Wd = _merged(lay["Wd"], lay["Ad"], lay["Bd"], s)
    if mask is not None:
        Wg = Wg * mask[:, None]
        Wu = Wu * mask[:, None]
    return (tsilu(X @ Wg.T) * (X @ Wu.T)) @ Wd.T


def test_ffn_all_channels_is_dense_swiglu():
    tok = synth.Tokens(batch=2, seq=6, ctx_len=np.array([4, 5], np.int32))
    lay = _ffn_layer(60)
    X = synth.gaussian((tok.T, 6), 1.0, 61)
    out, _ = O.ffn_fwd(X, tok.batch, tok.seq, tok.ctx_len, lay, np.arange(10))
    np.testing.assert_allclose(out, _dense_swiglu(X, lay), rtol=1e-11)


def test_ffn_slice_equals_masked_dense():
    tok = synth.Tokens(batch=2, seq=6, ctx_len=np.array([4, 5], np.int32))
    lay = _ffn_layer(62)
    X = synth.gaussian((tok.T, 6), 1.0, 63)
    idx = np.array([0, 2, 3, 7, 9])
    mask = np.zeros(10)
    mask[idx] = 1
    out, _ = O.ffn_fwd(X, tok.batch, tok.seq, tok.ctx_len, lay, idx)
    C, Oo = O.context_rows(tok.batch, tok.seq, tok.ctx_len)
    np.testing.assert_allclose(out[C], _dense_swiglu(X, lay, mask)[C], rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(out[Oo], _dense_swiglu(X, lay)[Oo], rtol=1e-11)


def _ffn_fd_check(lay, X, tok, idx, tol=1e-6):
    rg = synth.rng(88)
    dOut = rg.standard_normal((tok.T, lay["Wd"].shape[0]))

    def loss():
        out, _ = O.ffn_fwd(X, tok.batch, tok.seq, tok.ctx_len, lay, idx)
        return np.sum(out * dOut)

    out, saved = O.ffn_fwd(X, tok.batch, tok.seq, tok.ctx_len, lay, idx)
    gr = O.ffn_bwd(X, dOut, lay, idx, saved)
    np.testing.assert_allclose(gr["dX"], _fd(loss, X), rtol=tol, atol=1e-8)
    for name in ("Ag", "Bg", "Au", "Bu", "Ad", "Bd"):
        np.testing.assert_allclose(gr["d" + name], _fd(loss, lay[name]), rtol=tol, atol=1e-8)


def test_ffn_bwd_finite_differences():
    tok = synth.Tokens(batch=2, seq=6, ctx_len=np.array([4, 5], np.int32))
    lay = _ffn_layer(64)
    X = synth.gaussian((tok.T, 6), 1.0, 65)
    _ffn_fd_check(lay, X, tok, np.array([1, 2, 5, 6, 8]))


def test_ffn_zero_grad_rows_for_skipped_channels():
    """No output tokens: skipped channels get exactly zero LoRA-B rows (gate,
    up) and zero LoRA-A columns (down)."""
    tok = synth.Tokens(batch=2, seq=5, ctx_len=np.array([5, 5], np.int32))
    lay = _ffn_layer(66)
    X = synth.gaussian((tok.T, 6), 1.0, 67)
    dOut = synth.gaussian((tok.T, 6), 1.0, 68)
    idx = np.array([0, 4, 5, 9])
    skip = np.setdiff1d(np.arange(10), idx)
    out, saved = O.ffn_fwd(X, tok.batch, tok.seq, tok.ctx_len, lay, idx)
    gr = O.ffn_bwd(X, dOut, lay, idx, saved)
    assert np.all(gr["dBg"][skip] == 0) and np.all(gr["dBu"][skip] == 0)
    assert np.all(gr["dAd"][:, skip] == 0)
    assert np.any(gr["dBg"][idx] != 0) and np.any(gr["dAd"][:, idx] != 0)


def test_ffn_fwd_bwd_estimator_path_small_case():
    """End-to-end oracle on a reduced workload-0 shape: the chosen set is the
    top-k of the scores and equals the full-sparsity-0 dense result at s=0."""
    tok = synth.Tokens.uniform(1, 32)
    case = synth.ffn_case(tok, d=16, d_ff=40, r_svd=4, r_lora=4, sparsity=0.5)
    lay = dict(Wg=case.Wg.W, Wu=case.Wu.W, Wd=case.Wd.W, Ag=case.Ag, Bg=case.Bg, Au=case.Au,
               Bu=case.Bu, Ad=case.Ad, Bd=case.Bd, scale=1.0)
    for nm, sw in (("g", case.Wg), ("u", case.Wu)):
        lay["L" + nm], lay["U" + nm] = O.svd_prepare(sw.W, 4)
    res = O.ffn_fwd_bwd(case.X, case.dOut, tok.batch, tok.seq, tok.ctx_len, lay, 0.5)
    assert res["k"] == 20 and len(res["idx"]) == 20
    sc = res["scores"]
    mask = np.zeros(40, bool)
    mask[res["idx"]] = True
    assert sc[mask].min() >= sc[~mask].max()
    dense = O.ffn_fwd_bwd(case.X, case.dOut, tok.batch, tok.seq, tok.ctx_len, lay, 0.0)
    np.testing.assert_allclose(dense["out"], _dense_swiglu(case.X, lay), rtol=1e-10)


def test_context_rows_layout():
    C, Oo = O.context_rows(3, 4, [1, 4, 0])
    assert C.tolist() == [0, 4, 5, 6, 7]
    assert Oo.tolist() == [1, 2, 3, 8, 9, 10, 11]


# --------------------------------------------------------- planted mistakes
def test_planted_silu_grad_sign_is_caught(monkeypatch):
    monkeypatch.setattr(O, "silu_grad", lambda x: 1.0 / (1.0 + np.exp(x)) * (1 + x))
    tok = synth.Tokens(batch=1, seq=4, ctx_len=np.array([3], np.int32))
    lay = _ffn_layer(70, d=3, d_ff=4)
    X = synth.gaussian((tok.T, 3), 1.0, 71)
    with pytest.raises(AssertionError):
        _ffn_fd_check(lay, X, tok, np.array([0, 2]))


def test_planted_dropped_lora_term_is_caught(monkeypatch):
    real = O.linear_fwd

    def broken(side, X_ctx, X_out, b, s_, c, W0, A, B, scale, idx):
        return real(side, X_ctx, X_out, b, s_, c, W0, A, B, 0.0 if side == "out_rows" else scale, idx)

    monkeypatch.setattr(O, "linear_fwd", broken)
    with pytest.raises(AssertionError):
        test_linear_out_rows_slice_equals_masked_dense()


def test_planted_transposed_factor_is_caught(monkeypatch):
    real = O.ffn_scores
    monkeypatch.setattr(O, "ffn_scores", lambda Pg, Pu, Ug, Uu: real(Pu, Pg, Ug, Uu))
    with pytest.raises(AssertionError):
        test_ffn_score_full_rank_equals_exact_activation_norm()


def test_planted_tie_break_is_caught(monkeypatch):
    def upper_wins(score, k):
        order = np.lexsort((-np.arange(score.size), -np.asarray(score)))
        return np.sort(order[:k])
    monkeypatch.setattr(O, "topk_select", upper_wins)
    with pytest.raises(AssertionError):
        for seed in range(12):
            test_topk_brute_force_with_ties(seed)


def _qk_variant(query_group, key_offset):
    """estimate_select_qk with its index layout rebuilt from the oracle's own
    pieces, so a planted layout mistake can be checked against the pins."""
    def est(X, batch, seq, ctx_len, L_q, U_q, L_k, U_k, heads, kv_heads, head_dim, s):
        C, _ = O.context_rows(batch, seq, ctx_len)
        Xc = X[C]
        scores = O.qk_scores(Xc @ L_q, Xc @ L_k, U_q, U_k, heads, kv_heads, head_dim)
        k = O.keep_count(head_dim, s)
        sel = O.select_per_group(scores, k)
        group = heads // kv_heads
        idx_q = np.concatenate([h * head_dim + sel[query_group(h, group, kv_heads)]
                                for h in range(heads)])
        idx_k = np.concatenate([key_offset(g, group, head_dim) + sel[g] for g in range(kv_heads)])
        return idx_q, idx_k, k, scores
    return est


def test_planted_qk_layout_mistakes_are_caught():
    """The correct layout passes the hand-built pin; a query head mapped to the
    wrong group (h % kv_heads instead of h // group) or key heads offset by the
    query-head stride (g * group * head_dim) fail it."""
    _check_qk_hand_case(_qk_variant(lambda h, gr, kv: h // gr, lambda g, gr, hd: g * hd))
    with pytest.raises(AssertionError):
        _check_qk_hand_case(_qk_variant(lambda h, gr, kv: h % kv, lambda g, gr, hd: g * hd))
    with pytest.raises(AssertionError):
        _check_qk_hand_case(_qk_variant(lambda h, gr, kv: h // gr, lambda g, gr, hd: g * gr * hd))


def test_planted_group_select_mistake_is_caught(monkeypatch):
    """select_per_group that takes the k smallest instead of the k largest."""
    monkeypatch.setattr(O, "select_per_group",
                        lambda sc, k: np.stack([np.sort(np.argsort(r, kind="stable")[:k])
                                                for r in sc]))
    with pytest.raises(AssertionError):
        test_estimate_select_qk_hand_built_gqa_layout()


def test_planted_adjacent_pairing_is_caught(monkeypatch):
    """Pairs (2i, 2i + 1) instead of rotate-half (c, c + head_dim/2)."""
    def adjacent(P_q, P_k, U_q, U_k, heads, kv_heads, head_dim):
        Qh, Kh = P_q @ U_q.T, P_k @ U_k.T
        sq = np.sum(Qh * Qh, axis=0).reshape(heads, head_dim // 2, 2).sum(axis=2)
        sk = np.sum(Kh * Kh, axis=0).reshape(kv_heads, head_dim // 2, 2).sum(axis=2)
        grp = heads // kv_heads
        return np.stack([np.sqrt(sk[g]) * np.sqrt(sq[g * grp:(g + 1) * grp]).sum(axis=0)
                         for g in range(kv_heads)])
    monkeypatch.setattr(O, "qk_pair_scores", adjacent)
    with pytest.raises(AssertionError):
        test_qk_pair_scores_equal_post_rotary_pair_norms(3, 3)


def test_planted_l2_head_offset_is_caught(monkeypatch):
    """estimate_select_l2 listing the query heads' channels without the
    h*head_dim offset, or the value heads' with the query-head stride."""
    real = O.estimate_select_l2

    def no_offset(X, batch, seq, ctx_len, L, U, heads, kv_heads, head_dim, s):
        io, iv, k, sc = real(X, batch, seq, ctx_len, L, U, heads, kv_heads, head_dim, s)
        return io % head_dim, iv, k, sc

    def query_stride(X, batch, seq, ctx_len, L, U, heads, kv_heads, head_dim, s):
        io, iv, k, sc = real(X, batch, seq, ctx_len, L, U, heads, kv_heads, head_dim, s)
        grp = heads // kv_heads
        return io, (iv // head_dim) * grp * head_dim + iv % head_dim, k, sc
    for bad in (no_offset, query_stride):
        monkeypatch.setattr(O, "estimate_select_l2", bad)
        with pytest.raises(AssertionError):
            test_l2_scores_full_rank_exact_and_per_head_selection(4, 2)

def test_oracle_package_exports():
    for name in O.__all__:
        assert hasattr(oracle, name)


# ------------------------------------------------- projection-set variants
def _tiny_ffn(seed, d=12, d_ff=20, r=3, r_svd=4):
    rng_ = np.random.default_rng(seed)
    lay = {"scale": 0.7}
    for nm, n, k in (("g", d_ff, d), ("u", d_ff, d), ("d", d, d_ff)):
        lay["W" + nm] = rng_.normal(size=(n, k)) / np.sqrt(k)
        lay["A" + nm] = rng_.normal(size=(r, k)) * 0.3
        lay["B" + nm] = rng_.normal(size=(n, r)) * 0.3
    lay["Lg"], lay["Ug"] = O.svd_prepare(lay["Wg"], r_svd)
    lay["Lu"], lay["Uu"] = O.svd_prepare(lay["Wu"], r_svd)
    return lay


def test_per_sequence_sets_with_identical_sequences_equal_the_batch_set():
    """Pooling over identical sequences multiplies every score by the same
    factor: the per-batch set is each sequence's set, and the per-batch
    gradients are the per-sequence sums."""
    lay = _tiny_ffn(1)
    seq, d = 7, 12
    x1 = np.random.default_rng(2).normal(size=(seq, d))
    dy1 = np.random.default_rng(3).normal(size=(seq, d))
    X, dY = np.vstack([x1, x1, x1]), np.vstack([dy1, dy1, dy1])
    per = O.ffn_fwd_bwd_per_seq(X, dY, 3, seq, [5, 5, 5], lay, 0.5)
    bat = O.ffn_fwd_bwd(X, dY, 3, seq, [5, 5, 5], lay, 0.5)
    for s_ in per["idx"]:
        np.testing.assert_array_equal(s_, bat["idx"])
    for key in ("out", "dX", "dAg", "dBg", "dAu", "dBu", "dAd", "dBd"):
        np.testing.assert_allclose(per[key], bat[key], rtol=1e-12, atol=1e-13)


def test_per_sequence_matches_row_masked_dense_autograd():
    """Independent formulation: a dense SwiGLU FFN in PyTorch float64 whose
    context rows multiply the intermediate activations by their own
    sequence's 0/1 channel mask, gradients by autograd."""
    lay = _tiny_ffn(4)
    b, seq, d = 3, 6, 12
    ctx = [4, 6, 2]
    rng_ = np.random.default_rng(5)
    X, dY = rng_.normal(size=(b * seq, d)), rng_.normal(size=(b * seq, d))
    per = O.ffn_fwd_bwd_per_seq(X, dY, b, seq, ctx, lay, 0.6)
    assert len({tuple(s_) for s_ in per["idx"]}) > 1   # the sets do differ
    mask = np.ones((b * seq, 20))
    for bb in range(b):
        m = np.zeros(20)
        m[per["idx"][bb]] = 1.0
        mask[bb * seq: bb * seq + ctx[bb]] = m
    t = {k: torch.from_numpy(np.asarray(v, dtype=np.float64).copy()).requires_grad_()
         for k, v in lay.items() if k[0] in "AB"}
    W = {k: torch.from_numpy(lay[k]) for k in ("Wg", "Wu", "Wd")}
    tx = torch.from_numpy(X.copy()).requires_grad_()
    s_ = lay["scale"]
    g = tx @ W["Wg"].T + s_ * (tx @ t["Ag"].T) @ t["Bg"].T
    u = tx @ W["Wu"].T + s_ * (tx @ t["Au"].T) @ t["Bu"].T
    h = torch.nn.functional.silu(g) * u * torch.from_numpy(mask)
    y = h @ W["Wd"].T + s_ * (h @ t["Ad"].T) @ t["Bd"].T
    np.testing.assert_allclose(per["out"], y.detach().numpy(), rtol=1e-11, atol=1e-12)
    (y * torch.from_numpy(dY)).sum().backward()
    np.testing.assert_allclose(per["dX"], tx.grad.numpy(), rtol=1e-10, atol=1e-12)
    for k in ("Ag", "Bg", "Au", "Bu", "Ad", "Bd"):
        np.testing.assert_allclose(per["d" + k], t[k].grad.numpy(), rtol=1e-10, atol=1e-12)


def test_down_projection_only_equals_the_sliced_ffn():
    """Dropping a channel's activation before the down projection gives the
    sliced FFN's output: the gate/up values of a skipped channel reach the
    output only through its down-projection column."""
    lay = _tiny_ffn(6)
    b, seq = 2, 5
    X = np.random.default_rng(7).normal(size=(b * seq, 12))
    idx = np.array([0, 3, 4, 9, 15, 19])
    out, _ = O.ffn_fwd(X, b, seq, [3, 5], lay, idx)
    np.testing.assert_allclose(O.ffn_fwd_down_only(X, b, seq, [3, 5], lay, idx), out,
                               rtol=1e-12, atol=1e-13)
    full = O.ffn_fwd_down_only(X, b, seq, [0, 0], lay, idx)   # no context rows: dense
    dense, _ = O.ffn_fwd(X, b, seq, [0, 0], lay, np.arange(20))
    np.testing.assert_allclose(full, dense, rtol=1e-12, atol=1e-13)

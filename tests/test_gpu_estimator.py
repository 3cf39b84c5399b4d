"""GPU parity of the estimator and top-k kernels (through the C ABI) with the
CPU oracle: every rank template of the activation-norm score kernel, ragged
and empty context sets, long score lists, the Gram-form
criteria (QK-norm, rotate-half pairs, per-head L2, Gram FFN score), exact
tie-breaking, bit-reproducibility, and the offline prepare at the benchmark's
own weight shapes.  Scores are compared at relative Frobenius 1e-5 (fp32
accuracy), selections set-against-set with the near-tie rule.
"""
import numpy as np
import pytest
import torch

from oracle import slora_oracle as O
from contextual_sparsity_lora_svd_b200 import synth
from tests.helpers import check_selection, dev, host, rel_frob

pytestmark = pytest.mark.gpu

SCORE_TOL = 1e-5


@pytest.fixture(scope="module")
def L():
    from contextual_sparsity_lora_svd_b200 import _lib
    assert torch.cuda.is_available()
    return _lib


def _tok(batch, seq, ctx):
    return synth.Tokens(batch, seq, np.asarray(ctx, np.int32))


def f32(a):
    return dev(np.ascontiguousarray(a), torch.float32)


def _factors(n, d, r, seed, bf16=True):
    return O.svd_prepare(synth.decaying_weight(n, d, seed, bf16=bf16).W, r)


def _run(L, crit, X, tok, L0, U0, L1, U1, r, s, n_idx, n_scores, **kw):
    idx = torch.full((n_idx,), -1, dtype=torch.int32, device="cuda")
    scores = torch.full((n_scores,), -1.0, device="cuda")
    k = L.slora_estimate_select(crit, dev(X, torch.bfloat16), tok.batch, tok.seq, tok.ctx_len,
                                f32(L0), f32(U0), f32(L1) if L1 is not None else f32(L0),
                                f32(U1) if U1 is not None else f32(U0), r, s, idx,
                                scores_out=scores, **kw)
    torch.cuda.synchronize()
    return k, host(idx).astype(np.int64), host(scores)


# ------------------------------------------------- activation-norm score
@pytest.mark.parametrize("r", [3, 8, 12, 16, 24, 32, 48])
def test_ffn_activation_score_all_rank_templates(L, r):
    """One case per rank template (8 rank indices per K chunk), with a ragged
    context set (sequences of 29, 0 and 51 context tokens) and d_ff not a
    multiple of the channel block."""
    tok = _tok(3, 64, [29, 0, 51])
    d, d_ff, s = 64, 300, 0.5
    X = synth.round_bf16(synth.gaussian((tok.T, d), 1.0, 800 + r))
    Lg, Ug = _factors(d_ff, d, r, 801 + r)
    Lu, Uu = _factors(d_ff, d, r, 802 + r)
    io, ko, so = O.estimate_select_ffn(X, tok.batch, tok.seq, tok.ctx_len, Lg, Ug, Lu, Uu, s)
    k, gi, gs = _run(L, L.CRIT_FFN, X, tok, Lg, Ug, Lu, Uu, r, s, d_ff, d_ff)
    assert k == ko
    assert rel_frob(gs, so) < SCORE_TOL
    check_selection(gi[:k], io, so, k, f"ffn r={r}")


@pytest.mark.parametrize("s", [0.0, 0.3, 0.7, 0.99])
def test_ffn_activation_score_long_vector_standalone_select(L, s):
    """d_ff = 20000 channels (the top-k block with 64 register rows per
    thread); few context tokens keep the oracle quick."""
    tok = _tok(2, 40, [30, 25])
    d, d_ff, r = 32, 20000, 8
    rg = synth.rng(810)
    X = synth.round_bf16(rg.standard_normal((tok.T, d)))
    Lg, Lu = rg.standard_normal((d, r)) * 0.1, rg.standard_normal((d, r)) * 0.1
    Ug, Uu = rg.standard_normal((d_ff, r)), rg.standard_normal((d_ff, r))
    io, ko, so = O.estimate_select_ffn(X, tok.batch, tok.seq, tok.ctx_len, Lg, Ug, Lu, Uu, s)
    k, gi, gs = _run(L, L.CRIT_FFN, X, tok, Lg, Ug, Lu, Uu, r, s, d_ff, d_ff)
    assert k == ko
    assert rel_frob(gs, so) < SCORE_TOL
    check_selection(gi[:k], io, so, k, "ffn long")


def test_ffn_no_context_tokens_keeps_lowest_indices(L):
    """No context token: every score is 0, so the lowest k indices are kept."""
    tok = _tok(2, 16, [0, 0])
    d, d_ff, r = 32, 100, 8
    X = synth.round_bf16(synth.gaussian((tok.T, d), 1.0, 820))
    Lg, Ug = _factors(d_ff, d, r, 821)
    Lu, Uu = _factors(d_ff, d, r, 822)
    k, gi, gs = _run(L, L.CRIT_FFN, X, tok, Lg, Ug, Lu, Uu, r, 0.5, d_ff, d_ff)
    assert k == 50 and np.all(gs == 0.0)
    assert gi[:k].tolist() == list(range(50))


def test_ffn_score_bit_reproducible(L):
    tok = _tok(4, 128, [96, 96, 70, 128])
    d, d_ff, r = 128, 1000, 8
    X = synth.round_bf16(synth.gaussian((tok.T, d), 1.0, 830))
    Lg, Ug = _factors(d_ff, d, r, 831)
    Lu, Uu = _factors(d_ff, d, r, 832)
    a = _run(L, L.CRIT_FFN, X, tok, Lg, Ug, Lu, Uu, r, 0.5, d_ff, d_ff)
    b = _run(L, L.CRIT_FFN, X, tok, Lg, Ug, Lu, Uu, r, 0.5, d_ff, d_ff)
    assert np.array_equal(a[1], b[1]) and np.array_equal(a[2], b[2])


# ----------------------------------------------------------- Gram criteria
@pytest.mark.parametrize("s", [0.0, 0.5, 0.8])
def test_ffn_gram_criterion(L, s):
    tok = _tok(3, 50, [40, 12, 50])
    d, d_ff, r = 64, 700, 8
    X = synth.round_bf16(synth.gaussian((tok.T, d), 1.0, 840))
    Lg, Ug = _factors(d_ff, d, r, 841)
    Lu, Uu = _factors(d_ff, d, r, 842)
    io, ko, so = O.estimate_select_ffn_gram(X, tok.batch, tok.seq, tok.ctx_len, Lg, Ug, Lu, Uu, s)
    k, gi, gs = _run(L, L.CRIT_FFN_GRAM, X, tok, Lg, Ug, Lu, Uu, r, s, d_ff, d_ff)
    assert k == ko
    assert rel_frob(gs, so) < SCORE_TOL
    check_selection(gi[:k], io, so, k, "ffn gram")


def test_ffn_gram_criterion_long_vector(L):
    """20000 channels: the Gram scores span many blocks and the standalone
    top-k runs after them."""
    tok = _tok(1, 64, [48])
    d, d_ff, r = 32, 20000, 4
    rg = synth.rng(845)
    X = synth.round_bf16(rg.standard_normal((tok.T, d)))
    Lg, Lu = rg.standard_normal((d, r)), rg.standard_normal((d, r))
    Ug, Uu = rg.standard_normal((d_ff, r)), rg.standard_normal((d_ff, r))
    io, ko, so = O.estimate_select_ffn_gram(X, tok.batch, tok.seq, tok.ctx_len, Lg, Ug, Lu, Uu,
                                            0.6)
    k, gi, gs = _run(L, L.CRIT_FFN_GRAM, X, tok, Lg, Ug, Lu, Uu, r, 0.6, d_ff, d_ff)
    assert k == ko
    assert rel_frob(gs, so) < SCORE_TOL
    check_selection(gi[:k], io, so, k, "ffn gram long")


@pytest.mark.parametrize("heads,kv", [(4, 4), (8, 2)])
@pytest.mark.parametrize("s", [0.0, 0.5, 0.75])
def test_qk_rope_pair_criterion(L, heads, kv, s):
    tok = _tok(2, 48, [36, 20])
    d, hd, r = 64, 32, 8
    half = hd // 2
    X = synth.round_bf16(synth.gaussian((tok.T, d), 1.0, 850))
    Lq, Uq = _factors(heads * hd, d, r, 851)
    Lk, Uk = _factors(kv * hd, d, r, 852)
    iq, ik, kh, sc = O.estimate_select_qk_pairs(X, tok.batch, tok.seq, tok.ctx_len, Lq, Uq, Lk,
                                                Uk, heads, kv, hd, s)
    k, gi, gs = _run(L, L.CRIT_QK_ROPE_PAIR, X, tok, Lq, Uq, Lk, Uk, r, s, (heads + kv) * hd,
                     kv * half, heads=heads, kv_heads=kv, head_dim=hd)
    assert k == kh
    assert rel_frob(gs, sc.ravel()) < SCORE_TOL
    kp = kh // 2
    grp = heads // kv
    for g in range(kv):
        kg = gi[heads * kh + g * kh: heads * kh + (g + 1) * kh] - g * hd
        ko = ik[g * kh:(g + 1) * kh] - g * hd
        # pair firsts, then their partners c + half
        assert np.array_equal(kg[kp:], kg[:kp] + half)
        check_selection(kg[:kp], ko[:kp], sc[g], kp, f"pairs group {g}")
        for j in range(grp):
            h = g * grp + j
            assert np.array_equal(gi[h * kh:(h + 1) * kh] - h * hd, kg)


@pytest.mark.parametrize("heads,kv", [(6, 6), (8, 2)])
@pytest.mark.parametrize("s", [0.0, 0.5, 0.9])
def test_l2_norm_criterion(L, heads, kv, s):
    tok = _tok(3, 40, [30, 40, 5])
    d, hd, r = 64, 64, 8
    X = synth.round_bf16(synth.gaussian((tok.T, d), 1.0, 860))
    Lv, Uv = _factors(kv * hd, d, r, 861)
    io, iv, ko, so = O.estimate_select_l2(X, tok.batch, tok.seq, tok.ctx_len, Lv, Uv, heads, kv,
                                          hd, s)
    k, gi, gs = _run(L, L.CRIT_L2, X, tok, Lv, Uv, None, None, r, s, (heads + kv) * hd, kv * hd,
                     heads=heads, kv_heads=kv, head_dim=hd)
    assert k == ko
    assert rel_frob(gs, so.ravel()) < SCORE_TOL
    grp = heads // kv
    for g in range(kv):
        vg = gi[heads * k + g * k: heads * k + (g + 1) * k] - g * hd
        check_selection(vg, iv[g * k:(g + 1) * k] - g * hd, so[g], k, f"l2 value head {g}")
        for h in range(g * grp, (g + 1) * grp):
            assert np.array_equal(gi[h * k:(h + 1) * k] - h * hd, vg)


@pytest.mark.parametrize("n", [1025, 3000, 11008, 16384, 16385, 32768])
@pytest.mark.parametrize("distinct", [7, 0])
def test_long_list_select_is_the_exact_top_k_of_its_scores(L, n, distinct):
    """Selection from one long score list (every register-row template of the
    top-k block): the kept set must be exactly the top-k of the GPU's own
    scores with ties to the lower index.  With `distinct` > 0 every channel's
    factor rows come from that many base rows, so the scores take only that
    many values and tie bit for bit (same rows, same arithmetic), thousands
    of keys equal to the threshold spread over all rows; 0 draws every row."""
    tok = _tok(1, 48, [40])
    d, r = 32, 4
    rg = synth.rng(880 + n + distinct)
    X = synth.round_bf16(rg.standard_normal((tok.T, d)))
    Lg, Lu = rg.standard_normal((d, r)), rg.standard_normal((d, r))
    if distinct:
        pick = rg.integers(0, distinct, size=n)
        Ug = rg.standard_normal((distinct, r))[pick]
        Uu = rg.standard_normal((distinct, r))[pick]
    else:
        Ug, Uu = rg.standard_normal((n, r)), rg.standard_normal((n, r))
    for s in (0.01, 0.5, 0.93):
        k, gi, gs = _run(L, L.CRIT_FFN_GRAM, X, tok, Lg, Ug, Lu, Uu, r, s, n, n)
        assert k == O.keep_count(n, s)
        assert gi[:k].tolist() == O.topk_select(gs.astype(np.float64), k).tolist(), \
            f"n={n} s={s}"


def test_long_list_select_all_scores_equal(L):
    """No context token: all 11008 scores are 0 and the lowest k indices are
    kept (the top-k's all-keys-equal path)."""
    tok = _tok(2, 16, [0, 0])
    d, n, r = 32, 11008, 4
    rg = synth.rng(890)
    X = synth.round_bf16(rg.standard_normal((tok.T, d)))
    Lg, Lu = rg.standard_normal((d, r)), rg.standard_normal((d, r))
    Ug, Uu = rg.standard_normal((n, r)), rg.standard_normal((n, r))
    k, gi, gs = _run(L, L.CRIT_FFN, X, tok, Lg, Ug, Lu, Uu, r, 0.3, n, n)
    assert np.all(gs == 0.0)
    assert gi[:k].tolist() == list(range(k))


def test_exact_ties_go_to_the_lower_index(L):
    """Channels with identical factor rows get bit-identical scores on both
    sides, so the kept set must equal the oracle's exactly (ties to the lower
    index), per head."""
    tok = _tok(2, 32, [24, 30])
    d, H, hd, r = 32, 2, 64, 4
    rg = synth.rng(870)
    X = synth.round_bf16(rg.standard_normal((tok.T, d)))
    Lv = rg.standard_normal((d, r))
    base = rg.standard_normal((8, r))
    Uv = np.concatenate([base[rg.integers(0, 8, size=hd)] for _ in range(H)])  # 8 distinct rows
    for s in (0.25, 0.5, 0.9):
        io, iv, ko, so = O.estimate_select_l2(X, tok.batch, tok.seq, tok.ctx_len, Lv, Uv, H, H,
                                              hd, s)
        k, gi, gs = _run(L, L.CRIT_L2, X, tok, Lv, Uv, None, None, r, s, 2 * H * hd, H * hd,
                         heads=H, kv_heads=H, head_dim=hd)
        assert k == ko
        for h in range(H):
            sg = gs[h * hd:(h + 1) * hd]
            rows = Uv[h * hd:(h + 1) * hd]
            for a in range(hd):  # equal rows -> equal GPU scores, bit for bit
                same = np.all(rows == rows[a], axis=1)
                assert np.all(sg[same] == sg[a])
            # the GPU set is the top-k of its own scores, ties to the lower index
            want = O.topk_select(sg.astype(np.float64), k)
            assert gi[h * k:(h + 1) * k].tolist() == (h * hd + want).tolist()


# ------------------------------------------------------- prepare, full size
@pytest.mark.parametrize("n,k", [(11008, 4096), (4096, 11008)])
def test_svd_prepare_benchmark_shapes(L, n, k):
    """slora_svd_prepare on the Llama-2-7B FFN weight shapes at rank 8 (the
    factors the benchmark's estimator uses): the rank-8 product matches the
    oracle's truncated SVD of the same bf16 weight to 1e-5, U has orthonormal
    columns, and the transposed copy is exact."""
    r = 8
    sw = synth.decaying_weight(n, k, seed=1000 + n, bf16=True)
    Lo, Uo = O.svd_prepare(sw.W, r)
    W = dev(sw.W, torch.bfloat16)
    Lg = torch.zeros(k, r, device="cuda")
    Ug = torch.zeros(n, r, device="cuda")
    Wt = torch.zeros(k, n, device="cuda", dtype=torch.bfloat16)
    L.slora_svd_prepare(W, r, Lg, Ug, W_t=Wt, seed=7)
    torch.cuda.synchronize()
    got = host(Ug) @ host(Lg).T
    want = Uo @ Lo.T
    assert rel_frob(got, want) < 1e-5
    np.testing.assert_allclose(host(Ug).T @ host(Ug), np.eye(r), atol=1e-5)
    assert torch.equal(Wt, W.t().contiguous())


def test_estimate_select_with_prepared_factors_full_size(L):
    """The benchmark's estimator inputs: Llama-2-7B gate/up factors from
    slora_svd_prepare, 3072 context tokens.  The GPU's scores match the
    oracle's scores computed from the oracle's own SVD factors."""
    tok = synth.Tokens.uniform(8, 512, 0.25)
    d, d_ff, r = 4096, 11008, 8
    X = synth.round_bf16(synth.gaussian((tok.T, d), 1.0, 880))
    fac_o, fac_g = [], []
    for m in range(2):
        sw = synth.decaying_weight(d_ff, d, seed=881 + m, bf16=True)
        fac_o.append(O.svd_prepare(sw.W, r))
        Lg = torch.zeros(d, r, device="cuda")
        Ug = torch.zeros(d_ff, r, device="cuda")
        L.slora_svd_prepare(dev(sw.W, torch.bfloat16), r, Lg, Ug, seed=7)
        fac_g.append((Lg, Ug))
    (Lgo, Ugo), (Luo, Uuo) = fac_o
    io, ko, so = O.estimate_select_ffn(X, tok.batch, tok.seq, tok.ctx_len, Lgo, Ugo, Luo, Uuo, 0.5)
    idx = torch.full((d_ff,), -1, dtype=torch.int32, device="cuda")
    scores = torch.zeros(d_ff, device="cuda")
    (Lg, Ug), (Lu, Uu) = fac_g
    k = L.slora_estimate_select(L.CRIT_FFN, dev(X, torch.bfloat16), tok.batch, tok.seq,
                                tok.ctx_len, Lg, Ug, Lu, Uu, r, 0.5, idx, scores_out=scores)
    torch.cuda.synchronize()
    assert k == ko
    assert rel_frob(host(scores), so) < SCORE_TOL
    check_selection(host(idx)[:k], io, so, k, "ffn full size, prepared factors")

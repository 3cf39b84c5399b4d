"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Sizes are small enough for the oracle to finish in seconds while still
spanning several tiles and a ragged tail.  Outputs and gradients are compared
on the SAME channel set (the oracle's, passed to the GPU), selections are
compared set-against-set with the near-tie rule.
"""
import numpy as np
import pytest
import torch

from oracle import slora_oracle as O
from contextual_sparsity_lora_svd_b200 import synth
from tests.helpers import TOL, assert_close, check_selection, dev, host, rel_frob, tdtype

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    from contextual_sparsity_lora_svd_b200 import _lib
    assert torch.cuda.is_available()
    return _lib


def _tok(batch, seq, ctx):
    return synth.Tokens(batch, seq, np.asarray(ctx, np.int32))


# ------------------------------------------------------------------ prepare
@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("n,k,r", [(200, 96, 8), (96, 264, 4), (40, 24, 24)])
def test_svd_prepare(L, bf16, n, k, r):
    sw = synth.decaying_weight(n, k, seed=300 + n, bf16=bf16)
    Lo, Uo = O.svd_prepare(sw.W, r)
    dt = tdtype(bf16)
    W = dev(sw.W, dt)
    Lg = torch.zeros(k, r, device="cuda")
    Ug = torch.zeros(n, r, device="cuda")
    Wt = torch.zeros(k, n, device="cuda", dtype=dt)
    L.slora_svd_prepare(W, r, Lg, Ug, W_t=Wt, seed=5)
    torch.cuda.synchronize()
    assert_close(host(Ug) @ host(Lg).T, Uo @ Lo.T, 2e-5, "rank-r product")
    np.testing.assert_allclose(host(Ug).T @ host(Ug), np.eye(r), atol=1e-5)
    assert torch.equal(Wt, W.t().contiguous())


# ---------------------------------------------------------- estimate/select
def _ffn_est_inputs(bf16, tok, d, d_ff, r, seed):
    X = synth.gaussian((tok.T, d), 1.0, seed)
    if bf16:
        X = synth.round_bf16(X)
    fac = []
    for m in range(2):
        sw = synth.decaying_weight(d_ff, d, seed + 1 + m, bf16=bf16)
        fac.append(O.svd_prepare(sw.W, r))
    return X, fac


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("s", [0.0, 0.5, 0.9])
def test_estimate_select_ffn(L, bf16, s):
    tok = _tok(3, 40, [30, 17, 40])
    d, d_ff, r = 64, 200, 8
    X, ((Lg, Ug), (Lu, Uu)) = _ffn_est_inputs(bf16, tok, d, d_ff, r, 400)
    idx_o, k_o, sc_o = O.estimate_select_ffn(X, tok.batch, tok.seq, tok.ctx_len, Lg, Ug, Lu, Uu, s)
    idx = torch.full((d_ff,), -1, dtype=torch.int32, device="cuda")
    scores = torch.zeros(d_ff, device="cuda")
    f = lambda a: dev(a, torch.float32)
    k = L.slora_estimate_select(L.CRIT_FFN, dev(X, tdtype(bf16)), tok.batch, tok.seq, tok.ctx_len,
                                f(Lg), f(Ug), f(Lu), f(Uu), r, s, idx, scores_out=scores)
    torch.cuda.synchronize()
    assert k == k_o
    assert rel_frob(host(scores), sc_o) < 1e-5
    check_selection(host(idx)[:k], idx_o, sc_o, k, "ffn select")


@pytest.mark.parametrize("heads,kv", [(4, 4), (8, 2)])
@pytest.mark.parametrize("s", [0.5, 0.25])
def test_estimate_select_qk(L, heads, kv, s):
    tok = _tok(2, 48, [36, 20])
    d, hd, r = 64, 32, 8
    X = synth.round_bf16(synth.gaussian((tok.T, d), 1.0, 500))
    (Lq, Uq) = O.svd_prepare(synth.decaying_weight(heads * hd, d, 501, bf16=True).W, r)
    (Lk, Uk) = O.svd_prepare(synth.decaying_weight(kv * hd, d, 502, bf16=True).W, r)
    iq, ik, kh, sc = O.estimate_select_qk(X, tok.batch, tok.seq, tok.ctx_len, Lq, Uq, Lk, Uk,
                                          heads, kv, hd, s)
    idx = torch.full(((heads + kv) * hd,), -1, dtype=torch.int32, device="cuda")
    scores = torch.zeros(kv * hd, device="cuda")
    f = lambda a: dev(a, torch.float32)
    k = L.slora_estimate_select(L.CRIT_QK, dev(X, torch.bfloat16), tok.batch, tok.seq,
                                tok.ctx_len, f(Lq), f(Uq), f(Lk), f(Uk), r, s, idx,
                                heads=heads, kv_heads=kv, head_dim=hd, scores_out=scores)
    torch.cuda.synchronize()
    assert k == kh
    assert rel_frob(host(scores), sc.ravel()) < 1e-5
    gi = host(idx).astype(np.int64)
    grp = heads // kv
    for g in range(kv):
        local_g = gi[(heads + g) * 0 + heads * kh + g * kh: heads * kh + (g + 1) * kh] - g * hd
        local_o = ik[g * kh:(g + 1) * kh] - g * hd
        check_selection(local_g, local_o, sc[g], kh, f"group {g}")
        for j in range(grp):
            h = g * grp + j
            assert np.array_equal(gi[h * kh:(h + 1) * kh] - h * hd, local_g)


# ------------------------------------------------------------------ linear
def _lin(bf16, tok, k, n, r, seed):
    rnd = synth.round_bf16 if bf16 else (lambda a: a)
    X = rnd(synth.gaussian((tok.T, k), 1.0, seed))
    W0 = rnd(synth.gaussian((n, k), 0.05, seed + 1))
    A = rnd(synth.gaussian((r, k), 0.05, seed + 2))
    B = rnd(synth.gaussian((n, r), 0.05, seed + 3))
    return X, W0, A, B


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("side", ["none", "out_rows", "in_cols"])
def test_linear_fwd_bwd(L, bf16, side):
    tok = _tok(3, 50, [37, 50, 8])
    k, n, r, s = 136, 200, 8, 0.7
    X, W0, A, B = _lin(bf16, tok, k, n, r, 600)
    C, Orow = O.context_rows(tok.batch, tok.seq, tok.ctx_len)
    rg = synth.rng(601)
    lim = n if side == "out_rows" else k
    idx_o = np.sort(rg.choice(lim, size=lim // 2 + 3, replace=False))
    dt = tdtype(bf16)
    tol = TOL["bf16" if bf16 else "f32"]
    code = {"none": L.SLICE_NONE, "out_rows": L.SLICE_OUT_ROWS, "in_cols": L.SLICE_IN_COLS}[side]
    idx = dev(idx_o, torch.int32) if side != "none" else None
    if side == "in_cols":
        Xin, Xout = X[C][:, idx_o], X[Orow]
        Wdev = dev(W0.T.copy(), dt)
    else:
        Xin, Xout = X, None
        Wdev = dev(W0, dt)
    Yc_o, Yo_o, XA_o = O.linear_fwd(side, Xin, Xout, tok.batch, tok.seq, tok.ctx_len, W0, A, B, s,
                                    idx_o if side != "none" else None)
    Yc = torch.zeros(Yc_o.shape, dtype=dt, device="cuda")
    Yo = torch.zeros(Yo_o.shape, dtype=dt, device="cuda") if Yo_o is not None else None
    XA = torch.zeros(tok.T, r, device="cuda")
    Xin_d = dev(Xin, dt)
    Xout_d = dev(Xout, dt) if Xout is not None else None
    L.slora_linear_fwd(code, tok.batch, tok.seq, tok.ctx_len, k, n, Wdev, dev(A, dt), dev(B, dt), s,
                       idx, Xin_d, Yc, X_out=Xout_d, Y_out=Yo, XA_save=XA)
    torch.cuda.synchronize()
    assert_close(host(Yc), Yc_o, tol, "Y_ctx")
    if Yo is not None:
        assert_close(host(Yo), Yo_o, tol, "Y_out")
    assert_close(host(XA), XA_o, tol, "XA")
    # backward
    dY1 = rg.standard_normal(Yc_o.shape)
    dY2 = rg.standard_normal(Yo_o.shape) if Yo_o is not None else None
    if bf16:
        dY1 = synth.round_bf16(dY1)
        dY2 = synth.round_bf16(dY2) if dY2 is not None else None
    dXc_o, dXo_o, dA_o, dB_o = O.linear_bwd(side, Xin, Xout, XA_o, dY1, dY2, tok.batch, tok.seq,
                                            tok.ctx_len, W0, A, B, s,
                                            idx_o if side != "none" else None)
    dXc = torch.zeros(dXc_o.shape, dtype=dt, device="cuda")
    dXo = torch.zeros(dXo_o.shape, dtype=dt, device="cuda") if dXo_o is not None else None
    dA = torch.zeros(r, k, device="cuda")
    dB = torch.zeros(n, r, device="cuda")
    L.slora_linear_bwd(code, tok.batch, tok.seq, tok.ctx_len, k, n, Wdev, dev(A, dt), dev(B, dt), s,
                       idx, Xin_d, XA, dev(dY1, dt), dXc, dA, dB, X_out=Xout_d,
                       dY_out=dev(dY2, dt) if dY2 is not None else None, dX_out=dXo)
    torch.cuda.synchronize()
    assert_close(host(dXc), dXc_o, tol, "dX_ctx")
    if dXo is not None:
        assert_close(host(dXo), dXo_o, tol, "dX_out")
    assert_close(host(dA), dA_o, tol, "dA")
    assert_close(host(dB), dB_o, tol, "dB")


def test_linear_fwd_bwd_single_tile(L):
    """Every slice side with 128 rows in total (one M tile) and widths that are
    whole multiples of the tile: k = n = 128."""
    tok = _tok(2, 64, [48, 40])
    k, n, r, s = 128, 128, 8, 1.0
    X, W0, A, B = _lin(True, tok, k, n, r, 650)
    C, Orow = O.context_rows(tok.batch, tok.seq, tok.ctx_len)
    idx_o = np.sort(synth.rng(651).choice(n, size=64, replace=False))
    bf = torch.bfloat16
    for side in ("none", "out_rows", "in_cols"):
        code = {"none": L.SLICE_NONE, "out_rows": L.SLICE_OUT_ROWS,
                "in_cols": L.SLICE_IN_COLS}[side]
        sel = None if side == "none" else idx_o
        if side == "in_cols":
            Xin, Xout, Wdev = X[C][:, idx_o], X[Orow], dev(W0.T.copy(), bf)
        else:
            Xin, Xout, Wdev = X, None, dev(W0, bf)
        Yc_o, Yo_o, XA_o = O.linear_fwd(side, Xin, Xout, tok.batch, tok.seq, tok.ctx_len, W0, A, B,
                                        s, sel)
        Yc = torch.zeros(Yc_o.shape, dtype=bf, device="cuda")
        Yo = torch.zeros(Yo_o.shape, dtype=bf, device="cuda") if Yo_o is not None else None
        XA = torch.zeros(tok.T, r, device="cuda")
        idx = dev(sel, torch.int32) if sel is not None else None
        Xin_d, Xout_d = dev(Xin, bf), (dev(Xout, bf) if Xout is not None else None)
        L.slora_linear_fwd(code, tok.batch, tok.seq, tok.ctx_len, k, n, Wdev, dev(A, bf),
                           dev(B, bf), s, idx, Xin_d, Yc, X_out=Xout_d, Y_out=Yo, XA_save=XA)
        rg = synth.rng(652)
        dY1 = synth.round_bf16(rg.standard_normal(Yc_o.shape))
        dY2 = synth.round_bf16(rg.standard_normal(Yo_o.shape)) if Yo_o is not None else None
        dXc_o, dXo_o, dA_o, dB_o = O.linear_bwd(side, Xin, Xout, XA_o, dY1, dY2, tok.batch,
                                                tok.seq, tok.ctx_len, W0, A, B, s, sel)
        dXc = torch.zeros(dXc_o.shape, dtype=bf, device="cuda")
        dXo = torch.zeros(dXo_o.shape, dtype=bf, device="cuda") if dXo_o is not None else None
        dA, dB = torch.zeros(r, k, device="cuda"), torch.zeros(n, r, device="cuda")
        L.slora_linear_bwd(code, tok.batch, tok.seq, tok.ctx_len, k, n, Wdev, dev(A, bf),
                           dev(B, bf), s, idx, Xin_d, XA, dev(dY1, bf), dXc, dA, dB, X_out=Xout_d,
                           dY_out=dev(dY2, bf) if dY2 is not None else None, dX_out=dXo)
        torch.cuda.synchronize()
        tol = TOL["bf16"]
        assert_close(host(Yc), Yc_o, tol, f"{side} Y_ctx")
        if Yo is not None:
            assert_close(host(Yo), Yo_o, tol, f"{side} Y_out")
        assert_close(host(dXc), dXc_o, tol, f"{side} dX_ctx")
        if dXo is not None:
            assert_close(host(dXo), dXo_o, tol, f"{side} dX_out")
        assert_close(host(dA), dA_o, tol, f"{side} dA")
        assert_close(host(dB), dB_o, tol, f"{side} dB")


# --------------------------------------------------------------------- FFN
def _ffn_lay(case, r_svd):
    lay = dict(Wg=case.Wg.W, Wu=case.Wu.W, Wd=case.Wd.W, Ag=case.Ag, Bg=case.Bg, Au=case.Au,
               Bu=case.Bu, Ad=case.Ad, Bd=case.Bd, scale=case.lora_scale)
    lay["Lg"], lay["Ug"] = O.svd_prepare(case.Wg.W, r_svd)
    lay["Lu"], lay["Uu"] = O.svd_prepare(case.Wu.W, r_svd)
    return lay


def run_ffn_gpu(L, case, lay, idx_force=None):
    dt = tdtype(case.bf16)
    d, F, r = case.d, case.d_ff, case.r_lora
    t = {k: dev(lay[k], dt) for k in ("Wg", "Wu", "Ag", "Bg", "Au", "Bu", "Ad", "Bd")}
    t["Wd_t"] = dev(lay["Wd"].T.copy(), dt)
    for k in ("Lg", "Ug", "Lu", "Uu"):
        t[k] = dev(lay[k], torch.float32)
    layer = L.ffn_layer_struct(d, F, lay["Lg"].shape[1], r, case.lora_scale, t["Wg"], t["Wu"],
                               t["Wd_t"], t["Ag"], t["Bg"], t["Au"], t["Bu"], t["Ad"], t["Bd"],
                               t["Lg"], t["Ug"], t["Lu"], t["Uu"])
    T = case.tokens.T
    X, dOut = dev(case.X, dt), dev(case.dOut, dt)
    out = torch.zeros(T, d, dtype=dt, device="cuda")
    dX = torch.zeros(T, d, dtype=dt, device="cuda")
    g = {k: torch.zeros(sh, device="cuda") for k, sh in
         (("dAg", (r, d)), ("dBg", (F, r)), ("dAu", (r, d)), ("dBu", (F, r)), ("dAd", (r, F)),
          ("dBd", (d, r)))}
    grads = L.ffn_grads_struct(g["dAg"], g["dBg"], g["dAu"], g["dBu"], g["dAd"], g["dBd"])
    idx = torch.full((F,), -1, dtype=torch.int32, device="cuda")
    force = dev(np.asarray(idx_force), torch.int32) if idx_force is not None else None
    k = L.slora_ffn_fwd_bwd(layer, case.tokens.batch, case.tokens.seq, case.tokens.ctx_len,
                            case.sparsity, X, dOut, out, dX, grads, idx, idx_force=force)
    torch.cuda.synchronize()
    res = {kk: host(v) for kk, v in g.items()}
    res.update(out=host(out), dX=host(dX), idx=host(idx)[:k].astype(np.int64), k=k)
    return res


def _compare_ffn(res, ref, tol):
    for key in ("out", "dX", "dAg", "dBg", "dAu", "dBu", "dAd", "dBd"):
        assert_close(res[key], ref[key], tol, key)


@pytest.mark.parametrize("bf16", [False, True])
def test_ffn_workload0_full(L, bf16):
    """Workload 0 at its full size (T=256, d=256, d_ff=688), fp32 and bf16."""
    w = synth.WORKLOADS[0]
    tok = synth.Tokens.uniform(w["batch"], w["seq"], w["out_frac"])
    case = synth.ffn_case(tok, w["d"], w["d_ff"], w["r_svd"], w["r_lora"], w["sparsity"],
                          bf16=bf16, workload=0)
    lay = _ffn_lay(case, w["r_svd"])
    ref = O.ffn_fwd_bwd(case.X, case.dOut, tok.batch, tok.seq, tok.ctx_len, lay, case.sparsity)
    tol = TOL["bf16" if bf16 else "f32"]
    # (1) the GPU's own estimator + selection
    res = run_ffn_gpu(L, case, lay)
    assert res["k"] == ref["k"] == 344
    nd = check_selection(res["idx"], ref["idx"], ref["scores"], ref["k"], "ffn select")
    if nd == 0:
        _compare_ffn(res, ref, tol)
    # (2) the oracle's channel set forced on the GPU
    res2 = run_ffn_gpu(L, case, lay, idx_force=ref["idx"])
    assert np.array_equal(res2["idx"], ref["idx"])
    _compare_ffn(res2, ref, tol)


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("ctx", [[70, 33, 90], [90, 90, 90], [0, 0, 0], [1, 0, 89]])
def test_ffn_ragged_and_edges(L, bf16, ctx):
    """Ragged context lengths, no output rows, no context rows."""
    tok = _tok(3, 90, ctx)
    case = synth.ffn_case(tok, 72, 152, 6, 5, 0.3, bf16=bf16, workload=0, layer=3,
                          lora_scale=0.5)
    lay = _ffn_lay(case, 6)
    ref = O.ffn_fwd_bwd(case.X, case.dOut, tok.batch, tok.seq, tok.ctx_len, lay, case.sparsity)
    res = run_ffn_gpu(L, case, lay, idx_force=ref["idx"])
    _compare_ffn(res, ref, TOL["bf16" if bf16 else "f32"])
    if tok.T_O == 0:
        skip = np.setdiff1d(np.arange(case.d_ff), ref["idx"])
        assert np.all(res["dBg"][skip] == 0) and np.all(res["dBu"][skip] == 0)
        assert np.all(res["dAd"][:, skip] == 0)


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("s", [0.0, 0.99])
def test_ffn_sparsity_extremes(L, s, bf16):
    """Every channel kept, and one or two kept: in bf16 the context-row GEMMs then
    have N below one 32-channel epilogue chunk (clipped TMA boxes and stores)."""
    tok = _tok(2, 64, [48, 48])
    case = synth.ffn_case(tok, 64, 136, 8, 4, s, bf16=bf16, workload=0, layer=4)
    lay = _ffn_lay(case, 8)
    ref = O.ffn_fwd_bwd(case.X, case.dOut, tok.batch, tok.seq, tok.ctx_len, lay, s)
    tol = TOL["bf16" if bf16 else "f32"]
    res = run_ffn_gpu(L, case, lay)
    assert res["k"] == ref["k"]
    nd = check_selection(res["idx"], ref["idx"], ref["scores"], ref["k"], "select")
    if nd == 0:
        _compare_ffn(res, ref, tol)
    res2 = run_ffn_gpu(L, case, lay, idx_force=ref["idx"])
    _compare_ffn(res2, ref, tol)

"""GPU parity of the layer runners (contextual_sparsity_lora_svd_b200.layers)
that the benchmark's attention, stack and Llama-3 workloads time: one step of
the q/k/v/o linears (q/k sliced by QK-norm or rotate-half pairs, v/o dense or
sliced by the per-head L2 estimate, grouped-query heads) and one FFN layer
(sparse and dense), each output and gradient compared with the oracle on the
channel sets the GPU selected, and those sets compared with the oracle's
selection (near-tie rule)."""
import numpy as np
import pytest
import torch

from oracle import slora_oracle as O
from contextual_sparsity_lora_svd_b200 import synth
from tests.helpers import TOL, assert_close, check_selection, dev, host

pytestmark = pytest.mark.gpu
TOL_BF16 = TOL["bf16"]


@pytest.fixture(scope="module")
def L():
    from contextual_sparsity_lora_svd_b200 import _lib
    return _lib


def _bf(a):
    return dev(a, torch.bfloat16)


def _attn_case(H, KV, hd, d, r_svd, r_lora, tok, seed):
    rnd = synth.round_bf16
    nq, nkv = H * hd, KV * hd
    W = {"q": synth.decaying_weight(nq, d, seed + 1, bf16=True).W,
         "k": synth.decaying_weight(nkv, d, seed + 2, bf16=True).W,
         "v": synth.decaying_weight(nkv, d, seed + 3, bf16=True).W,
         "o": synth.decaying_weight(d, nq, seed + 4, bf16=True).W}
    A = {m: rnd(synth.gaussian((r_lora, W[m].shape[1]), 0.05, seed + 10 + i))
         for i, m in enumerate(W)}
    B = {m: rnd(synth.gaussian((W[m].shape[0], r_lora), 0.05, seed + 20 + i))
         for i, m in enumerate(W)}
    fac = {m: O.svd_prepare(W[m], r_svd) for m in ("q", "k", "v")}
    X = rnd(synth.gaussian((tok.T, d), 1.0, seed + 30))
    attn = rnd(synth.gaussian((tok.T, nq), 1.0, seed + 31))
    dYo = rnd(synth.gaussian((tok.T, d), 1.0, seed + 32))
    dq = rnd(synth.gaussian((tok.T, nq), 1.0, seed + 33))
    dk = rnd(synth.gaussian((tok.T, nkv), 1.0, seed + 34))
    dv = rnd(synth.gaussian((tok.T, nkv), 1.0, seed + 35))
    return W, A, B, fac, X, attn, dYo, dq, dk, dv


@pytest.mark.parametrize("H,KV,pairs,vo", [(4, 4, False, 0.0), (4, 2, True, 0.5),
                                           (6, 3, False, 0.5)])
def test_attention_linears_step(L, H, KV, pairs, vo):
    from contextual_sparsity_lora_svd_b200.layers import AttnLinears
    tok = synth.Tokens(2, 64, np.array([48, 40], np.int32))
    hd, d, rs, r, s = 32, 128, 4, 8, 0.5
    W, A, B, fac, X, attn, dYo, dq, dk, dv = _attn_case(H, KV, hd, d, rs, r, tok, 7000 + H)
    w = {"W" + m: _bf(W[m]) for m in W}
    w["Wo_t"] = _bf(W["o"].T.copy())
    for m in W:
        w["A" + m], w["B" + m] = _bf(A[m]), _bf(B[m])
    for m in fac:
        w["L" + m], w["U" + m] = dev(fac[m][0], torch.float32), dev(fac[m][1], torch.float32)
    run = AttnLinears(w, d, H, KV, hd, rs, r, 1.0, tok.batch, tok.seq, tok.ctx_len, s,
                      _bf(X), _bf(attn), _bf(dYo), _bf(dq), _bf(dk), _bf(dv), pairs=pairs,
                      vo_sparsity=vo)
    ws = torch.empty(run.workspace_bytes(), dtype=torch.uint8, device="cuda")
    # the four projections run as parallel branches; issued one after another
    # (the profiling mode) they must give the same bits
    run.serial = True
    run.step(ws)
    torch.cuda.synchronize()
    serial = [host(t).copy() for t in run.dX.values()] + [host(run.gflat).copy()]
    run.serial = False
    run.gflat.zero_()
    run.step(ws)
    torch.cuda.synchronize()
    par = [host(t) for t in run.dX.values()] + [host(run.gflat)]
    for a, b in zip(serial, par):
        assert np.array_equal(a, b), "parallel branches changed the result"
    C, Orow = O.context_rows(tok.batch, tok.seq, tok.ctx_len)
    # q/k selection against the oracle's
    est = O.estimate_select_qk_pairs if pairs else O.estimate_select_qk
    iq_o, ik_o, kh, sc = est(X, tok.batch, tok.seq, tok.ctx_len, *fac["q"], *fac["k"], H, KV,
                             hd, s)
    assert run.kh == kh
    gi = host(run.idx_qk).astype(np.int64)
    iq, ik = gi[:H * kh], gi[H * kh:H * kh + KV * kh]
    kp = kh // 2 if pairs else kh
    for g in range(KV):
        loc = ik[g * kh:(g + 1) * kh] - g * hd
        check_selection(loc[:kp], (ik_o[g * kh:(g + 1) * kh] - g * hd)[:kp], sc[g], kp,
                        f"qk group {g}")
    # every linear against the oracle on the GPU's channel sets
    got_dYc = {}
    for m, sel in (("q", iq), ("k", ik)):
        Yc, Yo, dYc, dYo_, XA = (host(t) for t in run.bufs[m])
        got_dYc[m] = (dYc, dYo_)
        Yc_o, Yo_o, XA_o = O.linear_fwd("out_rows", X, None, tok.batch, tok.seq, tok.ctx_len,
                                        W[m], A[m], B[m], 1.0, sel)
        dX_o, _, dA_o, dB_o = O.linear_bwd("out_rows", X, None, XA_o, dYc, dYo_, tok.batch,
                                           tok.seq, tok.ctx_len, W[m], A[m], B[m], 1.0, sel)
        assert_close(Yc, Yc_o, TOL_BF16, f"{m} Y_ctx")
        assert_close(Yo, Yo_o, TOL_BF16, f"{m} Y_out")
        assert_close(XA, XA_o, TOL_BF16, f"{m} XA")
        assert_close(host(run.dX[m]), dX_o, TOL_BF16, f"{m} dX")
        assert_close(host(run.grads["dA" + m]), dA_o, TOL_BF16, f"{m} dA")
        assert_close(host(run.grads["dB" + m]), dB_o, TOL_BF16, f"{m} dB")
    if vo > 0:
        io_o, iv_o, kv, scv = O.estimate_select_l2(X, tok.batch, tok.seq, tok.ctx_len, *fac["v"],
                                                   H, KV, hd, vo)
        gv = host(run.idx_vo).astype(np.int64)
        io, iv = gv[:H * kv], gv[H * kv:H * kv + KV * kv]
        for g in range(KV):
            check_selection(iv[g * kv:(g + 1) * kv] - g * hd, iv_o[g * kv:(g + 1) * kv] - g * hd,
                            scv[g], kv, f"v group {g}")
        Yc, Yo, dYc, dYo_, XAv = (host(t) for t in run.bufs["v"])
        Yc_o, Yo_o, XA_o = O.linear_fwd("out_rows", X, None, tok.batch, tok.seq, tok.ctx_len,
                                        W["v"], A["v"], B["v"], 1.0, iv)
        dX_o, _, dA_o, dB_o = O.linear_bwd("out_rows", X, None, XA_o, dYc, dYo_, tok.batch,
                                           tok.seq, tok.ctx_len, W["v"], A["v"], B["v"], 1.0, iv)
        assert_close(Yc, Yc_o, TOL_BF16, "v Y_ctx")
        assert_close(host(run.dX["v"]), dX_o, TOL_BF16, "v dX")
        assert_close(host(run.grads["dAv"]), dA_o, TOL_BF16, "v dA")
        assert_close(host(run.grads["dBv"]), dB_o, TOL_BF16, "v dB")
        Xoc, Xoo, Yof, XAo, dXoc, dXoo = (host(t) for t in run.bufs["o"])
        Y_o, _, XA_oo = O.linear_fwd("in_cols", Xoc, Xoo, tok.batch, tok.seq, tok.ctx_len, W["o"],
                                     A["o"], B["o"], 1.0, io)
        dXc_o, dXo_o, dA_o, dB_o = O.linear_bwd("in_cols", Xoc, Xoo, XA_oo, dYo, None, tok.batch,
                                                tok.seq, tok.ctx_len, W["o"], A["o"], B["o"], 1.0,
                                                io)
        assert_close(Yof, Y_o, TOL_BF16, "o Y")
        assert_close(dXoc, dXc_o, TOL_BF16, "o dX_ctx")
        assert_close(dXoo, dXo_o, TOL_BF16, "o dX_out")
        assert_close(host(run.grads["dAo"]), dA_o, TOL_BF16, "o dA")
        assert_close(host(run.grads["dBo"]), dB_o, TOL_BF16, "o dB")
    else:
        Yv, XAv = (host(t) for t in run.bufs["v"])
        Yv_o, _, XAv_o = O.linear_fwd("none", X, None, tok.batch, tok.seq, tok.ctx_len, W["v"],
                                      A["v"], B["v"], 1.0, None)
        dX_o, _, dA_o, dB_o = O.linear_bwd("none", X, None, XAv_o, dv, None, tok.batch, tok.seq,
                                           tok.ctx_len, W["v"], A["v"], B["v"], 1.0, None)
        assert_close(Yv, Yv_o, TOL_BF16, "v Y")
        assert_close(host(run.dX["v"]), dX_o, TOL_BF16, "v dX")
        assert_close(host(run.grads["dBv"]), dB_o, TOL_BF16, "v dB")
        Yof, XAo, dXo = (host(t) for t in run.bufs["o"])
        Y_o, _, XA_oo = O.linear_fwd("none", attn, None, tok.batch, tok.seq, tok.ctx_len, W["o"],
                                     A["o"], B["o"], 1.0, None)
        dX_o, _, dA_o, dB_o = O.linear_bwd("none", attn, None, XA_oo, dYo, None, tok.batch,
                                           tok.seq, tok.ctx_len, W["o"], A["o"], B["o"], 1.0,
                                           None)
        assert_close(Yof, Y_o, TOL_BF16, "o Y")
        assert_close(dXo, dX_o, TOL_BF16, "o dX")
        assert_close(host(run.grads["dAo"]), dA_o, TOL_BF16, "o dA")


@pytest.mark.parametrize("s", [0.0, 0.6])
def test_ffn_layer_runner_step(L, s):
    """FfnLayer: at s = 0 every channel runs (no estimator); otherwise the
    GPU's selection matches the oracle's and the outputs match the oracle on
    the GPU's set."""
    from contextual_sparsity_lora_svd_b200.layers import FfnLayer
    tok = synth.Tokens(2, 96, np.array([70, 96], np.int32))
    case = synth.ffn_case(tok, d=128, d_ff=344, r_svd=8, r_lora=8, sparsity=s, bf16=True,
                          workload=0, layer=5)
    lay = dict(Wg=case.Wg.W, Wu=case.Wu.W, Wd=case.Wd.W, Ag=case.Ag, Bg=case.Bg, Au=case.Au,
               Bu=case.Bu, Ad=case.Ad, Bd=case.Bd, scale=1.0)
    lay["Lg"], lay["Ug"] = O.svd_prepare(case.Wg.W, 8)
    lay["Lu"], lay["Uu"] = O.svd_prepare(case.Wu.W, 8)
    w = {k: _bf(lay[k]) for k in ("Wg", "Wu", "Ag", "Bg", "Au", "Bu", "Ad", "Bd")}
    w["Wd_t"] = _bf(lay["Wd"].T.copy())
    for k in ("Lg", "Ug", "Lu", "Uu"):
        w[k] = dev(lay[k], torch.float32)
    run = FfnLayer(w, 128, 344, 8, 8, 1.0, tok.batch, tok.seq, tok.ctx_len, s, _bf(case.X),
                   _bf(case.dOut))
    ws = torch.empty(run.workspace_bytes(), dtype=torch.uint8, device="cuda")
    run.step(ws)
    torch.cuda.synchronize()
    k = run.kept()
    gi = host(run.idx)[:k].astype(np.int64)
    if s == 0.0:
        assert k == 344 and gi.tolist() == list(range(344))
    else:
        io, ko, so = O.estimate_select_ffn(case.X, tok.batch, tok.seq, tok.ctx_len, lay["Lg"],
                                           lay["Ug"], lay["Lu"], lay["Uu"], s)
        assert k == ko
        check_selection(gi, io, so, k, "ffn runner")
    out, saved = O.ffn_fwd(case.X, tok.batch, tok.seq, tok.ctx_len, lay, gi)
    grads = O.ffn_bwd(case.X, case.dOut, lay, gi, saved)
    assert_close(host(run.out), out, TOL_BF16, "out")
    assert_close(host(run.dX), grads["dX"], TOL_BF16, "dX")
    for name, g in zip(("dAg", "dBg", "dAu", "dBu", "dAd", "dBd"), run.grads):
        assert_close(host(g), grads[name], TOL_BF16, name)

"""Parity at the full workload sizes, in the launch configuration bench.py
times: the Llama-2-7B-shaped FFN layer (batch 8 x seq 512, d 4096, d_ff 11008,
25% output tokens, SVD rank 8, LoRA rank 16, sparsity 50%) and the
Llama-2-7B-shaped attention projections (batch 4 x seq 1024, 32 heads x 128,
q/k sliced at 50% per head by QK-norm; v/o dense LoRA rank 16, and the v/o
variant sliced by the per-head L2 estimate).

The estimator factors are the construction's exact top-r singular triplets
(the weights are built from them), so both sides score with the same L, U.
The oracle is run in full (tens of seconds of fp64 BLAS)."""
import numpy as np
import pytest
import torch

from oracle import slora_oracle as O
from contextual_sparsity_lora_svd_b200 import synth
from tests.helpers import TOL, assert_close, check_selection, dev, host
from tests.test_gpu_parity import _compare_ffn, run_ffn_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    from contextual_sparsity_lora_svd_b200 import _lib
    return _lib


def _factors(sw, r):
    return sw.V[:, :r] * sw.s[None, :r], sw.U[:, :r].copy()


def test_ffn_llama2_7b_full_size(L):
    w = synth.WORKLOADS[1]
    tok = synth.Tokens.uniform(w["batch"], w["seq"], w["out_frac"])
    case = synth.ffn_case(tok, w["d"], w["d_ff"], w["r_svd"], w["r_lora"], w["sparsity"],
                          bf16=True, workload=1, fast=True)
    r = w["r_svd"]
    lay = dict(Wg=case.Wg.W, Wu=case.Wu.W, Wd=case.Wd.W, Ag=case.Ag, Bg=case.Bg, Au=case.Au,
               Bu=case.Bu, Ad=case.Ad, Bd=case.Bd, scale=case.lora_scale)
    lay["Lg"], lay["Ug"] = _factors(case.Wg, r)
    lay["Lu"], lay["Uu"] = _factors(case.Wu, r)
    idx_o, k_o, sc_o = O.estimate_select_ffn(case.X, tok.batch, tok.seq, tok.ctx_len, lay["Lg"],
                                             lay["Ug"], lay["Lu"], lay["Uu"], w["sparsity"])
    assert k_o == 5504
    # the GPU's own estimator + selection
    res = run_ffn_gpu(L, case, lay)
    assert res["k"] == k_o
    check_selection(res["idx"], idx_o, sc_o, k_o, "full-size FFN select")
    # sliced fwd/bwd on the oracle's channel set
    res2 = run_ffn_gpu(L, case, lay, idx_force=idx_o)
    out, saved = O.ffn_fwd(case.X, tok.batch, tok.seq, tok.ctx_len, lay, idx_o)
    grads = O.ffn_bwd(case.X, case.dOut, lay, idx_o, saved)
    _compare_ffn(res2, dict(out=out, **grads), TOL["bf16"])


def test_attention_projections_llama2_7b_full_size(L):
    w = synth.WORKLOADS[2]
    tok = synth.Tokens.uniform(w["batch"], w["seq"], w["out_frac"])
    H, KV, hd, rs = w["heads"], w["kv_heads"], w["head_dim"], w["r_svd"]
    case = synth.qk_case(tok, w["d"], H, KV, hd, rs, w["r_lora"], w["sparsity"], bf16=True,
                         workload=2, fast=True)
    Lq, Uq = _factors(case.Wq, rs)
    Lk, Uk = _factors(case.Wk, rs)
    iq, ik, kh, sc = O.estimate_select_qk(case.X, tok.batch, tok.seq, tok.ctx_len, Lq, Uq, Lk, Uk,
                                          H, KV, hd, w["sparsity"])
    f = lambda a: dev(a, torch.float32)
    Xd = dev(case.X, torch.bfloat16)
    idx = torch.full(((H + KV) * hd,), -1, dtype=torch.int32, device="cuda")
    k = L.slora_estimate_select(L.CRIT_QK, Xd, tok.batch, tok.seq, tok.ctx_len, f(Lq), f(Uq),
                                f(Lk), f(Uk), rs, w["sparsity"], idx, heads=H, kv_heads=KV,
                                head_dim=hd)
    torch.cuda.synchronize()
    assert k == kh == 64
    gi = host(idx).astype(np.int64)
    for g in range(KV):
        check_selection(gi[H * kh + g * kh:H * kh + (g + 1) * kh] - g * hd,
                        ik[g * kh:(g + 1) * kh] - g * hd, sc[g], kh, f"head {g}")
    # q and k projections sliced on the oracle's sets, v dense (NONE)
    C, Orow = O.context_rows(tok.batch, tok.seq, tok.ctx_len)
    s = case.lora_scale
    for name, W0, A, B, sel, dY in (("q", case.Wq.W, case.Aq, case.Bq, iq, case.dYq),
                                    ("k", case.Wk.W, case.Ak, case.Bk, ik, case.dYk)):
        n, kdim = W0.shape
        Yc_o, Yo_o, XA_o = O.linear_fwd("out_rows", case.X, None, tok.batch, tok.seq,
                                        tok.ctx_len, W0, A, B, s, sel)
        dYc = synth.round_bf16(dY[C][:, sel])
        dYo = dY[Orow]
        dX_o, _, dA_o, dB_o = O.linear_bwd("out_rows", case.X, None, XA_o, dYc, dYo, tok.batch,
                                           tok.seq, tok.ctx_len, W0, A, B, s, sel)
        bf = torch.bfloat16
        Wd_, Ad_, Bd_ = dev(W0, bf), dev(A, bf), dev(B, bf)
        idx_d = dev(sel, torch.int32)
        Yc = torch.zeros(Yc_o.shape, dtype=bf, device="cuda")
        Yo = torch.zeros(Yo_o.shape, dtype=bf, device="cuda")
        XA = torch.zeros(tok.T, A.shape[0], device="cuda")
        L.slora_linear_fwd(L.SLICE_OUT_ROWS, tok.batch, tok.seq, tok.ctx_len, kdim, n, Wd_, Ad_,
                           Bd_, s, idx_d, Xd, Yc, Y_out=Yo, XA_save=XA)
        dX = torch.zeros(tok.T, kdim, dtype=bf, device="cuda")
        dA = torch.zeros(A.shape, device="cuda")
        dB = torch.zeros(B.shape, device="cuda")
        L.slora_linear_bwd(L.SLICE_OUT_ROWS, tok.batch, tok.seq, tok.ctx_len, kdim, n, Wd_, Ad_,
                           Bd_, s, idx_d, Xd, XA, dev(dYc, bf), dX, dA, dB, dY_out=dev(dYo, bf))
        torch.cuda.synchronize()
        for what, got, want in (("Y_ctx", Yc, Yc_o), ("Y_out", Yo, Yo_o), ("dX", dX, dX_o),
                                ("dA", dA, dA_o), ("dB", dB, dB_o)):
            assert_close(host(got), want, TOL["bf16"], f"{name}:{what}")


def _linear_pair(L, side, tok, X_ctx, X_out, W0, A, B, s, sel, dY_ctx, dY_out):
    """One linear's forward and backward on the GPU (bf16) and in the oracle,
    on the same channel set; returns the list of (name, got, want)."""
    bf = torch.bfloat16
    C, Orow = O.context_rows(tok.batch, tok.seq, tok.ctx_len)
    n, k = W0.shape
    code = {"none": L.SLICE_NONE, "out_rows": L.SLICE_OUT_ROWS, "in_cols": L.SLICE_IN_COLS}[side]
    Yc_o, Yo_o, XA_o = O.linear_fwd(side, X_ctx, X_out, tok.batch, tok.seq, tok.ctx_len, W0, A,
                                    B, s, sel)
    dXc_o, dXo_o, dA_o, dB_o = O.linear_bwd(side, X_ctx, X_out, XA_o, dY_ctx, dY_out, tok.batch,
                                            tok.seq, tok.ctx_len, W0, A, B, s, sel)
    Wdev = dev(W0.T.copy() if side == "in_cols" else W0, bf)
    Ad_, Bd_ = dev(A, bf), dev(B, bf)
    idx_d = dev(sel, torch.int32) if sel is not None else None
    Xc = dev(X_ctx, bf)
    Xo = dev(X_out, bf) if X_out is not None else None
    Yc = torch.zeros(Yc_o.shape, dtype=bf, device="cuda")
    Yo = torch.zeros(Yo_o.shape, dtype=bf, device="cuda") if Yo_o is not None else None
    XA = torch.zeros(tok.T, A.shape[0], device="cuda")
    L.slora_linear_fwd(code, tok.batch, tok.seq, tok.ctx_len, k, n, Wdev, Ad_, Bd_, s, idx_d, Xc,
                       Yc, X_out=Xo, Y_out=Yo, XA_save=XA)
    dXc = torch.zeros(dXc_o.shape, dtype=bf, device="cuda")
    dXo = torch.zeros(dXo_o.shape, dtype=bf, device="cuda") if dXo_o is not None else None
    dA = torch.zeros(A.shape, device="cuda")
    dB = torch.zeros(B.shape, device="cuda")
    L.slora_linear_bwd(code, tok.batch, tok.seq, tok.ctx_len, k, n, Wdev, Ad_, Bd_, s, idx_d, Xc,
                       XA, dev(dY_ctx, bf), dXc, dA, dB, X_out=Xo,
                       dY_out=dev(dY_out, bf) if dY_out is not None else None, dX_out=dXo)
    torch.cuda.synchronize()
    out = [("Y_ctx", Yc, Yc_o), ("XA", XA, XA_o), ("dX_ctx", dXc, dXc_o), ("dA", dA, dA_o),
           ("dB", dB, dB_o)]
    if Yo is not None:
        out.append(("Y_out", Yo, Yo_o))
    if dXo is not None:
        out.append(("dX_out", dXo, dXo_o))
    return out


def test_value_and_output_projections_llama2_7b_full_size(L):
    """The attention workload's v and o LoRA linears at full size (batch 4 x
    seq 1024, d 4096, 32 heads x 128, LoRA rank 16): v dense (SLICE_NONE); then
    the v/o projection-set variant, v sliced on its output channels
    (SLICE_OUT_ROWS) and o on the matching input channels (SLICE_IN_COLS) by
    the per-head L2 estimate at 50%, the GPU's selection checked against the
    oracle's and both linears compared on the oracle's channel sets."""
    w = synth.WORKLOADS[2]
    tok = synth.Tokens.uniform(w["batch"], w["seq"], w["out_frac"])
    H, hd, d, rs, r = w["heads"], w["head_dim"], w["d"], w["r_svd"], w["r_lora"]
    rnd = synth.round_bf16
    X = rnd(synth.gaussian((tok.T, d), 1.0, 2200))
    Wv = synth.decaying_weight(H * hd, d, 2201, bf16=True, fast=True)
    Wo = synth.decaying_weight(d, H * hd, 2202, bf16=True, fast=True)
    Av, Bv = rnd(synth.gaussian((r, d), 0.02, 2203)), rnd(synth.gaussian((H * hd, r), 0.02, 2204))
    Ao, Bo = rnd(synth.gaussian((r, H * hd), 0.02, 2205)), rnd(synth.gaussian((d, r), 0.02, 2206))
    attn = rnd(synth.gaussian((tok.T, H * hd), 1.0, 2207))  # stand-in for the attention output
    dYv = rnd(synth.gaussian((tok.T, H * hd), 1.0, 2208))
    dYo = rnd(synth.gaussian((tok.T, d), 1.0, 2209))
    C, Orow = O.context_rows(tok.batch, tok.seq, tok.ctx_len)
    # v dense
    for what, got, want in _linear_pair(L, "none", tok, X, None, Wv.W, Av, Bv, 1.0, None, dYv,
                                        None):
        assert_close(host(got), want, TOL["bf16"], f"v dense:{what}")
    # the v/o selection: GPU estimator against the oracle's
    Lv, Uv = _factors(Wv, rs)
    io, iv, kh, sc = O.estimate_select_l2(X, tok.batch, tok.seq, tok.ctx_len, Lv, Uv, H, H, hd,
                                          0.5)
    idx = torch.full((2 * H * hd,), -1, dtype=torch.int32, device="cuda")
    f = lambda a: dev(a, torch.float32)
    k = L.slora_estimate_select(L.CRIT_L2, dev(X, torch.bfloat16), tok.batch, tok.seq,
                                tok.ctx_len, f(Lv), f(Uv), f(Lv), f(Uv), rs, 0.5, idx, heads=H,
                                kv_heads=H, head_dim=hd)
    torch.cuda.synchronize()
    assert k == kh == 64
    gi = host(idx).astype(np.int64)
    for h in range(H):
        check_selection(gi[H * kh + h * kh:H * kh + (h + 1) * kh] - h * hd,
                        iv[h * kh:(h + 1) * kh] - h * hd, sc[h], kh, f"v head {h}")
    # v sliced on output channels iv, o on input channels io (the same channels)
    assert np.array_equal(io, iv)
    for what, got, want in _linear_pair(L, "out_rows", tok, X, None, Wv.W, Av, Bv, 1.0, iv,
                                        rnd(dYv[C][:, iv]), dYv[Orow]):
        assert_close(host(got), want, TOL["bf16"], f"v sliced:{what}")
    for what, got, want in _linear_pair(L, "in_cols", tok, attn[C][:, io], attn[Orow], Wo.W, Ao,
                                        Bo, 1.0, io, dYo, None):
        assert_close(host(got), want, TOL["bf16"], f"o sliced:{what}")

"""Parity at the full workload sizes, in the launch configuration bench.py
times: the Llama-2-7B-shaped FFN layer (batch 8 x seq 512, d 4096, d_ff 11008,
25% output tokens, SVD rank 8, LoRA rank 16, sparsity 50%) and the
Llama-2-7B-shaped attention projections (batch 4 x seq 1024, 32 heads x 128,
q/k sliced at 50% per head by QK-norm, v/o dense LoRA rank 16).

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

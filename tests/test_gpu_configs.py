"""Parity of the two remaining workloads.

32-layer Llama-2-7B-shaped stack.  Every layer is an independent call of the
same kernels, so the stack is covered layer by layer at its distinct
sparsities (dense layers 0-3, then the FFN 0.5->0.9 and QK 0.3->0.6 ramps):
the first dense layer, the first ramp layer and the last layer, FFN and q/k,
on fewer tokens than the stack's 4 x 1024 so the fp64 oracle runs the whole
layer.

Llama-3-8B-shaped layer (d_ff 14336, GQA 32 q / 8 kv heads).  The estimator
and selection run at the full 8192 tokens per batch over the sequence-length
sweep; the sliced FFN and q/k forward/backward run on 512 tokens over the
sparsity x SVD-rank sweep.

The estimator factors are the construction's exact top-r singular triplets,
so both sides score with the same factors."""
import numpy as np
import pytest
import torch

from oracle import slora_oracle as O
from contextual_sparsity_lora_svd_b200 import synth
from tests.helpers import TOL, assert_close, check_selection, dev, host
from tests.test_gpu_parity import _compare_ffn, run_ffn_gpu


def _factors(sw, r):
    return sw.V[:, :r] * sw.s[None, :r], sw.U[:, :r].copy()


def _lay(case, r):
    lay = dict(Wg=case.Wg.W, Wu=case.Wu.W, Wd=case.Wd.W, Ag=case.Ag, Bg=case.Bg, Au=case.Au,
               Bu=case.Bu, Ad=case.Ad, Bd=case.Bd, scale=case.lora_scale)
    lay["Lg"], lay["Ug"] = _factors(case.Wg, r)
    lay["Lu"], lay["Uu"] = _factors(case.Wu, r)
    return lay


# ------------------------------------------------------------- pins (CPU)
def test_stack_sparsity_ramp():
    """The per-layer sparsities of the stack: dense first four layers, then
    linear ramps whose end points are the configuration's."""
    ffn, qk = zip(*(synth.stack_sparsity(l) for l in range(32)))
    assert ffn[:4] == (0.0,) * 4 and qk[:4] == (0.0,) * 4
    assert ffn[4] == pytest.approx(0.5) and ffn[31] == pytest.approx(0.9)
    assert qk[4] == pytest.approx(0.3) and qk[31] == pytest.approx(0.6)
    steps = np.diff(ffn[4:])
    assert np.allclose(steps, 0.4 / 27) and np.allclose(np.diff(qk[4:]), 0.3 / 27)
    with pytest.raises(ValueError):
        synth.stack_sparsity(32)


def test_llama3_workload_shapes():
    w = synth.WORKLOADS[4]
    assert w["heads"] // w["kv_heads"] == 4 and w["d_ff"] == 14336
    for seq in w["seqs"]:
        assert w["tokens"] % seq == 0
    # the kept-channel counts of the sparsity sweep (skip count rounds down)
    assert [O.keep_count(w["d_ff"], s) for s in w["sparsities"]] == [14336, 10036, 7168, 4301,
                                                                     1434]


# ------------------------------------------------------ stack (GPU)
@pytest.fixture(scope="module")
def L():
    from contextual_sparsity_lora_svd_b200 import _lib
    return _lib


STACK_LAYERS = (0, 4, 31)


@pytest.mark.gpu
@pytest.mark.parametrize("layer", STACK_LAYERS)
def test_stack_layer_ffn(L, layer):
    w = synth.WORKLOADS[3]
    s_ffn, _ = synth.stack_sparsity(layer)
    tok = synth.Tokens.uniform(2, 256, w["out_frac"])
    case = synth.ffn_case(tok, w["d"], w["d_ff"], w["r_svd"], w["r_lora"], s_ffn, bf16=True,
                          workload=3, layer=layer, fast=True)
    lay = _lay(case, w["r_svd"])
    ref = O.ffn_fwd_bwd(case.X, case.dOut, tok.batch, tok.seq, tok.ctx_len, lay, s_ffn)
    res = run_ffn_gpu(L, case, lay)
    assert res["k"] == ref["k"] == O.keep_count(w["d_ff"], s_ffn)
    nd = check_selection(res["idx"], ref["idx"], ref["scores"], ref["k"], f"layer {layer}")
    if nd == 0:
        _compare_ffn(res, ref, TOL["bf16"])
    res2 = run_ffn_gpu(L, case, lay, idx_force=ref["idx"])
    _compare_ffn(res2, ref, TOL["bf16"])


def _qk_layer(L, case, tok, r, s, H, KV, hd):
    """GPU q/k selection against the oracle, then the q and k projections
    (fwd + bwd) on the oracle's sets."""
    Lq, Uq = _factors(case.Wq, r)
    Lk, Uk = _factors(case.Wk, r)
    iq, ik, kh, sc = O.estimate_select_qk(case.X, tok.batch, tok.seq, tok.ctx_len, Lq, Uq, Lk, Uk,
                                          H, KV, hd, s)
    f = lambda a: dev(a, torch.float32)
    Xd = dev(case.X, torch.bfloat16)
    idx = torch.full(((H + KV) * hd,), -1, dtype=torch.int32, device="cuda")
    k = L.slora_estimate_select(L.CRIT_QK, Xd, tok.batch, tok.seq, tok.ctx_len, f(Lq), f(Uq),
                                f(Lk), f(Uk), r, s, idx, heads=H, kv_heads=KV, head_dim=hd)
    torch.cuda.synchronize()
    assert k == kh == O.keep_count(hd, s)
    gi = host(idx).astype(np.int64)
    for g in range(KV):
        check_selection(gi[H * kh + g * kh:H * kh + (g + 1) * kh] - g * hd,
                        ik[g * kh:(g + 1) * kh] - g * hd, sc[g], kh, f"kv group {g}")
    C, Orow = O.context_rows(tok.batch, tok.seq, tok.ctx_len)
    sl = case.lora_scale
    for name, W0, A, B, sel, dY in (("q", case.Wq.W, case.Aq, case.Bq, iq, case.dYq),
                                    ("k", case.Wk.W, case.Ak, case.Bk, ik, case.dYk)):
        n, kdim = W0.shape
        Yc_o, Yo_o, XA_o = O.linear_fwd("out_rows", case.X, None, tok.batch, tok.seq, tok.ctx_len,
                                        W0, A, B, sl, sel)
        dYc = synth.round_bf16(dY[C][:, sel])
        dYo = dY[Orow]
        dX_o, _, dA_o, dB_o = O.linear_bwd("out_rows", case.X, None, XA_o, dYc, dYo, tok.batch,
                                           tok.seq, tok.ctx_len, W0, A, B, sl, sel)
        bf = torch.bfloat16
        Wd_, Ad_, Bd_ = dev(W0, bf), dev(A, bf), dev(B, bf)
        idx_d = dev(sel, torch.int32)
        Yc = torch.zeros(Yc_o.shape, dtype=bf, device="cuda")
        Yo = torch.zeros(Yo_o.shape, dtype=bf, device="cuda")
        XA = torch.zeros(tok.T, A.shape[0], device="cuda")
        L.slora_linear_fwd(L.SLICE_OUT_ROWS, tok.batch, tok.seq, tok.ctx_len, kdim, n, Wd_, Ad_,
                           Bd_, sl, idx_d, Xd, Yc, Y_out=Yo, XA_save=XA)
        dX = torch.zeros(tok.T, kdim, dtype=bf, device="cuda")
        dA = torch.zeros(A.shape, device="cuda")
        dB = torch.zeros(B.shape, device="cuda")
        L.slora_linear_bwd(L.SLICE_OUT_ROWS, tok.batch, tok.seq, tok.ctx_len, kdim, n, Wd_, Ad_,
                           Bd_, sl, idx_d, Xd, XA, dev(dYc, bf), dX, dA, dB, dY_out=dev(dYo, bf))
        torch.cuda.synchronize()
        for what, got, want in (("Y_ctx", Yc, Yc_o), ("Y_out", Yo, Yo_o), ("dX", dX, dX_o),
                                ("dA", dA, dA_o), ("dB", dB, dB_o)):
            assert_close(host(got), want, TOL["bf16"], f"{name}:{what}")


@pytest.mark.gpu
@pytest.mark.parametrize("layer", STACK_LAYERS)
def test_stack_layer_qk(L, layer):
    w = synth.WORKLOADS[3]
    _, s_qk = synth.stack_sparsity(layer)
    tok = synth.Tokens.uniform(2, 256, w["out_frac"])
    H, hd = w["heads"], w["head_dim"]
    case = synth.qk_case(tok, w["d"], H, H, hd, w["r_svd"], w["r_lora"], s_qk, bf16=True,
                         workload=3, layer=layer, fast=True)
    _qk_layer(L, case, tok, w["r_svd"], s_qk, H, H, hd)


# ------------------------------------------------ Llama-3-8B (GPU)
@pytest.fixture(scope="module")
def llama3_ffn():
    """One Llama-3-8B-shaped FFN layer on 512 tokens (2 x 256, 75% context)."""
    w = synth.WORKLOADS[4]
    tok = synth.Tokens.uniform(2, 256, w["out_frac"])
    return tok, synth.ffn_case(tok, w["d"], w["d_ff"], 8, w["r_lora"], 0.5, bf16=True,
                               workload=4, layer=0, fast=True)


@pytest.mark.gpu
@pytest.mark.parametrize("s,r", [(0.0, 8), (0.3, 4), (0.7, 16), (0.9, 8)])
def test_llama3_ffn_sparsity_rank_sweep(L, llama3_ffn, s, r):
    tok, case = llama3_ffn
    case.sparsity = s
    lay = _lay(case, r)
    ref = O.ffn_fwd_bwd(case.X, case.dOut, tok.batch, tok.seq, tok.ctx_len, lay, s)
    res = run_ffn_gpu(L, case, lay)
    assert res["k"] == ref["k"]
    check_selection(res["idx"], ref["idx"], ref["scores"], ref["k"], f"s={s} r={r}")
    res2 = run_ffn_gpu(L, case, lay, idx_force=ref["idx"])
    _compare_ffn(res2, ref, TOL["bf16"])


@pytest.fixture(scope="module")
def llama3_weights():
    w = synth.WORKLOADS[4]
    Wg = synth.decaying_weight(w["d_ff"], w["d"], 4002, bf16=True, fast=True)
    Wu = synth.decaying_weight(w["d_ff"], w["d"], 4003, bf16=True, fast=True)
    return Wg, Wu


@pytest.mark.gpu
@pytest.mark.parametrize("seq", [256, 1024, 4096])
def test_llama3_ffn_selection_full_tokens(L, llama3_weights, seq):
    """Estimator + top-k at the full 8192 tokens per batch, across the
    sequence-length sweep (75% of each sequence is context)."""
    w = synth.WORKLOADS[4]
    tok = synth.Tokens.uniform(w["tokens"] // seq, seq, w["out_frac"])
    X = synth.round_bf16(synth.gaussian((tok.T, w["d"]), 1.0, 4000 + seq))
    Wg, Wu = llama3_weights
    r = 8
    Lg, Ug = _factors(Wg, r)
    Lu, Uu = _factors(Wu, r)
    idx_o, k_o, sc_o = O.estimate_select_ffn(X, tok.batch, tok.seq, tok.ctx_len, Lg, Ug, Lu, Uu,
                                             0.5)
    f = lambda a: dev(a, torch.float32)
    idx = torch.full((w["d_ff"],), -1, dtype=torch.int32, device="cuda")
    k = L.slora_estimate_select(L.CRIT_FFN, dev(X, torch.bfloat16), tok.batch, tok.seq,
                                tok.ctx_len, f(Lg), f(Ug), f(Lu), f(Uu), r, 0.5, idx)
    torch.cuda.synchronize()
    assert k == k_o == 7168
    check_selection(host(idx)[:k].astype(np.int64), idx_o, sc_o, k_o, f"seq {seq}")


@pytest.mark.gpu
@pytest.mark.parametrize("s,r", [(0.3, 4), (0.5, 8), (0.9, 16)])
def test_llama3_gqa_qk(L, s, r):
    """GQA q/k: one channel set per kv group shared by its 4 q heads, scored
    by ||K_g,c|| times the sum of the group's ||Q_h,c||; projections on 512
    tokens."""
    w = synth.WORKLOADS[4]
    tok = synth.Tokens.uniform(2, 256, w["out_frac"])
    H, KV, hd = w["heads"], w["kv_heads"], w["head_dim"]
    case = synth.qk_case(tok, w["d"], H, KV, hd, r, w["r_lora"], s, bf16=True, workload=4,
                         layer=1, fast=True)
    _qk_layer(L, case, tok, r, s, H, KV, hd)

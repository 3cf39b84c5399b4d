"""GPU parity of the whole decoder-stack training step (layers.DecoderStack):
RMS norms, q/k selection and sliced q/k, v, o linears, rotary packing, the
causal attention core, residuals and the sparse FFN, forward through every
layer and backward in reverse, compared with the float64 stack oracle on the
channel sets the GPU selected.  Each selection is checked against the
oracle's estimator run on the GPU's own normalised input of that layer (the
near-tie rule), and the output, the input gradient and every layer's LoRA
gradients against the oracle's step."""
import numpy as np
import pytest
import torch

from oracle import slora_oracle as SO
from oracle import stack_oracle as S
from contextual_sparsity_lora_svd_b200 import synth
from tests.helpers import TOL, assert_close, check_selection, dev, host

pytestmark = pytest.mark.gpu
TOLB = TOL["bf16"]
# Tolerance of a 3-layer stack against float64.  Every call of the step meets
# the single-call bf16 bound (1e-2) on its own inputs; composed, each layer
# reads activations that already carry the rounding of the layers below
# (measured: n1, Q, K, V 2-6e-3 off float64), and the q/k LoRA gradients pass
# through the softmax derivative dS = P (dP - rowsum(dO O)), whose cancellation
# turns a 2^-9 rounding of Q, K, V, dO into ~4e-3 of dQ, dK even with exact
# arithmetic inside the kernel (float64 emulation).  Measured maximum over
# both cases: 1.3e-2 (q/k gradients of the top layer); the bound is 2e-2.
TOL_STACK = 2e-2


def _rb(a):
    return synth.round_bf16(np.asarray(a, dtype=np.float64))


def make_stack(nl, d, H, KV, hd, d_ff, r_svd, r, seed):
    """Per layer: the oracle's float64 dict (bf16-rounded values) and the
    device tensors of the same values."""
    nq, nkv = H * hd, KV * hd
    lays, devs = [], []
    for l in range(nl):
        sd = seed + 100 * l
        lay = dict(scale=1.0)
        for i, (nm, n, k) in enumerate((("q", nq, d), ("k", nkv, d), ("v", nkv, d),
                                        ("o", d, nq), ("g", d_ff, d), ("u", d_ff, d),
                                        ("d", d, d_ff))):
            lay["W" + nm] = synth.decaying_weight(n, k, sd + i, rms=k ** -0.5, bf16=True).W
            lay["A" + nm] = _rb(synth.gaussian((r, k), 0.05, sd + 10 + i))
            lay["B" + nm] = _rb(synth.gaussian((n, r), 0.05, sd + 20 + i))
        rng = np.random.default_rng(sd + 30)
        lay["g1"] = _rb(1.0 + 0.1 * rng.normal(size=d))
        lay["g2"] = _rb(1.0 + 0.1 * rng.normal(size=d))
        for nm in ("q", "k", "g", "u"):
            lay["L" + nm], lay["U" + nm] = SO.svd_prepare(lay["W" + nm], r_svd)
        w = {k: dev(v, torch.bfloat16) for k, v in lay.items()
             if k[0] in "WABg" and k not in ("Wd",)}
        w["Wd_t"] = dev(lay["Wd"].T.copy(), torch.bfloat16)
        for nm in ("q", "k", "g", "u"):
            w["L" + nm] = dev(lay["L" + nm], torch.float32)
            w["U" + nm] = dev(lay["U" + nm], torch.float32)
        lays.append(lay)
        devs.append(w)
    return lays, devs


@pytest.mark.parametrize("H,KV,hd,ctx", [(4, 4, 64, [72, 60]), (4, 2, 128, [96, 50])])
def test_decoder_stack_step_matches_oracle(H, KV, hd, ctx):
    from contextual_sparsity_lora_svd_b200.layers import DecoderStack
    nl, d, d_ff, r_svd, r, b, seq = 3, 256, 688, 8, 8, 2, 96
    qk_s, ffn_s = [0.0, 0.5, 0.25], [0.0, 0.5, 0.7]
    lays, devs = make_stack(nl, d, H, KV, hd, d_ff, r_svd, r, seed=11 + H + hd)
    rng = np.random.default_rng(5)
    X, dY = _rb(rng.normal(size=(b * seq, d))), _rb(rng.normal(size=(b * seq, d)))
    run = DecoderStack(devs, d, H, KV, hd, d_ff, r_svd, r, 1.0, b, seq, ctx, qk_s, ffn_s,
                       dev(X, torch.bfloat16), dev(dY, torch.bfloat16))
    ws = torch.empty(run.workspace_bytes(), dtype=torch.uint8, device="cuda")
    run.step(ws)
    torch.cuda.synchronize()
    sets = []
    for l in range(nl):
        n1 = host(run.saved[l]["n1"])
        if qk_s[l] > 0:
            kh = run.kh[l]
            gi = host(run.idx_qk[l]).astype(np.int64)
            iq, ik = gi[:H * kh], gi[H * kh:H * kh + KV * kh]
            oq, ok_, k_o, sc = SO.estimate_select_qk(n1, b, seq, ctx, lays[l]["Lq"],
                                                     lays[l]["Uq"], lays[l]["Lk"], lays[l]["Uk"],
                                                     H, KV, hd, qk_s[l])
            assert kh == k_o
            for g in range(KV):
                check_selection(ik[g * kh:(g + 1) * kh] - g * hd, ok_[g * kh:(g + 1) * kh] - g * hd,
                                sc[g], kh, f"layer {l} group {g}")
            grp = H // KV
            for h in range(H):   # every q head of a group carries its group's set
                assert np.array_equal(iq[h * kh:(h + 1) * kh] - h * hd,
                                      ik[(h // grp) * kh:(h // grp + 1) * kh] - (h // grp) * hd)
        else:
            iq = ik = None
        kf = run.k_ffn[l]
        fi = host(run.idx_ffn[l])[:kf].astype(np.int64)
        if ffn_s[l] > 0:
            n2 = host(run.saved[l]["n2"])
            of, ko, so = SO.estimate_select_ffn(n2, b, seq, ctx, lays[l]["Lg"], lays[l]["Ug"],
                                                lays[l]["Lu"], lays[l]["Uu"], ffn_s[l])
            assert kf == ko
            check_selection(fi, of, so, kf, f"layer {l} ffn")
        else:
            assert kf == d_ff and np.array_equal(fi, np.arange(d_ff))
        sets.append((iq, ik, fi))
    ref = S.stack_fwd_bwd(X, dY, lays, b, seq, ctx, H, KV, hd, idx_force=sets)
    assert_close(host(run.y), ref["y"], TOLB, "stack output")
    assert_close(host(run.dX), ref["dx"], TOLB, "stack input gradient")
    for l in range(nl):
        for key, val in ref["grads"][l].items():
            assert_close(host(run.grads[l][key]), val, TOL_STACK, f"layer {l} {key}")


def test_decoder_stack_graph_replay_is_reproducible():
    """The step captured in a CUDA graph and replayed twice gives the same
    output and LoRA-B gradients (dQ's atomic order may move the last bits of
    the q/k-side gradients, so those are compared within rounding)."""
    from contextual_sparsity_lora_svd_b200.layers import DecoderStack
    nl, d, H, KV, hd, d_ff, b, seq = 2, 256, 4, 4, 64, 688, 2, 64
    lays, devs = make_stack(nl, d, H, KV, hd, d_ff, 8, 8, seed=77)
    rng = np.random.default_rng(9)
    X, dY = _rb(rng.normal(size=(b * seq, d))), _rb(rng.normal(size=(b * seq, d)))
    run = DecoderStack(devs, d, H, KV, hd, d_ff, 8, 8, 1.0, b, seq, [48, 40], [0.5, 0.5],
                       [0.5, 0.5], dev(X, torch.bfloat16), dev(dY, torch.bfloat16))
    ws = torch.empty(run.workspace_bytes(), dtype=torch.uint8, device="cuda")
    run.step(ws)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            run.step(ws, s)
    outs = []
    for _ in range(2):
        g.replay()
        torch.cuda.synchronize()
        outs.append((host(run.y), host(run.gflat)))
    assert np.array_equal(outs[0][0], outs[1][0])
    assert_close(outs[1][1], outs[0][1], 1e-5, "gradients across replays")

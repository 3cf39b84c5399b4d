"""GPU parity of the projection-set variants: one channel set per sequence
for the SwiGLU FFN (slora_ffn_fwd_bwd_per_seq), in bf16 and fp32.  Each
sequence's selection is checked against the oracle's selection on that
sequence (near-tie rule), then the outputs and the summed LoRA gradients
against the oracle run on the GPU's sets."""
import numpy as np
import pytest
import torch

from oracle import slora_oracle as O
from contextual_sparsity_lora_svd_b200 import synth
from tests.helpers import TOL, assert_close, check_selection, dev, host, tdtype

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    from contextual_sparsity_lora_svd_b200 import _lib
    return _lib


@pytest.mark.parametrize("bf16", [True, False])
def test_ffn_per_sequence_sets(L, bf16):
    tok = synth.Tokens(3, 96, np.array([70, 50, 96], np.int32))
    case = synth.ffn_case(tok, d=128, d_ff=344, r_svd=8, r_lora=8, sparsity=0.5, bf16=bf16,
                          workload=0, layer=9)
    lay = dict(Wg=case.Wg.W, Wu=case.Wu.W, Wd=case.Wd.W, Ag=case.Ag, Bg=case.Bg, Au=case.Au,
               Bu=case.Bu, Ad=case.Ad, Bd=case.Bd, scale=case.lora_scale)
    lay["Lg"], lay["Ug"] = O.svd_prepare(case.Wg.W, 8)
    lay["Lu"], lay["Uu"] = O.svd_prepare(case.Wu.W, 8)
    dt = tdtype(bf16)
    t = {k: dev(lay[k], dt) for k in ("Wg", "Wu", "Ag", "Bg", "Au", "Bu", "Ad", "Bd")}
    t["Wd_t"] = dev(lay["Wd"].T.copy(), dt)
    f = {k: dev(lay[k], torch.float32) for k in ("Lg", "Ug", "Lu", "Uu")}
    layer = L.ffn_layer_struct(128, 344, 8, 8, case.lora_scale, t["Wg"], t["Wu"], t["Wd_t"],
                               t["Ag"], t["Bg"], t["Au"], t["Bu"], t["Ad"], t["Bd"], f["Lg"],
                               f["Ug"], f["Lu"], f["Uu"])
    T = tok.T
    out = torch.zeros(T, 128, dtype=dt, device="cuda")
    dX = torch.zeros(T, 128, dtype=dt, device="cuda")
    g = {k: torch.zeros(sh, device="cuda") for k, sh in
         (("dAg", (8, 128)), ("dBg", (344, 8)), ("dAu", (8, 128)), ("dBu", (344, 8)),
          ("dAd", (8, 344)), ("dBd", (128, 8)))}
    grads = L.ffn_grads_struct(g["dAg"], g["dBg"], g["dAu"], g["dBu"], g["dAd"], g["dBd"])
    idx = torch.full((3 * 344,), -1, dtype=torch.int32, device="cuda")
    k = L.slora_ffn_fwd_bwd(layer, tok.batch, tok.seq, tok.ctx_len, 0.5, dev(case.X, dt),
                            dev(case.dOut, dt), out, dX, grads, idx, per_sequence=True)
    torch.cuda.synchronize()
    assert k == 172
    sets = []
    gi = host(idx).astype(np.int64).reshape(3, 344)
    for b in range(3):
        rows = slice(b * 96, (b + 1) * 96)
        io, ko, so = O.estimate_select_ffn(case.X[rows], 1, 96, [int(tok.ctx_len[b])], lay["Lg"],
                                           lay["Ug"], lay["Lu"], lay["Uu"], 0.5)
        check_selection(gi[b, :k], io, so, k, f"sequence {b}")
        sets.append(gi[b, :k])
    assert len({tuple(s) for s in sets}) > 1
    ref = O.ffn_fwd_bwd_per_seq(case.X, case.dOut, 3, 96, tok.ctx_len, lay, 0.5, idx_force=sets)
    tol = TOL["bf16" if bf16 else "f32"]
    assert_close(host(out), ref["out"], tol, "out")
    assert_close(host(dX), ref["dX"], tol, "dX")
    for name, v in g.items():
        assert_close(host(v), ref[name], tol, name)
    # the forced per-sequence sets reproduce the same step
    out2 = torch.zeros_like(out)
    force = dev(np.concatenate(sets), torch.int32)
    L.slora_ffn_fwd_bwd(layer, tok.batch, tok.seq, tok.ctx_len, 0.5, dev(case.X, dt),
                        dev(case.dOut, dt), out2, dX, grads, idx, idx_force=force,
                        per_sequence=True)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)


def test_ffn_per_sequence_lanes_match_single_sequence_calls(L):
    """Six sequences run in four concurrent lanes (two lanes take two
    sequences each, reusing their sub-workspace): every sequence's output
    rows, input gradient and index list equal, bit for bit, a separate call
    on that sequence alone; the LoRA gradients equal the sequence-ordered sum
    of the separate calls' gradients; and a CUDA-graph replay of the call
    reproduces the eager result exactly."""
    B, seq, d, F, r = 6, 64, 128, 344, 8
    tok = synth.Tokens(B, seq, np.array([48, 64, 30, 0, 57, 41], np.int32))
    case = synth.ffn_case(tok, d=d, d_ff=F, r_svd=8, r_lora=r, sparsity=0.5, bf16=True,
                          workload=0, layer=13)
    dt = torch.bfloat16
    t = {k: dev(getattr(case, k), dt) for k in ("Ag", "Bg", "Au", "Bu", "Ad", "Bd")}
    W = {"Wg": dev(case.Wg.W, dt), "Wu": dev(case.Wu.W, dt), "Wd_t": dev(case.Wd.W.T.copy(), dt)}
    fac = {}
    fac["Lg"], fac["Ug"] = (dev(a, torch.float32) for a in O.svd_prepare(case.Wg.W, 8))
    fac["Lu"], fac["Uu"] = (dev(a, torch.float32) for a in O.svd_prepare(case.Wu.W, 8))
    layer = L.ffn_layer_struct(d, F, 8, r, case.lora_scale, W["Wg"], W["Wu"], W["Wd_t"], t["Ag"],
                               t["Bg"], t["Au"], t["Bu"], t["Ad"], t["Bd"], fac["Lg"], fac["Ug"],
                               fac["Lu"], fac["Uu"])
    X, dOut = dev(case.X, dt), dev(case.dOut, dt)
    shapes = (("dAg", (r, d)), ("dBg", (F, r)), ("dAu", (r, d)), ("dBu", (F, r)),
              ("dAd", (r, F)), ("dBd", (d, r)))

    def run(per_seq_tok, Xs, dOs, graph=False):
        T = Xs.shape[0]
        out = torch.zeros(T, d, dtype=dt, device="cuda")
        dX = torch.zeros(T, d, dtype=dt, device="cuda")
        g = {k: torch.zeros(sh, device="cuda") for k, sh in shapes}
        grads = L.ffn_grads_struct(*(g[k] for k, _ in shapes))
        idx = torch.full((per_seq_tok.batch * F,), -1, dtype=torch.int32, device="cuda")
        call = lambda: L.slora_ffn_fwd_bwd(layer, per_seq_tok.batch, per_seq_tok.seq,
                                           per_seq_tok.ctx_len, 0.5, Xs, dOs, out, dX, grads,
                                           idx, per_sequence=True)
        k = call()
        if graph:
            torch.cuda.synchronize()
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                cg = torch.cuda.CUDAGraph()
                with torch.cuda.graph(cg, stream=s):
                    call()
            res = []
            for _ in range(2):
                for v in g.values():
                    v.zero_()
                cg.replay()
                torch.cuda.synchronize()
                res.append((out.clone(), dX.clone(), {n: v.clone() for n, v in g.items()}))
            return k, idx, res
        torch.cuda.synchronize()
        return k, idx, (out, dX, g)

    k, idx, (out, dX, g) = run(tok, X, dOut)
    acc = {n: torch.zeros(sh, device="cuda") for n, sh in shapes}
    for b in range(B):
        rows = slice(b * seq, (b + 1) * seq)
        tb = synth.Tokens(1, seq, tok.ctx_len[b:b + 1].copy())
        kb, ib, (ob, xb, gb) = run(tb, X[rows].contiguous(), dOut[rows].contiguous())
        assert kb == k
        assert torch.equal(idx[b * F:b * F + k], ib[:k]), f"sequence {b} selection"
        assert torch.equal(out[rows], ob), f"sequence {b} output"
        assert torch.equal(dX[rows], xb), f"sequence {b} input gradient"
        for n in acc:
            acc[n] += gb[n]
    for n in acc:
        torch.testing.assert_close(g[n], acc[n], rtol=1e-5, atol=1e-6)
    _, _, res = run(tok, X, dOut, graph=True)
    for o2, x2, g2 in res:
        assert torch.equal(o2, out) and torch.equal(x2, dX)
        for n in g:
            assert torch.equal(g2[n], g[n]), n

"""The FFN call can be captured in a CUDA graph and replayed.

A step issues a few dozen launches; a caller that replays a captured step
(as bench.py does) must get exactly what the eager call gives: every buffer,
tensor map and counter of the call is fixed for a given workspace, and the
call's own counters are reset at its start.  Two replays and one eager run
on the same inputs are compared bit for bit (the path has no atomics in its
arithmetic), on the estimator path and on a forced channel set."""
import numpy as np
import pytest
import torch

from oracle import slora_oracle as O
from contextual_sparsity_lora_svd_b200 import synth
from tests.helpers import TOL, assert_close, host
from tests.test_gpu_parity import _ffn_lay

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    from contextual_sparsity_lora_svd_b200 import _lib
    return _lib


def _setup(L, case, lay, force):
    bf = torch.bfloat16
    dev = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(dt).cuda()
    d, F, r = case.d, case.d_ff, case.r_lora
    t = {k: dev(lay[k], bf) for k in ("Wg", "Wu", "Ag", "Bg", "Au", "Bu", "Ad", "Bd")}
    t["Wd_t"] = dev(lay["Wd"].T.copy(), bf)
    for k in ("Lg", "Ug", "Lu", "Uu"):
        t[k] = dev(lay[k], torch.float32)
    layer = L.ffn_layer_struct(d, F, lay["Lg"].shape[1], r, case.lora_scale, t["Wg"], t["Wu"],
                               t["Wd_t"], t["Ag"], t["Bg"], t["Au"], t["Bu"], t["Ad"], t["Bd"],
                               t["Lg"], t["Ug"], t["Lu"], t["Uu"])
    T = case.tokens.T
    io = dict(X=dev(case.X, bf), dOut=dev(case.dOut, bf),
              out=torch.zeros(T, d, dtype=bf, device="cuda"),
              dX=torch.zeros(T, d, dtype=bf, device="cuda"),
              idx=torch.full((F,), -1, dtype=torch.int32, device="cuda"))
    shapes = [(r, d), (F, r), (r, d), (F, r), (r, F), (d, r)]
    io["g"] = [torch.zeros(a, b, device="cuda") for a, b in shapes]
    grads = L.ffn_grads_struct(*io["g"])
    tok = case.tokens
    force_t = dev(np.asarray(force), torch.int32) if force is not None else None
    args, keep = L.ffn_args(L.BF16, layer, tok.batch, tok.seq, tok.ctx_len, case.sparsity,
                            io["X"], io["dOut"], io["out"], io["dX"], grads, io["idx"], force_t)
    need = L.workspace_size("slora_ffn_fwd_bwd", args)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    return io, (args, keep, t, layer, grads, force_t, ws, L.c_sz(need))


def _call(L, held, stream):
    import ctypes
    args, keep, t, layer, grads, force_t, ws, have = held
    st = L.lib().slora_ffn_fwd_bwd(*args, L.ptr(ws), ctypes.byref(have), stream.cuda_stream)
    assert st == 0, L.lib().slora_last_error_string()


def _snapshot(io):
    return [io["out"].clone(), io["dX"].clone(), io["idx"].clone()] + [g.clone() for g in io["g"]]


@pytest.mark.parametrize("forced", [False, True])
def test_graph_replay_matches_eager(L, forced):
    tok = synth.Tokens(3, 256, np.asarray([192, 130, 256], np.int32))
    case = synth.ffn_case(tok, 512, 1200, 8, 16, 0.5, bf16=True, workload=0, layer=8)
    lay = _ffn_lay(case, 8)
    ref = O.ffn_fwd_bwd(case.X, case.dOut, tok.batch, tok.seq, tok.ctx_len, lay, case.sparsity)
    io, held = _setup(L, case, lay, ref["idx"] if forced else None)
    s = torch.cuda.current_stream()
    _call(L, held, s)  # eager (also the warm-up before capture)
    torch.cuda.synchronize()
    eager = _snapshot(io)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _call(L, held, torch.cuda.current_stream())
    for _ in range(2):
        for x in (io["out"], io["dX"], *io["g"]):
            x.zero_()
        io["idx"].fill_(-1)
        g.replay()
        torch.cuda.synchronize()
        for a, b in zip(_snapshot(io), eager):
            assert torch.equal(a, b)
    # and the replayed result is the method's result
    if forced:
        assert_close(host(io["out"]), ref["out"], TOL["bf16"], "out")
        assert_close(host(io["dX"]), ref["dX"], TOL["bf16"], "dX")
        for k, gi in zip(("dAg", "dBg", "dAu", "dBu", "dAd", "dBd"), io["g"]):
            assert_close(host(gi), ref[k], TOL["bf16"], k)

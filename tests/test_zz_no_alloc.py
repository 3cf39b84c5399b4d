"""slora_estimate_select_noalloc, the entry point for callers that cannot give
the library a workspace (it runs on a scratch buffer the library keeps in
device memory), must produce what slora_estimate_select produces with a
caller workspace, call after call, and refuse problems too large for its
buffer.  This file is collected last so that a failure here leaves every other
test already run; it passes alone in a fresh process as well."""
import ctypes

import numpy as np
import pytest
import torch

from oracle import slora_oracle as O
from contextual_sparsity_lora_svd_b200 import synth
from tests.helpers import dev, host, rel_frob

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    from contextual_sparsity_lora_svd_b200 import _lib
    assert torch.cuda.is_available()
    return _lib


def _ffn_inputs(bf16):
    tok = synth.Tokens(3, 96, np.asarray([72, 40, 96], np.int32))
    d, d_ff, r = 256, 688, 8
    X = synth.gaussian((tok.T, d), 1.0, 900)
    if bf16:
        X = synth.round_bf16(X)
    fac = [O.svd_prepare(synth.decaying_weight(d_ff, d, 901 + m, bf16=bf16).W, r) for m in range(2)]
    return tok, X, fac, d_ff, r


@pytest.mark.parametrize("bf16", [True, False])
def test_noalloc_matches_workspace_call_twice(L, bf16):
    tok, X, ((Lg, Ug), (Lu, Uu)), d_ff, r = _ffn_inputs(bf16)
    f = lambda a: dev(a, torch.float32)
    Xd = dev(X, torch.bfloat16 if bf16 else torch.float32)
    args = (L.CRIT_FFN, Xd, tok.batch, tok.seq, tok.ctx_len, f(Lg), f(Ug), f(Lu), f(Uu), r, 0.5)
    idx_ref = torch.full((d_ff,), -1, dtype=torch.int32, device="cuda")
    sc_ref = torch.zeros(d_ff, device="cuda")
    k_ref = L.slora_estimate_select(*args, idx_ref, scores_out=sc_ref)
    for _ in range(2):  # two calls in a row on the shared buffer
        idx = torch.full((d_ff,), -1, dtype=torch.int32, device="cuda")
        sc = torch.zeros(d_ff, device="cuda")
        k = L.slora_estimate_select_noalloc(*args, idx, scores_out=sc)
        torch.cuda.synchronize()
        assert k == k_ref
        assert rel_frob(host(sc), host(sc_ref)) <= 1e-5
        assert torch.equal(idx[:k], idx_ref[:k_ref])


def test_noalloc_qk_matches_workspace_call(L):
    tok = synth.Tokens(2, 64, np.asarray([48, 20], np.int32))
    d, H, KV, hd, r = 128, 4, 2, 32, 8
    X = synth.round_bf16(synth.gaussian((tok.T, d), 1.0, 910))
    Lq, Uq = O.svd_prepare(synth.decaying_weight(H * hd, d, 911, bf16=True).W, r)
    Lk, Uk = O.svd_prepare(synth.decaying_weight(KV * hd, d, 912, bf16=True).W, r)
    f = lambda a: dev(a, torch.float32)
    args = (L.CRIT_QK, dev(X, torch.bfloat16), tok.batch, tok.seq, tok.ctx_len, f(Lq), f(Uq),
            f(Lk), f(Uk), r, 0.5)
    n_idx = (H + KV) * hd
    ref = torch.full((n_idx,), -1, dtype=torch.int32, device="cuda")
    k_ref = L.slora_estimate_select(*args, ref, heads=H, kv_heads=KV, head_dim=hd)
    for _ in range(2):
        got = torch.full((n_idx,), -1, dtype=torch.int32, device="cuda")
        k = L.slora_estimate_select_noalloc(*args, got, heads=H, kv_heads=KV, head_dim=hd)
        torch.cuda.synchronize()
        assert k == k_ref and torch.equal(got, ref)


def test_noalloc_refuses_oversized_problem(L):
    """A problem whose scratch need exceeds the built-in buffer is refused
    with SLORA_ERR_WORKSPACE before anything is launched."""
    cap = L.noalloc_scratch_bytes()
    assert cap == 32 << 20
    batch, seq, d, n, r = 64, 2048, 4096, 14336, 16  # far beyond 32 MiB of scratch
    tok, keep = L.make_tokens(batch, seq, [seq] * batch)
    k_out = ctypes.c_int32(0)
    FAKE = 0x10000
    need = L.workspace_size("slora_estimate_select",
                            [L.CRIT_FFN, FAKE, L.BF16, ctypes.byref(tok), d, FAKE, FAKE, n, FAKE,
                             FAKE, n, r, 0, 0, 0, 0.5, FAKE, ctypes.byref(k_out), None])
    assert need > cap
    st = L.lib().slora_estimate_select_noalloc(L.CRIT_FFN, FAKE, L.BF16, ctypes.byref(tok), d,
                                               FAKE, FAKE, n, FAKE, FAKE, n, r, 0, 0, 0, 0.5,
                                               FAKE, ctypes.byref(k_out), None, None)
    assert st == 4  # SLORA_ERR_WORKSPACE
    assert b"built-in buffer" in L.lib().slora_last_error_string()

"""Error paths on the GPU, made without faulting it.

A wait budget of 0 cycles makes the skinny-contraction stream kernel's
pipeline waits give up at their first unsuccessful poll: the call must leave
the device usable, the expiry must be reported by slora_device_error as
SLORA_ERR_TIMEOUT, and the next call with the default budget must be correct
again.  Gathers given out-of-range channel indices read zeros and raise the
device flag instead of reading outside the weight: every caller-supplied
channel list is copied through a check that replaces such entries by
channel 0 before any kernel reads through it."""
import numpy as np
import pytest
import torch

from oracle import slora_oracle as O
from contextual_sparsity_lora_svd_b200 import synth
from tests.helpers import TOL
from tests.test_gpu_parity import _compare_ffn, _ffn_lay, run_ffn_gpu

pytestmark = pytest.mark.gpu

SLORA_ERR_INVALID_ARG, SLORA_ERR_TIMEOUT = 1, 7


@pytest.fixture(scope="module")
def L():
    from contextual_sparsity_lora_svd_b200 import _lib
    return _lib


@pytest.fixture(scope="module")
def small_case():
    tok = synth.Tokens(2, 192, np.asarray([144, 100], np.int32))
    case = synth.ffn_case(tok, 256, 688, 8, 16, 0.5, bf16=True, workload=0, layer=7)
    lay = _ffn_lay(case, 8)
    ref = O.ffn_fwd_bwd(case.X, case.dOut, tok.batch, tok.seq, tok.ctx_len, lay, case.sparsity)
    return case, lay, ref


def test_expired_wait_is_reported_and_device_recovers(L, small_case):
    case, lay, ref = small_case
    lib = L.lib()
    assert lib.slora_device_error(1) == 0  # start clean
    assert lib.slora_set_wait_budget(0) == 0
    try:
        run_ffn_gpu(L, case, lay, idx_force=ref["idx"])  # outputs undefined
    finally:
        assert lib.slora_set_wait_budget(-1) == 0
    assert lib.slora_device_error(1) == SLORA_ERR_TIMEOUT
    assert b"wait expired" in lib.slora_last_error_string()
    assert lib.slora_device_error(0) == 0  # the flag was cleared
    res = run_ffn_gpu(L, case, lay, idx_force=ref["idx"])
    _compare_ffn(res, ref, TOL["bf16"])
    assert lib.slora_device_error(0) == 0


def test_out_of_range_channel_index_is_refused(L, small_case):
    case, lay, ref = small_case
    lib = L.lib()
    assert lib.slora_device_error(1) == 0
    bad = ref["idx"].copy()
    bad[3] = case.d_ff + 5  # outside the weight
    run_ffn_gpu(L, case, lay, idx_force=bad)
    assert lib.slora_device_error(1) == SLORA_ERR_INVALID_ARG
    assert b"outside its weight" in lib.slora_last_error_string()
    res = run_ffn_gpu(L, case, lay, idx_force=ref["idx"])
    _compare_ffn(res, ref, TOL["bf16"])
    assert lib.slora_device_error(0) == 0


@pytest.mark.parametrize("side", ["out_rows", "in_cols"])
def test_linear_out_of_range_index_is_refused(L, side):
    """The linear calls sanitize their channel list the same way."""
    lib = L.lib()
    assert lib.slora_device_error(1) == 0
    tok = synth.Tokens(2, 64, np.asarray([40, 64], np.int32))
    n, k, r = 96, 64, 4
    bf = torch.bfloat16
    W = torch.randn(n, k, device="cuda").to(bf) if side == "out_rows" else \
        torch.randn(k, n, device="cuda").to(bf)
    A = torch.randn(r, k, device="cuda").to(bf)
    B = torch.randn(n, r, device="cuda").to(bf)
    lim = n if side == "out_rows" else k
    idx = torch.arange(0, lim, 2, dtype=torch.int32, device="cuda")
    idx[5] = lim + 40
    ni = idx.numel()
    code = L.SLICE_OUT_ROWS if side == "out_rows" else L.SLICE_IN_COLS
    XA = torch.zeros(tok.T, r, device="cuda")
    if side == "out_rows":  # X [T x k] in, Y_ctx [T_C x n_idx] and Y_out [T_O x n] out
        Xc = torch.randn(tok.T, k, device="cuda").to(bf)
        Yc = torch.zeros(tok.T_C, ni, dtype=bf, device="cuda")
        kw = dict(Y_out=torch.zeros(tok.T_O, n, dtype=bf, device="cuda"), XA_save=XA)
    else:  # X_ctx [T_C x n_idx] and X_out [T_O x k] in, Y [T x n] out
        Xc = torch.randn(tok.T_C, ni, device="cuda").to(bf)
        Yc = torch.zeros(tok.T, n, dtype=bf, device="cuda")
        kw = dict(X_out=torch.randn(tok.T_O, k, device="cuda").to(bf), XA_save=XA)
    L.slora_linear_fwd(code, tok.batch, tok.seq, tok.ctx_len, k, n, W, A, B, 1.0, idx, Xc, Yc,
                       **kw)
    torch.cuda.synchronize()
    assert lib.slora_device_error(1) == SLORA_ERR_INVALID_ARG
    assert lib.slora_device_error(0) == 0

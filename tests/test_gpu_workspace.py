"""Every entry point stays inside the workspace whose size it reported, and
reads only workspace it wrote itself.

Each call here gets a workspace of exactly the queried size, cut from the
front of a larger buffer filled with a byte pattern (0xA5, or 0xFF which
reads as NaN); after the call the 1 MiB tail must be untouched and the
outputs must still match the oracle.  A run that takes more workspace than its
size query promised writes into the tail (in-bounds memory) instead of past
the end of an allocation, so the test fails without faulting the device.
The calls are the parity cases of test_gpu_parity and test_gpu_tc, so the
outputs are checked against the oracle as well."""
import ctypes

import pytest
import torch

from tests import test_gpu_parity as P
from tests import test_gpu_tc as TC

pytestmark = pytest.mark.gpu

GUARD = 1 << 20


# 0xA5 bytes read back as tiny bf16 / fp32 values; 0xFF bytes read back as
# NaN, so a kernel that reads workspace its call never wrote turns the call's
# outputs into NaN and the parity check fails
@pytest.fixture(params=[0xA5, 0xFF], ids=["fillA5", "fillNaN"])
def GL(monkeypatch, request):
    from contextual_sparsity_lora_svd_b200 import _lib as L
    seen = []
    pattern = request.param

    def guarded_run(fn_name, args_before_ws, ws, stream):
        need = L.workspace_size(fn_name, args_before_ws)
        buf = torch.full((need + GUARD,), pattern, dtype=torch.uint8, device="cuda")
        have = ctypes.c_size_t(need)
        st = getattr(L.lib(), fn_name)(*args_before_ws, L.ptr(buf), ctypes.byref(have),
                                       L._stream(stream))
        L._check(fn_name, st)
        torch.cuda.synchronize()
        spill = int((buf[need:] != pattern).sum())
        assert spill == 0, f"{fn_name} wrote {spill} bytes past its {need}-byte workspace"
        seen.append(fn_name)
        return buf

    monkeypatch.setattr(L, "_run", guarded_run)
    L.seen = seen
    return L


@pytest.mark.parametrize("bf16", [False, True])
def test_guard_svd_prepare(GL, bf16):
    P.test_svd_prepare(GL, bf16, 200, 96, 8)
    assert "slora_svd_prepare" in GL.seen


@pytest.mark.parametrize("bf16", [False, True])
def test_guard_estimate_select(GL, bf16):
    P.test_estimate_select_ffn(GL, bf16, 0.5)
    P.test_estimate_select_qk(GL, 8, 2, 0.5)
    assert "slora_estimate_select" in GL.seen


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("side", ["none", "out_rows", "in_cols"])
def test_guard_linear(GL, bf16, side):
    P.test_linear_fwd_bwd(GL, bf16, side)
    assert {"slora_linear_fwd", "slora_linear_bwd"} <= set(GL.seen)


@pytest.mark.parametrize("bf16", [False, True])
def test_guard_ffn(GL, bf16):
    # the estimator path and the forced-selection path, plus ragged edges
    P.test_ffn_workload0_full(GL, bf16)
    P.test_ffn_ragged_and_edges(GL, bf16, [70, 33, 90])
    P.test_ffn_ragged_and_edges(GL, bf16, [0, 0, 0])
    assert "slora_ffn_fwd_bwd" in GL.seen


def test_guard_ffn_multi_tile(GL):
    TC.test_ffn_tc_multi_tile(GL, [129, 1, 200], 264, 1000, 0.7, 16)
    assert "slora_ffn_fwd_bwd" in GL.seen


def test_guard_linear_single_tile(GL):
    """One 128-row M tile (an odd tile count for the cluster-pair GEMM)."""
    P.test_linear_fwd_bwd_single_tile(GL)
    assert {"slora_linear_fwd", "slora_linear_bwd"} <= set(GL.seen)

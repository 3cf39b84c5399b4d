"""Parity of the bf16 tcgen05 path at sizes spanning several 128x256 tiles,
ragged sequence lengths (tiles shorter than 128 rows), channel counts that are
not multiples of the tile width, both LoRA ranks used by the workloads and one
above the ranks the GEMM epilogues project."""
import numpy as np
import pytest
import torch

from oracle import slora_oracle as O
from contextual_sparsity_lora_svd_b200 import synth
from tests.helpers import TOL, assert_close, check_selection
from tests.test_gpu_parity import _ffn_lay, _compare_ffn, run_ffn_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    from contextual_sparsity_lora_svd_b200 import _lib
    return _lib


@pytest.mark.parametrize("ctx,d,d_ff,s,r", [
    ([300, 170, 320], 512, 1200, 0.5, 16),
    ([256, 256], 768, 2048, 0.3, 8),
    ([129, 1, 200], 264, 1000, 0.7, 16),
    # rank above 16: no rank projections in the GEMM epilogues (hA and
    # [dG Bg | dU Bu] by separate contractions), TMA epilogue without slices
    ([300, 170, 320], 512, 1200, 0.5, 24),
])
def test_ffn_tc_multi_tile(L, ctx, d, d_ff, s, r):
    tok = synth.Tokens(len(ctx), 320 if len(ctx) != 2 else 384, np.asarray(ctx, np.int32))
    case = synth.ffn_case(tok, d, d_ff, 8, r, s, bf16=True, workload=0, layer=5,
                          lora_scale=0.75)
    lay = _ffn_lay(case, 8)
    ref = O.ffn_fwd_bwd(case.X, case.dOut, tok.batch, tok.seq, tok.ctx_len, lay, s)
    res = run_ffn_gpu(L, case, lay, idx_force=ref["idx"])
    _compare_ffn(res, ref, TOL["bf16"])
    res2 = run_ffn_gpu(L, case, lay)
    nd = check_selection(res2["idx"], ref["idx"], ref["scores"], ref["k"], "select")
    if nd == 0:
        _compare_ffn(res2, ref, TOL["bf16"])


def test_ffn_tc_repeatable(L):
    """Two runs on the same inputs give bit-identical outputs (fixed-order
    reductions everywhere, no atomics in the data path)."""
    tok = synth.Tokens(2, 256, np.asarray([192, 192], np.int32))
    case = synth.ffn_case(tok, 256, 688, 8, 16, 0.5, bf16=True, workload=0, layer=6)
    lay = _ffn_lay(case, 8)
    a = run_ffn_gpu(L, case, lay)
    b = run_ffn_gpu(L, case, lay)
    for k in ("out", "dX", "dAg", "dBg", "dAu", "dBu", "dAd", "dBd", "idx"):
        assert np.array_equal(a[k], b[k]), k

"""The C-ABI library loads and exports what include/slora.h declares; host-side
validation and workspace queries work without a GPU (no compute is called)."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "slora.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(slora_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    from contextual_sparsity_lora_svd_b200 import build
    build.build()
    from contextual_sparsity_lora_svd_b200 import _lib
    return _lib


def test_header_declares_the_five_calls():
    names = _declared()
    for n in ("slora_svd_prepare", "slora_estimate_select", "slora_linear_fwd",
              "slora_linear_bwd", "slora_ffn_fwd_bwd"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (slora_\w+)", out))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    for n in _declared():
        assert hasattr(L.lib(), n)
    assert sorted(L.EXPORTS) == _declared()


def test_version(L):
    assert L.version() == 100


FAKE = 0x10000  # 16-byte aligned dummy address: never dereferenced by validation/queries


def _ffn_query(L, **over):
    lay = L.ffn_layer_struct(256, 688, 8, 8, 1.0, *([FAKE] * 9), FAKE, FAKE, FAKE, FAKE)
    g = L.ffn_grads_struct(*([FAKE] * 6))
    args, keep = L.ffn_args(L.F32, lay, 1, 256, [192], over.get("s", 0.5), FAKE, FAKE, FAKE, FAKE,
                            g, FAKE)
    return L.workspace_size("slora_ffn_fwd_bwd", args), keep


def test_ffn_workspace_query_and_k(L):
    need, keep = _ffn_query(L)
    assert need > 0
    assert keep[2].value == 344


@pytest.mark.parametrize("s", [-0.1, 1.0, float("nan")])
def test_bad_sparsity_rejected(L, s):
    with pytest.raises(L.SloraError) as e:
        _ffn_query(L, s=s)
    assert e.value.status == 1


def test_misaligned_pointer_rejected(L):
    lay = L.ffn_layer_struct(256, 688, 8, 8, 1.0, FAKE + 2, *([FAKE] * 8), FAKE, FAKE, FAKE, FAKE)
    g = L.ffn_grads_struct(*([FAKE] * 6))
    args, keep = L.ffn_args(L.F32, lay, 1, 256, [192], 0.5, FAKE, FAKE, FAKE, FAKE, g, FAKE)
    with pytest.raises(L.SloraError) as e:
        L.workspace_size("slora_ffn_fwd_bwd", args)
    assert e.value.status == 3


def test_bad_shapes_rejected(L):
    tok, keep = L.make_tokens(2, 8, [3, 9])  # ctx_len > seq
    args = [L.SLICE_OUT_ROWS, ctypes.byref(tok), 16, 32, FAKE, FAKE, FAKE, 4, 1.0, 1, FAKE, 4,
            FAKE, FAKE, FAKE, FAKE, FAKE]
    args = [L.F32] + args[1:]
    with pytest.raises(L.SloraError) as e:
        L.workspace_size("slora_linear_fwd", args)
    assert e.value.status == 2
    tok2, keep2 = L.make_tokens(2, 8, [3, 8])
    ok = [L.F32, ctypes.byref(tok2), 16, 32, FAKE, FAKE, FAKE, 4, 1.0, L.SLICE_OUT_ROWS, FAKE, 4,
          FAKE, FAKE, FAKE, FAKE, FAKE]
    assert L.workspace_size("slora_linear_fwd", ok) > 0
    bad_idx = list(ok)
    bad_idx[11] = 33  # n_idx > n
    with pytest.raises(L.SloraError):
        L.workspace_size("slora_linear_fwd", bad_idx)
    bad_row = list(ok)
    bad_row[2] = 18  # k not a multiple of 4 (16-byte rows)
    with pytest.raises(L.SloraError):
        L.workspace_size("slora_linear_fwd", bad_row)


def test_estimate_select_query_qk_layout(L):
    tok, keep = L.make_tokens(4, 16, [12] * 4)
    k_out = ctypes.c_int32(0)
    args = [L.CRIT_QK, FAKE, L.BF16, ctypes.byref(tok), 64, FAKE, FAKE, 8 * 16, FAKE, FAKE, 2 * 16,
            8, 8, 2, 16, 0.5, FAKE, ctypes.byref(k_out), None]
    assert L.workspace_size("slora_estimate_select", args) > 0
    assert k_out.value == 8
    args[7] = 8 * 16 + 1  # n0 != heads*head_dim
    with pytest.raises(L.SloraError):
        L.workspace_size("slora_estimate_select", args)


def test_prepare_rank_limits(L):
    args = [FAKE, 64, 32, L.F32, 49, 0, 0, FAKE, FAKE, None]
    with pytest.raises(L.SloraError):
        L.workspace_size("slora_svd_prepare", args)
    args[4] = 8
    assert L.workspace_size("slora_svd_prepare", args) > 0


@pytest.mark.parametrize("ctx", [[0, 0, 0], [90, 90, 90], [1, 0, 89], [70, 33, 90]])
@pytest.mark.parametrize("s", [0.0, 0.3, 0.99])
@pytest.mark.parametrize("bf16", [False, True])
def test_ffn_workspace_query_edge_layouts(L, ctx, s, bf16):
    """Workspace planning handles empty context / output row sets and tiny k."""
    lay = L.ffn_layer_struct(72, 152, 6, 5, 0.5, *([FAKE] * 13))
    g = L.ffn_grads_struct(*([FAKE] * 6))
    args, keep = L.ffn_args(L.BF16 if bf16 else L.F32, lay, 3, 90, ctx, s, FAKE, FAKE, FAKE,
                            FAKE, g, FAKE)
    assert L.workspace_size("slora_ffn_fwd_bwd", args) > 0
    assert keep[2].value == 152 - int(np.floor(s * 152 + 1e-9))


def test_library_has_no_unresolved_internal_symbols(L):
    out = subprocess.run(["nm", "-D", "--undefined-only", L.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    assert "slora" not in out, out


def _est_query(L, crit, n0, n1, heads, kv, hd, s=0.5, L1=FAKE, U1=FAKE, d=64):
    tok, keep = L.make_tokens(4, 16, [12] * 4)
    k_out = ctypes.c_int32(0)
    args = [crit, FAKE, L.BF16, ctypes.byref(tok), d, FAKE, FAKE, n0, L1, U1, n1, 8, heads, kv,
            hd, s, FAKE, ctypes.byref(k_out), None]
    return L.workspace_size("slora_estimate_select", args), k_out.value


def test_estimate_select_query_variant_criteria(L):
    # rotate-half pairs: k_h = 2 * (16 - floor(0.5 * 16)) channels per head
    need, k = _est_query(L, L.CRIT_QK_ROPE_PAIR, 8 * 32, 2 * 32, 8, 2, 32)
    assert need > 0 and k == 16
    need, k = _est_query(L, L.CRIT_QK_ROPE_PAIR, 8 * 32, 2 * 32, 8, 2, 32, s=0.3)
    assert k == 2 * (16 - 4)
    with pytest.raises(L.SloraError) as e:  # odd head_dim has no rotate-half pairs
        _est_query(L, L.CRIT_QK_ROPE_PAIR, 8 * 33, 2 * 33, 8, 2, 33)
    assert e.value.status == 2
    # per-head L2 norm of one projection: the second factor pair may be NULL
    need, k = _est_query(L, L.CRIT_L2, 2 * 64, 0, 6, 2, 64, s=0.25, L1=None, U1=None)
    assert need > 0 and k == 48
    with pytest.raises(L.SloraError):  # n0 must be kv_heads * head_dim
        _est_query(L, L.CRIT_L2, 6 * 64, 0, 6, 2, 64, L1=None, U1=None)
    with pytest.raises(L.SloraError):  # heads a multiple of kv_heads
        _est_query(L, L.CRIT_L2, 4 * 64, 0, 6, 4, 64, L1=None, U1=None)
    # Gram FFN score: gate and up widths must agree; one selection spans <= 32768
    need, k = _est_query(L, L.CRIT_FFN_GRAM, 688, 688, 0, 0, 0)
    assert need > 0 and k == 344
    with pytest.raises(L.SloraError):
        _est_query(L, L.CRIT_FFN_GRAM, 688, 680, 0, 0, 0)
    with pytest.raises(L.SloraError) as e:
        _est_query(L, L.CRIT_FFN, 40000, 40000, 0, 0, 0)
    assert e.value.status == 2
    with pytest.raises(L.SloraError) as e:
        _est_query(L, 9, 688, 688, 0, 0, 0)
    assert e.value.status == 1


# ------------------------------------------- decoder-layer pieces (host side)
def _status(L, name, args):
    need = ctypes.c_size_t(0)
    return getattr(L.lib(), name)(*args, None, ctypes.byref(need), None), int(need.value)


def test_attention_and_norm_validation(L):
    tok, keep = L.make_tokens(2, 100, [75, 75])
    a = lambda dt, H, KV, hd, q=FAKE: [dt, ctypes.byref(tok), H, KV, hd, q, FAKE, FAKE, FAKE, FAKE]
    assert _status(L, "slora_attention_fwd", a(L.BF16, 4, 2, 128)) == (0, 0)
    assert _status(L, "slora_attention_fwd", a(L.F32, 4, 2, 128))[0] == 5       # UNSUPPORTED
    assert _status(L, "slora_attention_fwd", a(L.BF16, 4, 2, 96))[0] == 2       # SHAPE
    assert _status(L, "slora_attention_fwd", a(L.BF16, 4, 3, 64))[0] == 2       # heads % kv
    assert _status(L, "slora_attention_fwd", a(L.BF16, 4, 2, 64, FAKE + 8))[0] == 3  # ALIGN
    bw = [L.BF16, ctypes.byref(tok), 4, 2, 64] + [FAKE] * 9
    st, need = _status(L, "slora_attention_bwd", bw)
    assert st == 0 and need >= 200 * 4 * 4       # D: one float per (row, query head)
    nf = lambda T, d, A, N: [L.BF16, T, d, ctypes.c_float(1e-5), FAKE, A, FAKE, FAKE, N, FAKE]
    assert _status(L, "slora_rmsnorm_fwd", nf(16, 64, None, FAKE))[0] == 0
    assert _status(L, "slora_rmsnorm_fwd", nf(16, 60, None, FAKE))[0] == 2      # d % 8
    assert _status(L, "slora_rmsnorm_fwd", nf(16, 64, None, None))[0] == 1      # nothing out
    nb = [L.BF16, 16, 64, FAKE, FAKE, FAKE, None, None, None, None, FAKE]
    assert _status(L, "slora_rmsnorm_bwd", nb)[0] == 1                          # dN0 required
    del keep


def test_rope_validation_and_workspace(L):
    tok, keep = L.make_tokens(2, 100, [75, 70])
    base = ctypes.c_double(10000.0)
    dense = [L.BF16, ctypes.byref(tok), 512, 128, base, None, 0, FAKE, None, None, FAKE]
    st, need_dense = _status(L, "slora_rope_pack", dense)
    assert st == 0 and need_dense >= 100 * 64 * 8          # cos/sin table per (position, pair)
    sliced = [L.BF16, ctypes.byref(tok), 512, 128, base, FAKE, 256, None, FAKE, FAKE, FAKE]
    st, need = _status(L, "slora_rope_pack", sliced)
    assert st == 0 and need >= need_dense + 200 * 4 + 512 * 4  # + row kinds and channel map
    bad = list(sliced)
    bad[3] = 96
    assert _status(L, "slora_rope_pack", bad)[0] == 2
    bad = list(sliced)
    bad[6] = 513
    assert _status(L, "slora_rope_pack", bad)[0] == 2                           # n_idx > n
    bad = list(sliced)
    bad[4] = ctypes.c_double(1.0)
    assert _status(L, "slora_rope_pack", bad)[0] == 1                           # base <= 1
    un = [L.BF16, ctypes.byref(tok), 512, 128, base, FAKE, 256, FAKE, None, FAKE, FAKE]
    assert _status(L, "slora_rope_unpack", un)[0] == 0
    un[9] = None                                                                # dY_out missing
    assert _status(L, "slora_rope_unpack", un)[0] == 1
    del keep


def test_ffn_forward_only_needs_no_backward_buffers(L):
    lay = L.ffn_layer_struct(256, 688, 8, 8, 1.0, *([FAKE] * 9), FAKE, FAKE, FAKE, FAKE)
    args, keep = L.ffn_args(L.BF16, lay, 1, 256, [192], 0.5, FAKE, None, FAKE, None, None, FAKE)
    assert L.workspace_size("slora_ffn_fwd_bwd", args) > 0
    args, keep = L.ffn_args(L.BF16, lay, 1, 256, [192], 0.5, FAKE, FAKE, FAKE, None, None, FAKE)
    with pytest.raises(L.SloraError):
        L.workspace_size("slora_ffn_fwd_bwd", args)

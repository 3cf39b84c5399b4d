"""ctypes binding of libslora.so (the C ABI in include/slora.h).

Argument marshalling only: each function takes torch tensors (device memory
owned by the caller) or raw integer pointers, passes their addresses to the C
call of the same name on the current CUDA stream, and raises SloraError on a
non-zero status.  Workspace is taken from a caller tensor or, when omitted,
allocated once per call with torch (plumbing, not compute).  Nothing here
computes any part of the method; a missing library raises at import time.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libslora.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m contextual_sparsity_lora_svd_b200.build` "
        "(the CUDA library is required; there is no fallback)")
_lib = ctypes.CDLL(LIB_PATH)

c_int, c_i32, c_i64, c_u64, c_f32, c_vp, c_sz = (ctypes.c_int, ctypes.c_int32, ctypes.c_int64,
                                                  ctypes.c_uint64, ctypes.c_float, ctypes.c_void_p,
                                                  ctypes.c_size_t)
P_SZ = ctypes.POINTER(c_sz)
P_I32 = ctypes.POINTER(c_i32)

F32, BF16 = 0, 1
CRIT_FFN, CRIT_QK, CRIT_FFN_GRAM, CRIT_QK_ROPE_PAIR, CRIT_L2 = 0, 1, 2, 3, 4
SLICE_NONE, SLICE_OUT_ROWS, SLICE_IN_COLS = 0, 1, 2

STATUS = {0: "OK", 1: "INVALID_ARG", 2: "SHAPE", 3: "ALIGN", 4: "WORKSPACE", 5: "UNSUPPORTED",
          6: "CUDA", 7: "TIMEOUT"}


class SloraError(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__(f"{fn}: {STATUS.get(status, status)} ({status}): {msg}")
        self.status = status


class Tokens(ctypes.Structure):
    _fields_ = [("batch", c_i32), ("seq", c_i32), ("ctx_len", P_I32)]


class FfnLayer(ctypes.Structure):
    _fields_ = [("d", c_i64), ("d_ff", c_i64), ("r_svd", c_i32), ("r_lora", c_i32),
                ("lora_scale", c_f32),
                ("Wg", c_vp), ("Wu", c_vp), ("Wd_t", c_vp),
                ("Ag", c_vp), ("Bg", c_vp), ("Au", c_vp), ("Bu", c_vp), ("Ad", c_vp), ("Bd", c_vp),
                ("Lg", c_vp), ("Ug", c_vp), ("Lu", c_vp), ("Uu", c_vp)]


class FfnGrads(ctypes.Structure):
    _fields_ = [("dAg", c_vp), ("dBg", c_vp), ("dAu", c_vp), ("dBu", c_vp), ("dAd", c_vp),
                ("dBd", c_vp)]


def _sig(name, res, args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = args
    return f


_lib_err = _sig("slora_last_error_string", ctypes.c_char_p, [])
_sig("slora_version", c_int, [])
_sig("slora_device_error", c_int, [c_int])
_sig("slora_set_wait_budget", c_int, [c_i64])
_sig("slora_svd_prepare", c_int,
     [c_vp, c_i64, c_i64, c_int, c_int, c_int, c_u64, c_vp, c_vp, c_vp, c_vp, P_SZ, c_vp])
_sig("slora_estimate_select", c_int,
     [c_int, c_vp, c_int, ctypes.POINTER(Tokens), c_i64, c_vp, c_vp, c_i64, c_vp, c_vp, c_i64,
      c_int, c_int, c_int, c_int, ctypes.c_double, c_vp, P_I32, c_vp, c_vp, P_SZ, c_vp])
_LIN = [c_int, ctypes.POINTER(Tokens), c_i64, c_i64, c_vp, c_vp, c_vp, c_int, c_f32, c_int, c_vp,
        c_i32]
_sig("slora_linear_fwd", c_int, _LIN + [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, P_SZ, c_vp])
_sig("slora_linear_bwd", c_int,
     _LIN + [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, P_SZ, c_vp])
_sig("slora_ffn_fwd_bwd", c_int,
     [c_int, ctypes.POINTER(FfnLayer), ctypes.POINTER(Tokens), ctypes.c_double, c_vp, c_vp, c_vp,
      c_vp,
      ctypes.POINTER(FfnGrads), c_vp, P_I32, c_vp, c_i32, c_vp, P_SZ, c_vp])

_sig("slora_ffn_bwd", c_int,
     [c_int, ctypes.POINTER(FfnLayer), ctypes.POINTER(Tokens), ctypes.c_double, c_vp, c_vp, c_vp,
      c_vp, ctypes.POINTER(FfnGrads), c_vp, P_I32, c_vp, c_i32, c_vp, P_SZ, c_vp])
_sig("slora_ffn_fwd_bwd_per_seq", c_int,
     [c_int, ctypes.POINTER(FfnLayer), ctypes.POINTER(Tokens), ctypes.c_double, c_vp, c_vp, c_vp,
      c_vp, ctypes.POINTER(FfnGrads), c_vp, P_I32, c_vp, c_i32, c_vp, P_SZ, c_vp])
_sig("slora_rope_pack", c_int,
     [c_int, ctypes.POINTER(Tokens), c_i64, c_int, ctypes.c_double, c_vp, c_i32, c_vp, c_vp, c_vp,
      c_vp, c_vp, P_SZ, c_vp])
_sig("slora_rope_unpack", c_int,
     [c_int, ctypes.POINTER(Tokens), c_i64, c_int, ctypes.c_double, c_vp, c_i32, c_vp, c_vp, c_vp,
      c_vp, c_vp, P_SZ, c_vp])
_sig("slora_attention_fwd", c_int,
     [c_int, ctypes.POINTER(Tokens), c_int, c_int, c_int, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, P_SZ,
      c_vp])
_sig("slora_attention_bwd", c_int,
     [c_int, ctypes.POINTER(Tokens), c_int, c_int, c_int, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
      c_vp, c_vp, c_vp, P_SZ, c_vp])
_sig("slora_rmsnorm_fwd", c_int,
     [c_int, c_i64, c_i64, c_f32, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, P_SZ, c_vp])
_sig("slora_rmsnorm_bwd", c_int,
     [c_int, c_i64, c_i64, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, P_SZ, c_vp])

_sig("slora_noalloc_scratch_bytes", c_sz, [])
_sig("slora_estimate_select_noalloc", c_int,
     [c_int, c_vp, c_int, ctypes.POINTER(Tokens), c_i64, c_vp, c_vp, c_i64, c_vp, c_vp, c_i64,
      c_int, c_int, c_int, c_int, ctypes.c_double, c_vp, P_I32, c_vp, c_vp])
_sig("slora_launch_count", c_i64, [])
_sig("slora_profile_enable", None, [c_int])
_sig("slora_profile_read", c_int, [ctypes.c_char_p, ctypes.POINTER(c_i64),
                                   ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)])

EXPORTS = sorted(["slora_last_error_string", "slora_version", "slora_svd_prepare",
                  "slora_estimate_select", "slora_linear_fwd", "slora_linear_bwd",
                  "slora_ffn_fwd_bwd", "slora_launch_count", "slora_profile_enable",
                  "slora_profile_read", "slora_noalloc_scratch_bytes",
                  "slora_estimate_select_noalloc", "slora_device_error",
                  "slora_set_wait_budget", "slora_ffn_bwd", "slora_ffn_fwd_bwd_per_seq",
                  "slora_rope_pack", "slora_rope_unpack",
                  "slora_attention_fwd", "slora_attention_bwd", "slora_rmsnorm_fwd",
                  "slora_rmsnorm_bwd"])


def lib():
    return _lib


def version() -> int:
    return _lib.slora_version()


def launch_count() -> int:
    return int(_lib.slora_launch_count())


def profile_enable(on: bool) -> None:
    _lib.slora_profile_enable(1 if on else 0)


def profile_read(kernel_class: str) -> tuple[int, float, float]:
    """(launches, total_ms, work) recorded for a kernel class since enabling."""
    n, ms, w = c_i64(0), ctypes.c_double(0), ctypes.c_double(0)
    _check("slora_profile_read", _lib.slora_profile_read(kernel_class.encode(), ctypes.byref(n),
                                                         ctypes.byref(ms), ctypes.byref(w)))
    return int(n.value), float(ms.value), float(w.value)


KERNEL_CLASSES = ["gemm_tc", "gemm_simt", "estimate", "select", "elementwise", "aux", "prepare",
                  "skinny", "compact", "attention", "norm"]


def ptr(x) -> int | None:
    """Device address of a tensor (None/0 -> NULL)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x or None
    return x.data_ptr() or None


def dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream or None


def _check(fn, st):
    if st != 0:
        raise SloraError(fn, st, _lib_err().decode())


def make_tokens(batch: int, seq: int, ctx_len) -> tuple[Tokens, object]:
    """ctypes token struct; returns (struct, keep-alive host array)."""
    arr = (c_i32 * batch)(*[int(c) for c in ctx_len])
    return Tokens(batch, seq, ctypes.cast(arr, P_I32)), arr


def _run(fn_name, args_before_ws, ws, stream):
    """Query the workspace size, take/allocate it, run the call."""
    f = getattr(_lib, fn_name)
    need = c_sz(0)
    _check(fn_name, f(*args_before_ws, None, ctypes.byref(need), _stream(stream)))
    owned = None
    if ws is None:
        owned = torch.empty(max(int(need.value), 16), dtype=torch.uint8, device="cuda")
        ws = owned
    have = c_sz(ws.numel() * ws.element_size())
    _check(fn_name, f(*args_before_ws, ptr(ws), ctypes.byref(have), _stream(stream)))
    return owned


def workspace_size(fn_name, args_before_ws) -> int:
    f = getattr(_lib, fn_name)
    need = c_sz(0)
    _check(fn_name, f(*args_before_ws, None, ctypes.byref(need), None))
    return int(need.value)


# ------------------------------------------------------------------ calls
def slora_svd_prepare(W, rank, L, U, W_t=None, n_iter=0, seed=0, ws=None, stream=None):
    n, k = W.shape
    return _run("slora_svd_prepare",
                [ptr(W), n, k, dtype_code(W), rank, n_iter, seed, ptr(L), ptr(U), ptr(W_t)],
                ws, stream)


def slora_estimate_select(crit, X, batch, seq, ctx_len, L0, U0, L1, U1, rank, sparsity, idx_out,
                          heads=0, kv_heads=0, head_dim=0, scores_out=None, ws=None, stream=None):
    """Returns k_keep (FFN) or k_h (QK)."""
    tok, keep = make_tokens(batch, seq, ctx_len)
    k_out = c_i32(0)
    _run("slora_estimate_select",
         [crit, ptr(X), dtype_code(X), ctypes.byref(tok), X.shape[1], ptr(L0), ptr(U0),
          U0.shape[0], ptr(L1), ptr(U1), U1.shape[0], rank, heads, kv_heads, head_dim,
          float(sparsity), ptr(idx_out), ctypes.byref(k_out), ptr(scores_out)], ws, stream)
    del keep
    return int(k_out.value)


def slora_estimate_select_noalloc(crit, X, batch, seq, ctx_len, L0, U0, L1, U1, rank, sparsity,
                                  idx_out, heads=0, kv_heads=0, head_dim=0, scores_out=None,
                                  stream=None):
    """slora_estimate_select with the library's built-in scratch buffer (no
    workspace argument, nothing allocated).  Returns k_keep (FFN) or k_h (QK)."""
    tok, keep = make_tokens(batch, seq, ctx_len)
    k_out = c_i32(0)
    _check("slora_estimate_select_noalloc", _lib.slora_estimate_select_noalloc(
        crit, ptr(X), dtype_code(X), ctypes.byref(tok), X.shape[1], ptr(L0), ptr(U0),
        U0.shape[0], ptr(L1), ptr(U1), U1.shape[0], rank, heads, kv_heads, head_dim,
        float(sparsity), ptr(idx_out), ctypes.byref(k_out), ptr(scores_out), _stream(stream)))
    del keep
    return int(k_out.value)


def noalloc_scratch_bytes() -> int:
    return int(_lib.slora_noalloc_scratch_bytes())


def slora_linear_fwd(side, batch, seq, ctx_len, k, n, W, A, B, lora_scale, idx, X_ctx,
                     Y_ctx, X_out=None, Y_out=None, XA_save=None, ws=None, stream=None):
    tok, keep = make_tokens(batch, seq, ctx_len)
    n_idx = 0 if idx is None else idx.numel()
    _run("slora_linear_fwd",
         [dtype_code(W), ctypes.byref(tok), k, n, ptr(W), ptr(A), ptr(B), A.shape[0],
          float(lora_scale), side, ptr(idx), n_idx, ptr(X_ctx), ptr(X_out), ptr(Y_ctx),
          ptr(Y_out), ptr(XA_save)], ws, stream)
    del keep


def slora_linear_bwd(side, batch, seq, ctx_len, k, n, W, A, B, lora_scale, idx, X_ctx, XA_save,
                     dY_ctx, dX_ctx, dA, dB, X_out=None, dY_out=None, dX_out=None, ws=None,
                     stream=None):
    tok, keep = make_tokens(batch, seq, ctx_len)
    n_idx = 0 if idx is None else idx.numel()
    _run("slora_linear_bwd",
         [dtype_code(W), ctypes.byref(tok), k, n, ptr(W), ptr(A), ptr(B), A.shape[0],
          float(lora_scale), side, ptr(idx), n_idx, ptr(X_ctx), ptr(X_out), ptr(XA_save),
          ptr(dY_ctx), ptr(dY_out), ptr(dX_ctx), ptr(dX_out), ptr(dA), ptr(dB)], ws, stream)
    del keep


def ffn_layer_struct(d, d_ff, r_svd, r_lora, lora_scale, Wg, Wu, Wd_t, Ag, Bg, Au, Bu, Ad, Bd,
                     Lg=None, Ug=None, Lu=None, Uu=None) -> FfnLayer:
    return FfnLayer(d, d_ff, r_svd, r_lora, float(lora_scale), ptr(Wg), ptr(Wu), ptr(Wd_t),
                    ptr(Ag), ptr(Bg), ptr(Au), ptr(Bu), ptr(Ad), ptr(Bd), ptr(Lg), ptr(Ug),
                    ptr(Lu), ptr(Uu))


def ffn_grads_struct(dAg, dBg, dAu, dBu, dAd, dBd) -> FfnGrads:
    return FfnGrads(ptr(dAg), ptr(dBg), ptr(dAu), ptr(dBu), ptr(dAd), ptr(dBd))


def ffn_args(dt, layer, batch, seq, ctx_len, sparsity, X, dOut, out, dX, grads, idx_out,
             idx_force=None):
    """Positional arguments of slora_ffn_fwd_bwd before (ws, ws_bytes, stream)
    plus the objects that must stay alive while they are used."""
    tok, keep = make_tokens(batch, seq, ctx_len)
    k_out = c_i32(0)
    k_force = 0 if idx_force is None else idx_force.numel()
    args = [dt, ctypes.byref(layer), ctypes.byref(tok), float(sparsity), ptr(X), ptr(dOut),
            ptr(out), ptr(dX), None if grads is None else ctypes.byref(grads), ptr(idx_out),
            ctypes.byref(k_out),
            ptr(idx_force), k_force]
    return args, (tok, keep, k_out, layer, grads)


def slora_ffn_fwd_bwd(layer: FfnLayer, batch, seq, ctx_len, sparsity, X, dOut, out, dX,
                      grads: FfnGrads, idx_out, idx_force=None, ws=None, stream=None,
                      per_sequence=False) -> int:
    """Returns k_keep.  per_sequence: one channel set per sequence
    (slora_ffn_fwd_bwd_per_seq; idx_out is [batch x d_ff], idx_force
    [batch x k_force])."""
    args, keep = ffn_args(dtype_code(X), layer, batch, seq, ctx_len, sparsity, X, dOut, out, dX,
                          grads, idx_out, idx_force)
    if per_sequence and idx_force is not None:
        args[-1] = idx_force.numel() // batch
    _run("slora_ffn_fwd_bwd_per_seq" if per_sequence else "slora_ffn_fwd_bwd", args, ws, stream)
    return int(keep[2].value)


def slora_ffn_bwd(layer: FfnLayer, batch, seq, ctx_len, sparsity, X, dOut, out, dX,
                  grads: FfnGrads, idx_out, ws, idx_force=None, stream=None) -> int:
    """The backward half on the workspace `ws` of an earlier forward-only
    slora_ffn_fwd_bwd call with the same arguments.  Returns k_keep."""
    args, keep = ffn_args(dtype_code(X), layer, batch, seq, ctx_len, sparsity, X, dOut, out, dX,
                          grads, idx_out, idx_force)
    _run("slora_ffn_bwd", args, ws, stream)
    return int(keep[2].value)


def ffn_workspace_bytes(layer: FfnLayer, batch, seq, ctx_len, sparsity, X, out, idx_out,
                        idx_force=None) -> int:
    args, keep = ffn_args(dtype_code(X), layer, batch, seq, ctx_len, sparsity, X, None, out, None,
                          None, idx_out, idx_force)
    return workspace_size("slora_ffn_fwd_bwd", args)


# ------------------------------------------- decoder-layer pieces
ROPE_BASE = 10000.0
RMS_EPS = 1e-5


def slora_rope_pack(batch, seq, ctx_len, n, head_dim, Y_rot, Y=None, Y_ctx=None, Y_out=None,
                    idx=None, rope_base=ROPE_BASE, ws=None, stream=None):
    tok, keep = make_tokens(batch, seq, ctx_len)
    n_idx = 0 if idx is None else idx.numel()
    _run("slora_rope_pack", [BF16, ctypes.byref(tok), n, head_dim, float(rope_base), ptr(idx),
                             n_idx, ptr(Y), ptr(Y_ctx), ptr(Y_out), ptr(Y_rot)], ws, stream)
    del keep


def slora_rope_unpack(batch, seq, ctx_len, n, head_dim, G, dY=None, dY_ctx=None, dY_out=None,
                      idx=None, rope_base=ROPE_BASE, ws=None, stream=None):
    tok, keep = make_tokens(batch, seq, ctx_len)
    n_idx = 0 if idx is None else idx.numel()
    _run("slora_rope_unpack", [BF16, ctypes.byref(tok), n, head_dim, float(rope_base), ptr(idx),
                               n_idx, ptr(G), ptr(dY), ptr(dY_ctx), ptr(dY_out)], ws, stream)
    del keep


def slora_attention_fwd(batch, seq, heads, kv_heads, head_dim, Q, K, V, O, lse, stream=None):
    tok, keep = make_tokens(batch, seq, [seq] * batch)
    _run("slora_attention_fwd", [BF16, ctypes.byref(tok), heads, kv_heads, head_dim, ptr(Q),
                                 ptr(K), ptr(V), ptr(O), ptr(lse)], None, stream)
    del keep


def slora_attention_bwd(batch, seq, heads, kv_heads, head_dim, Q, K, V, O, lse, dO, dQ, dK, dV,
                        ws=None, stream=None):
    tok, keep = make_tokens(batch, seq, [seq] * batch)
    _run("slora_attention_bwd", [BF16, ctypes.byref(tok), heads, kv_heads, head_dim, ptr(Q),
                                 ptr(K), ptr(V), ptr(O), ptr(lse), ptr(dO), ptr(dQ), ptr(dK),
                                 ptr(dV)], ws, stream)
    del keep


def slora_rmsnorm_fwd(X, g, N=None, A=None, H=None, rstd=None, eps=RMS_EPS, stream=None):
    T, d = X.shape
    _run("slora_rmsnorm_fwd", [BF16, T, d, float(eps), ptr(X), ptr(A), ptr(g), ptr(H), ptr(N),
                               ptr(rstd)], None, stream)


def slora_rmsnorm_bwd(H, rstd, g, dN0, dX, dN1=None, dN2=None, dRes=None, stream=None):
    T, d = H.shape
    _run("slora_rmsnorm_bwd", [BF16, T, d, ptr(H), ptr(rstd), ptr(g), ptr(dN0), ptr(dN1),
                               ptr(dN2), ptr(dRes), ptr(dX)], None, stream)

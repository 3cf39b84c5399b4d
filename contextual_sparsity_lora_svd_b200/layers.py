"""Device-side layer runners: the buffers of one transformer layer's LoRA
linears and the order of the library calls that make one training step.

Each runner holds device tensors (weights, LoRA factors, estimator factors,
activations, outputs, gradients), prepares the C-ABI argument lists once, and
issues the step's calls on one stream with a caller-owned workspace, so a step
can be captured into a CUDA graph and replayed.  Nothing here computes any
part of the method: every number is produced by libslora's kernels.

  FfnLayer      one SwiGLU FFN: slora_ffn_fwd_bwd (estimate, select, sliced
                forward and backward; a ratio of 0 runs every channel through
                idx_force, the dense path).
  AttnLinears   the q/k/v/o LoRA linears of one attention layer around a
                stand-in for the attention core (its output is an input
                tensor: the core itself is not part of this library).  q/k are
                sliced per head by the QK-norm criterion (or the rotate-half
                pair criterion); v/o are dense, or, with `vo_sparsity` > 0,
                v is sliced on its output channels and o on the matching input
                channels by the per-head L2 criterion (SparseLoRA article,
                sections 1 and 6).
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib as L

__all__ = ["FfnLayer", "AttnLinears", "lora_grad_shapes_ffn"]


def _bf16_empty(*shape):
    return torch.empty(*shape, dtype=torch.bfloat16, device="cuda")


def lora_grad_shapes_ffn(d, d_ff, r):
    return [(r, d), (d_ff, r), (r, d), (d_ff, r), (r, d_ff), (d, r)]


class _Call:
    """One library call with its argument list fixed (before ws, ws_bytes,
    stream) and the objects that must stay alive while it is used."""

    def __init__(self, name, args, keep=()):
        self.fn = getattr(L.lib(), name)
        self.name, self.args, self.keep = name, args, keep

    def need(self) -> int:
        need = L.c_sz(0)
        L._check(self.name, self.fn(*self.args, None, ctypes.byref(need), None))
        return int(need.value)

    def __call__(self, ws_ptr, ws_bytes, stream):
        L._check(self.name, self.fn(*self.args, ws_ptr, ctypes.byref(ws_bytes), stream))


class _Runner:
    calls: list

    def workspace_bytes(self) -> int:
        return max([c.need() for c in self.calls] + [16])

    def step(self, ws: torch.Tensor, stream=None):
        st = (stream or torch.cuda.current_stream()).cuda_stream
        ptr, nb = ws.data_ptr(), L.c_sz(ws.numel())
        for c in self.calls:
            c(ptr, nb, st)


class FfnLayer(_Runner):
    """One SwiGLU FFN layer step.  `w` holds device tensors Wg, Wu [d_ff x d],
    Wd_t [d_ff x d] (the transposed down weight), Ag, Bg, Au, Bu, Ad, Bd (bf16)
    and the fp32 estimator factors Lg, Ug, Lu, Uu."""

    def __init__(self, w, d, d_ff, r_svd, r_lora, scale, batch, seq, ctx_len, sparsity, X, dOut):
        # the argument lists hold raw device addresses of w, X and dOut, which
        # the runner keeps alive
        self.w, self.d, self.d_ff, self.r = w, d, d_ff, r_lora
        self.sparsity = float(sparsity)
        T = batch * seq
        self.X, self.dOut = X, dOut
        self.out, self.dX = _bf16_empty(T, d), _bf16_empty(T, d)
        shapes = lora_grad_shapes_ffn(d, d_ff, r_lora)
        self.gflat = torch.zeros(sum(a * b for a, b in shapes), device="cuda")
        self.grads, o = [], 0
        for a, b in shapes:
            self.grads.append(self.gflat[o:o + a * b].view(a, b))
            o += a * b
        self.idx = torch.empty(d_ff, dtype=torch.int32, device="cuda")
        # a ratio of 0 is the dense path: every channel, no estimator
        self.force = (torch.arange(d_ff, dtype=torch.int32, device="cuda")
                      if self.sparsity == 0.0 else None)
        self.layer = L.ffn_layer_struct(d, d_ff, r_svd, r_lora, scale, w["Wg"], w["Wu"],
                                        w["Wd_t"], w["Ag"], w["Bg"], w["Au"], w["Bu"], w["Ad"],
                                        w["Bd"], w.get("Lg"), w.get("Ug"), w.get("Lu"),
                                        w.get("Uu"))
        self.gstruct = L.ffn_grads_struct(*self.grads)
        args, keep = L.ffn_args(L.BF16, self.layer, batch, seq, ctx_len, self.sparsity, X, dOut,
                                self.out, self.dX, self.gstruct, self.idx, self.force)
        self.calls = [_Call("slora_ffn_fwd_bwd", args, keep + (self.layer, self.gstruct))]
        self._kout = keep[2]

    def kept(self) -> int:
        return int(self._kout.value)


class AttnLinears(_Runner):
    """The four LoRA linears of one attention layer for one step.

    `w` holds Wq [H*hd x d], Wk, Wv [KV*hd x d], Wo [d x H*hd] (plus Wo_t
    [H*hd x d] when v/o are sliced), A*/B* LoRA factors (bf16), and the
    fp32 estimator factors Lq, Uq, Lk, Uk (and Lv, Uv for the v/o criterion).
    X [T x d] is the layer input; attn_out [T x H*hd] stands in for the output
    of the attention core (the input of o); dY_o [T x d] is the upstream
    gradient of o; dq, dk, dv stand in for the gradients the core returns.
    """

    def __init__(self, w, d, heads, kv_heads, head_dim, r_svd, r_lora, scale, batch, seq, ctx_len,
                 qk_sparsity, X, attn_out, dY_o, dq, dk, dv, pairs=False, vo_sparsity=0.0):
        self.w = w
        # the argument lists below hold raw device addresses: keep every
        # caller tensor they point into alive as long as the runner
        self._inputs = (X, attn_out, dY_o, dq, dk, dv)
        H, KV, hd = heads, kv_heads, head_dim
        nq, nkv = H * hd, KV * hd
        T = batch * seq
        tok, tok_keep = L.make_tokens(batch, seq, ctx_len)
        self._tok, self._tok_keep = tok, tok_keep
        TC = int(sum(int(c) for c in ctx_len))
        TO = T - TC
        self.T, self.TC, self.TO = T, TC, TO
        s = float(scale)
        calls = []
        f32 = lambda *sh: torch.empty(*sh, device="cuda")
        self.bufs = {}

        def est_call(crit, L0, U0, n0, L1, U1, n1, sp, ncols, nsc):
            idx = torch.empty(ncols, dtype=torch.int32, device="cuda")
            k_out = L.c_i32(0)
            scores = f32(nsc)
            args = [crit, L.ptr(X), L.BF16, ctypes.byref(tok), d, L.ptr(L0), L.ptr(U0), n0,
                    L.ptr(L1), L.ptr(U1), n1, r_svd, H, KV, hd, float(sp), L.ptr(idx),
                    ctypes.byref(k_out), L.ptr(scores)]
            c = _Call("slora_estimate_select", args, (k_out, idx, scores))
            c.need()  # validates and fills k_out (channels kept per head)
            return c, idx, int(k_out.value)

        def lin(name, side, k, n, W, A, B, idx, n_idx, X_ctx, X_out, Y_ctx, Y_out, XA, dY_ctx,
                dY_out, dX_ctx, dX_out, dA, dB):
            base = [L.BF16, ctypes.byref(tok), k, n, L.ptr(W), L.ptr(A), L.ptr(B), A.shape[0], s,
                    side, L.ptr(idx), n_idx]
            fwd = _Call("slora_linear_fwd", base + [L.ptr(X_ctx), L.ptr(X_out), L.ptr(Y_ctx),
                                                    L.ptr(Y_out), L.ptr(XA)])
            bwd = _Call("slora_linear_bwd", base + [L.ptr(X_ctx), L.ptr(X_out), L.ptr(XA),
                                                    L.ptr(dY_ctx), L.ptr(dY_out),
                                                    L.ptr(dX_ctx), L.ptr(dX_out), L.ptr(dA),
                                                    L.ptr(dB)])
            return fwd, bwd

        r = r_lora
        # the eight LoRA gradients are views of one flat fp32 buffer (one
        # all-reduce, one read-back); every view starts on 16 bytes
        shapes = []
        for nm, n, k in (("q", nq, d), ("k", nkv, d), ("v", nkv, d), ("o", d, nq)):
            shapes += [("dA" + nm, (r, k)), ("dB" + nm, (n, r))]
        sizes = [(a * b + 3) // 4 * 4 for _, (a, b) in shapes]
        self.gflat = torch.zeros(sum(sizes), device="cuda")
        grads, o = {}, 0
        for (key, (a, b)), sz in zip(shapes, sizes):
            grads[key] = self.gflat[o:o + a * b].view(a, b)
            o += sz
        self.grads = grads
        self.dX = {nm: _bf16_empty(T, d) for nm in ("q", "k", "v")}
        fwds, bwds = [], []
        # ---- q / k: sliced per head on their output channels
        self.kh = hd
        if qk_sparsity > 0.0:
            crit = L.CRIT_QK_ROPE_PAIR if pairs else L.CRIT_QK
            c, idx, kh = est_call(crit, w["Lq"], w["Uq"], nq, w["Lk"], w["Uk"], nkv, qk_sparsity,
                                  (H + KV) * hd, KV * (hd // 2 if pairs else hd))
            calls.append(c)
            self.kh, self.idx_qk = kh, idx
            iq, ik = idx[:H * kh], idx[H * kh:H * kh + KV * kh]
            for nm, n, ii, dY_full in (("q", nq, iq, dq), ("k", nkv, ik, dk)):
                ni = ii.numel()
                Yc, Yo = _bf16_empty(TC, ni), _bf16_empty(TO, n)
                dYc, dYo = _bf16_empty(TC, ni), _bf16_empty(TO, n)
                dYc.normal_()
                dYo.normal_()
                XA = f32(T, r)
                self.bufs[nm] = (Yc, Yo, dYc, dYo, XA)
                f, b = lin(nm, L.SLICE_OUT_ROWS, d, n, w["W" + nm], w["A" + nm], w["B" + nm], ii,
                           ni, X, None, Yc, Yo, XA, dYc, dYo, self.dX[nm], None,
                           grads["dA" + nm], grads["dB" + nm])
                fwds.append(f)
                bwds.append(b)
        else:
            for nm, n, dY_full in (("q", nq, dq), ("k", nkv, dk)):
                Y, XA = _bf16_empty(T, n), f32(T, r)
                self.bufs[nm] = (Y, XA)
                f, b = lin(nm, L.SLICE_NONE, d, n, w["W" + nm], w["A" + nm], w["B" + nm], None, 0,
                           X, None, Y, None, XA, dY_full, None, self.dX[nm], None,
                           grads["dA" + nm], grads["dB" + nm])
                fwds.append(f)
                bwds.append(b)
        # ---- v / o
        self.kv_keep = hd
        if vo_sparsity > 0.0:
            c, idx, kv = est_call(L.CRIT_L2, w["Lv"], w["Uv"], nkv, w["Lv"], w["Uv"], nkv,
                                  vo_sparsity, (H + KV) * hd, KV * hd)
            calls.append(c)
            self.kv_keep, self.idx_vo = kv, idx
            io, iv = idx[:H * kv], idx[H * kv:H * kv + KV * kv]
            nv, no = iv.numel(), io.numel()
            Yc, Yo = _bf16_empty(TC, nv), _bf16_empty(TO, nkv)
            dYc, dYo = _bf16_empty(TC, nv), _bf16_empty(TO, nkv)
            dYc.normal_()
            dYo.normal_()
            XAv = f32(T, r)
            f, b = lin("v", L.SLICE_OUT_ROWS, d, nkv, w["Wv"], w["Av"], w["Bv"], iv, nv, X, None,
                       Yc, Yo, XAv, dYc, dYo, self.dX["v"], None, grads["dAv"], grads["dBv"])
            fwds.append(f)
            bwds.append(b)
            # o reads only the kept input channels for context rows: its compact
            # context input stands in for the attention output on those channels
            Xoc, Xoo = _bf16_empty(TC, no), _bf16_empty(TO, nq)
            Xoc.normal_()
            Xoo.normal_()
            Yo_full, XAo = _bf16_empty(T, d), f32(T, r)
            dXoc, dXoo = _bf16_empty(TC, no), _bf16_empty(TO, nq)
            self.bufs["v"] = (Yc, Yo, dYc, dYo, XAv)
            self.bufs["o"] = (Xoc, Xoo, Yo_full, XAo, dXoc, dXoo)
            f, b = lin("o", L.SLICE_IN_COLS, nq, d, w["Wo_t"], w["Ao"], w["Bo"], io, no, Xoc, Xoo,
                       Yo_full, None, XAo, dY_o, None, dXoc, dXoo, grads["dAo"], grads["dBo"])
            fwds.append(f)
            bwds.append(b)
        else:
            Yv, XAv = _bf16_empty(T, nkv), f32(T, r)
            f, b = lin("v", L.SLICE_NONE, d, nkv, w["Wv"], w["Av"], w["Bv"], None, 0, X, None, Yv,
                       None, XAv, dv, None, self.dX["v"], None, grads["dAv"], grads["dBv"])
            fwds.append(f)
            bwds.append(b)
            Yo_full, XAo, dXo = _bf16_empty(T, d), f32(T, r), _bf16_empty(T, nq)
            self.bufs["v"] = (Yv, XAv)
            self.bufs["o"] = (Yo_full, XAo, dXo)
            f, b = lin("o", L.SLICE_NONE, nq, d, w["Wo"], w["Ao"], w["Bo"], None, 0, attn_out,
                       None, Yo_full, None, XAo, dY_o, None, dXo, None, grads["dAo"],
                       grads["dBo"])
            fwds.append(f)
            bwds.append(b)
        # step: estimators, forwards (q, k, v, o), backwards in reverse order
        self.calls = calls + fwds + bwds[::-1]
        self.X, self.attn_out, self.dY_o = X, attn_out, dY_o

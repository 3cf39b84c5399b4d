"""Device-side layer runners: the buffers of one transformer layer's LoRA
linears and the order of the library calls that make one training step.

Each runner holds device tensors (weights, LoRA factors, estimator factors,
activations, outputs, gradients), prepares the C-ABI argument lists once, and
issues the step's calls on one stream with a caller-owned workspace, so a step
can be captured into a CUDA graph and replayed.  Nothing here computes any
part of the method: every number is produced by libslora's kernels.

  FfnLayer      one SwiGLU FFN: slora_ffn_fwd_bwd (estimate, select, sliced
                forward and backward; a ratio of 0 runs every channel through
                idx_force, the dense path), or with per_sequence one channel set
                per sequence (slora_ffn_fwd_bwd_per_seq).
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
    stream) and the objects that must stay alive while it is used.  A call
    with `own_ws` (a device tensor) runs on that workspace instead of the
    runner's shared one (state kept from one call to a later one)."""

    def __init__(self, name, args, keep=(), own_ws=None):
        self.fn = getattr(L.lib(), name)
        self.name, self.args, self.keep, self.own_ws = name, args, keep, own_ws

    def need(self) -> int:
        need = L.c_sz(0)
        L._check(self.name, self.fn(*self.args, None, ctypes.byref(need), None))
        return int(need.value)

    def __call__(self, ws_ptr, ws_bytes, stream):
        if self.own_ws is not None:
            ws_ptr, ws_bytes = self.own_ws.data_ptr(), L.c_sz(self.own_ws.numel())
        L._check(self.name, self.fn(*self.args, ws_ptr, ctypes.byref(ws_bytes), stream))


class _Par:
    """Independent call lists issued at once: the first runs on the runner's
    stream and workspace, list i > 0 on the runner's branch stream i - 1 with
    its own branch workspace.  The branches fork from the runner's stream
    and are joined back into it (events, so this holds inside a CUDA-graph
    capture too).  The lists must not share any buffer they write."""

    def __init__(self, *branches):
        self.branches = [list(b) for b in branches]
        self.fork = torch.cuda.Event()
        self.joins = [torch.cuda.Event() for _ in self.branches[1:]]


class _Runner:
    calls: list
    _bstreams: list = []
    _bws: list = []
    # serial: the branches of each _Par group run one after another on the
    # runner's stream (each still on its own workspace); for per-launch
    # timings that must not include other branches' work
    serial = False

    def _main_calls(self):
        for c in self.calls:
            if isinstance(c, _Par):
                yield from c.branches[0]
            else:
                yield c

    def workspace_bytes(self) -> int:
        return max([c.need() for c in self._main_calls() if c.own_ws is None] + [16])

    def _setup_branches(self):
        """Streams and workspaces of the branches of the _Par groups."""
        pars = [c for c in self.calls if isinstance(c, _Par)]
        nb = max([len(c.branches) for c in pars] + [1])
        self._bstreams = [torch.cuda.Stream() for _ in range(nb - 1)]
        self._bws = []
        for i in range(1, nb):
            need = max([16] + [x.need() for c in pars if len(c.branches) > i
                               for x in c.branches[i]])
            self._bws.append(torch.empty(need, dtype=torch.uint8, device="cuda"))

    def step(self, ws: torch.Tensor, stream=None):
        cur = stream or torch.cuda.current_stream()
        st = cur.cuda_stream
        ptr, nb = ws.data_ptr(), L.c_sz(ws.numel())
        for c in self.calls:
            if not isinstance(c, _Par):
                c(ptr, nb, st)
                continue
            if self.serial:
                for x in c.branches[0]:
                    x(ptr, nb, st)
                for i, br in enumerate(c.branches[1:]):
                    bw = self._bws[i]
                    for x in br:
                        x(bw.data_ptr(), L.c_sz(bw.numel()), st)
                continue
            c.fork.record(cur)
            for i, br in enumerate(c.branches[1:]):
                bs, bw = self._bstreams[i], self._bws[i]
                bs.wait_event(c.fork)
                for x in br:
                    x(bw.data_ptr(), L.c_sz(bw.numel()), bs.cuda_stream)
                c.joins[i].record(bs)
            for x in c.branches[0]:
                x(ptr, nb, st)
            for e in c.joins:
                cur.wait_event(e)


class FfnLayer(_Runner):
    """One SwiGLU FFN layer step.  `w` holds device tensors Wg, Wu [d_ff x d],
    Wd_t [d_ff x d] (the transposed down weight), Ag, Bg, Au, Bu, Ad, Bd (bf16)
    and the fp32 estimator factors Lg, Ug, Lu, Uu."""

    def __init__(self, w, d, d_ff, r_svd, r_lora, scale, batch, seq, ctx_len, sparsity, X, dOut,
                 per_sequence=False):
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
        # per_sequence: one channel set per sequence (idx holds batch sets of d_ff)
        self.idx = torch.empty(d_ff * (batch if per_sequence else 1), dtype=torch.int32,
                               device="cuda")
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
        name = "slora_ffn_fwd_bwd_per_seq" if per_sequence else "slora_ffn_fwd_bwd"
        self.calls = [_Call(name, args, keep + (self.layer, self.gstruct))]
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
        # step: estimators; q, k and v forwards at once (each writes only its
        # own buffers), then o, whose input in a layer is the attention output
        # over q, k, v; backward: o first (its input gradient feeds the
        # attention backward), then q, k and v at once
        self.calls = calls + [_Par([fwds[0]], [fwds[1]], [fwds[2]]), fwds[3], bwds[3],
                              _Par([bwds[2]], [bwds[1]], [bwds[0]])]
        self.X, self.attn_out, self.dY_o = X, attn_out, dY_o
        self._setup_branches()


class DecoderStack(_Runner):
    """One training step of a stack of decoder layers, every number on
    libslora's kernels:

      forward, per layer:  n1 = rms(x); q/k channel selection on n1 (QK-norm,
        per head) for sparse layers; q, k (sliced on context rows), v, o LoRA
        linears; rotary packing of q, k; causal attention; h = x + o(attn);
        n2 = rms(h); FFN forward only (its own estimate + select);
        x' = h + ffn (fused into the next normalisation);
      backward, last layer first: the FFN's sparse backward from the state
        its forward call left in the layer's own workspace, the norm backward
        with the residual, o backward, attention backward, rotary unpacking, q/k/v
        backward, the norm backward summing the three branch gradients and the
        residual.

    `layers` holds one dict per layer of device tensors: g1, g2 (RMS gains,
    bf16 [d]), Wq, Wk, Wv, Wo and their A*/B* LoRA factors, the FFN weights
    Wg, Wu, Wd_t with Ag..Bd, and the fp32 estimator factors Lq, Uq, Lk, Uk,
    Lg, Ug, Lu, Uu.  `qk_sparsity` / `ffn_sparsity` give each layer's ratio (0:
    dense).  X [T x d] is the stack input, dY [T x d] the gradient of its
    output.  After step(): `y` is the output, `dX` the input gradient,
    `grads[l]` layer l's LoRA gradients (views of `gflat`), `idx_qk[l]` /
    `idx_ffn[l]` (first `k_ffn[l]` entries) the channel sets used."""

    GRAD_ORDER = ("q", "k", "v", "o")

    def __init__(self, layers, d, heads, kv_heads, head_dim, d_ff, r_svd, r_lora, scale, batch,
                 seq, ctx_len, qk_sparsity, ffn_sparsity, X, dY, rope_base=10000.0,
                 eps=1e-5):
        H, KV, hd = heads, kv_heads, head_dim
        nq, nkv, T = H * hd, KV * hd, batch * seq
        tok, tok_keep = L.make_tokens(batch, seq, ctx_len)
        self._keep = [tok, tok_keep, X, dY, layers]
        TC = int(sum(int(c) for c in ctx_len))
        TO = T - TC
        s = float(scale)
        r = r_lora
        bf = _bf16_empty
        f32 = lambda *sh: torch.empty(*sh, device="cuda")
        nl = len(layers)
        self.nl = nl
        # ---- saved activations, per layer
        self.x = [X] + [bf(T, d) for _ in range(nl - 1)]
        self.y = bf(T, d)
        sv = []
        for _ in range(nl):
            sv.append(dict(n1=bf(T, d), r1=f32(T), Qr=bf(T, nq), Kr=bf(T, nkv), V=bf(T, nkv),
                           O=bf(T, nq), lse=f32(batch, H, seq), XAq=f32(T, r), XAk=f32(T, r),
                           XAv=f32(T, r), XAo=f32(T, r), h=bf(T, d), n2=bf(T, d), r2=f32(T)))
        self.saved = sv
        # ---- scratch shared by the layers
        a_out, f_out = bf(T, d), bf(T, d)
        dn2, dh, dxq, dxk, dxv = bf(T, d), bf(T, d), bf(T, d), bf(T, d), bf(T, d)
        dx_pp = [bf(T, d), bf(T, d)]
        dO_att = bf(T, nq)
        dQr, dKr, dV = f32(T, nq), f32(T, nkv), bf(T, nkv)
        self._scratch = (a_out, f_out, dn2, dh, dxq, dxk, dxv, dx_pp, dO_att, dQr, dKr, dV)
        # ---- gradients: one flat fp32 buffer, 16-byte aligned views
        shapes = []
        for nm, n, k in (("q", nq, d), ("k", nkv, d), ("v", nkv, d), ("o", d, nq)):
            shapes += [("dA" + nm, (r, k)), ("dB" + nm, (n, r))]
        shapes += list(zip(("dAg", "dBg", "dAu", "dBu", "dAd", "dBd"),
                           lora_grad_shapes_ffn(d, d_ff, r)))
        sizes = [(a * b + 3) // 4 * 4 for _, (a, b) in shapes]
        per = sum(sizes)
        self.gflat = torch.zeros(nl * per, device="cuda")
        self.grads = []
        for l in range(nl):
            g, o = {}, l * per
            for (key, (a, b)), sz in zip(shapes, sizes):
                g[key] = self.gflat[o:o + a * b].view(a, b)
                o += sz
            self.grads.append(g)

        calls, bwd = [], []
        self.idx_qk, self.idx_ffn, self.k_ffn, self.kh = [], [], [], []
        self._structs = []
        for l, w in enumerate(layers):
            S_ = sv[l]
            G = self.grads[l]
            # -- input normalisation (the first layer reads X; later ones add
            # the previous FFN output to the previous residual)
            if l == 0:
                calls.append(_Call("slora_rmsnorm_fwd", [L.BF16, T, d, L.c_f32(eps), L.ptr(X),
                                                         None, L.ptr(w["g1"]), None,
                                                         L.ptr(S_["n1"]), L.ptr(S_["r1"])]))
            else:
                calls.append(_Call("slora_rmsnorm_fwd",
                                   [L.BF16, T, d, L.c_f32(eps), L.ptr(sv[l - 1]["h"]),
                                    L.ptr(f_out), L.ptr(w["g1"]), L.ptr(self.x[l]),
                                    L.ptr(S_["n1"]), L.ptr(S_["r1"])]))
            n1 = S_["n1"]
            # -- q/k channel selection
            sq = float(qk_sparsity[l])
            if sq > 0.0:
                idx = torch.empty(nq + nkv, dtype=torch.int32, device="cuda")
                k_out = L.c_i32(0)
                scores = f32(KV * hd)
                c = _Call("slora_estimate_select",
                          [L.CRIT_QK, L.ptr(n1), L.BF16, ctypes.byref(tok), d, L.ptr(w["Lq"]),
                           L.ptr(w["Uq"]), nq, L.ptr(w["Lk"]), L.ptr(w["Uk"]), nkv, r_svd, H, KV,
                           hd, sq, L.ptr(idx), ctypes.byref(k_out), L.ptr(scores)],
                          (k_out, idx, scores))
                c.need()
                kh = int(k_out.value)
                calls.append(c)
                iq, ik = idx[:H * kh], idx[H * kh:H * kh + KV * kh]
            else:
                idx, kh, iq, ik = None, hd, None, None
            self.idx_qk.append(idx)
            self.kh.append(kh)
            # -- q, k, v, o linears and the attention core
            proj = {}
            for nm, n, ii in (("q", nq, iq), ("k", nkv, ik)):
                base = [L.BF16, ctypes.byref(tok), d, n, L.ptr(w["W" + nm]), L.ptr(w["A" + nm]),
                        L.ptr(w["B" + nm]), r, s]
                XA = S_["XA" + nm]
                R = S_["Qr" if nm == "q" else "Kr"]
                dR = dQr if nm == "q" else dKr
                dXn = dxq if nm == "q" else dxk
                if ii is not None:
                    ni = ii.numel()
                    Yc, Yo, dYc, dYo = bf(TC, ni), bf(TO, n), bf(TC, ni), bf(TO, n)
                    self._keep += [Yc, Yo, dYc, dYo]
                    fwd = _Call("slora_linear_fwd", base + [L.SLICE_OUT_ROWS, L.ptr(ii), ni,
                                                            L.ptr(n1), None, L.ptr(Yc),
                                                            L.ptr(Yo), L.ptr(XA)])
                    rope = _Call("slora_rope_pack", [L.BF16, ctypes.byref(tok), n, hd,
                                                     float(rope_base), L.ptr(ii), ni, None,
                                                     L.ptr(Yc), L.ptr(Yo), L.ptr(R)])
                    unrope = _Call("slora_rope_unpack", [L.BF16, ctypes.byref(tok), n, hd,
                                                         float(rope_base), L.ptr(ii), ni,
                                                         L.ptr(dR), None, L.ptr(dYc),
                                                         L.ptr(dYo)])
                    back = _Call("slora_linear_bwd", base + [L.SLICE_OUT_ROWS, L.ptr(ii), ni,
                                                             L.ptr(n1), None, L.ptr(XA),
                                                             L.ptr(dYc), L.ptr(dYo), L.ptr(dXn),
                                                             None, L.ptr(G["dA" + nm]),
                                                             L.ptr(G["dB" + nm])])
                else:
                    Y, dYd = bf(T, n), bf(T, n)
                    self._keep += [Y, dYd]
                    fwd = _Call("slora_linear_fwd", base + [L.SLICE_NONE, None, 0, L.ptr(n1),
                                                            None, L.ptr(Y), None, L.ptr(XA)])
                    rope = _Call("slora_rope_pack", [L.BF16, ctypes.byref(tok), n, hd,
                                                     float(rope_base), None, 0, L.ptr(Y), None,
                                                     None, L.ptr(R)])
                    unrope = _Call("slora_rope_unpack", [L.BF16, ctypes.byref(tok), n, hd,
                                                         float(rope_base), None, 0, L.ptr(dR),
                                                         L.ptr(dYd), None, None])
                    back = _Call("slora_linear_bwd", base + [L.SLICE_NONE, None, 0, L.ptr(n1),
                                                             None, L.ptr(XA), L.ptr(dYd), None,
                                                             L.ptr(dXn), None,
                                                             L.ptr(G["dA" + nm]),
                                                             L.ptr(G["dB" + nm])])
                proj[nm] = (fwd, rope, unrope, back)
            vbase = [L.BF16, ctypes.byref(tok), d, nkv, L.ptr(w["Wv"]), L.ptr(w["Av"]),
                     L.ptr(w["Bv"]), r, s, L.SLICE_NONE, None, 0]
            v_f = _Call("slora_linear_fwd", vbase + [L.ptr(n1), None, L.ptr(S_["V"]), None,
                                                     L.ptr(S_["XAv"])])
            v_b = _Call("slora_linear_bwd", vbase + [L.ptr(n1), None, L.ptr(S_["XAv"]),
                                                     L.ptr(dV), None, L.ptr(dxv), None,
                                                     L.ptr(G["dAv"]), L.ptr(G["dBv"])])
            att_f = _Call("slora_attention_fwd", [L.BF16, ctypes.byref(tok), H, KV, hd,
                                                  L.ptr(S_["Qr"]), L.ptr(S_["Kr"]),
                                                  L.ptr(S_["V"]), L.ptr(S_["O"]),
                                                  L.ptr(S_["lse"])])
            att_b = _Call("slora_attention_bwd", [L.BF16, ctypes.byref(tok), H, KV, hd,
                                                  L.ptr(S_["Qr"]), L.ptr(S_["Kr"]),
                                                  L.ptr(S_["V"]), L.ptr(S_["O"]),
                                                  L.ptr(S_["lse"]), L.ptr(dO_att), L.ptr(dQr),
                                                  L.ptr(dKr), L.ptr(dV)])
            obase = [L.BF16, ctypes.byref(tok), nq, d, L.ptr(w["Wo"]), L.ptr(w["Ao"]),
                     L.ptr(w["Bo"]), r, s, L.SLICE_NONE, None, 0]
            o_f = _Call("slora_linear_fwd", obase + [L.ptr(S_["O"]), None, L.ptr(a_out), None,
                                                     L.ptr(S_["XAo"])])
            o_b = _Call("slora_linear_bwd", obase + [L.ptr(S_["O"]), None, L.ptr(S_["XAo"]),
                                                     L.ptr(dh), None, L.ptr(dO_att), None,
                                                     L.ptr(G["dAo"]), L.ptr(G["dBo"])])
            # q, k and v (with the rotary packing of q and k) run at once
            calls += [_Par([proj["q"][0], proj["q"][1]], [proj["k"][0], proj["k"][1]], [v_f]),
                      att_f, o_f]
            # -- residual + second normalisation, FFN forward (its own selection)
            calls.append(_Call("slora_rmsnorm_fwd", [L.BF16, T, d, L.c_f32(eps),
                                                     L.ptr(self.x[l]), L.ptr(a_out),
                                                     L.ptr(w["g2"]), L.ptr(S_["h"]),
                                                     L.ptr(S_["n2"]), L.ptr(S_["r2"])]))
            sf = float(ffn_sparsity[l])
            fidx = torch.empty(d_ff, dtype=torch.int32, device="cuda")
            force = torch.arange(d_ff, dtype=torch.int32, device="cuda") if sf == 0.0 else None
            lay = L.ffn_layer_struct(d, d_ff, r_svd, r, s, w["Wg"], w["Wu"], w["Wd_t"], w["Ag"],
                                     w["Bg"], w["Au"], w["Bu"], w["Ad"], w["Bd"], w["Lg"],
                                     w["Ug"], w["Lu"], w["Uu"])
            fgs = L.ffn_grads_struct(G["dAg"], G["dBg"], G["dAu"], G["dBu"], G["dAd"], G["dBd"])
            fa, fk = L.ffn_args(L.BF16, lay, batch, seq, ctx_len, sf, S_["n2"], None, f_out, None,
                                None, fidx, force)
            ffn_f = _Call("slora_ffn_fwd_bwd", fa, fk + (lay, force))
            # the layer's FFN workspace keeps its forward state for the backward
            ffn_ws = torch.empty(max(ffn_f.need(), 16), dtype=torch.uint8, device="cuda")
            ffn_f.own_ws = ffn_ws
            kf = int(fk[2].value)
            self.idx_ffn.append(fidx)
            self.k_ffn.append(kf)
            calls.append(ffn_f)
            # backward of this layer (issued in reverse layer order below)
            self._structs += [lay, fgs]
            bwd.append(dict(fgs=fgs, lay=lay, fidx=fidx, kf=kf, sf=sf, force=force, ws=ffn_ws,
                            q=proj["q"], k=proj["k"], v_b=v_b, att_b=att_b, o_b=o_b, w=w, S=S_))
        # -- the stack output: last residual + last FFN output
        calls.append(_Call("slora_rmsnorm_fwd", [L.BF16, T, d, L.c_f32(eps),
                                                 L.ptr(sv[-1]["h"]), L.ptr(f_out),
                                                 L.ptr(layers[-1]["g2"]), L.ptr(self.y), None,
                                                 None]))
        # ---- backward, last layer first
        dx_cur = dY
        for l in range(nl - 1, -1, -1):
            B = bwd[l]
            S_, w = B["S"], B["w"]
            dx_next = dx_pp[(nl - 1 - l) % 2]
            # the FFN backward resumes from the state its forward left in the
            # layer's workspace (same arguments as the forward call)
            fa, fk = L.ffn_args(L.BF16, B["lay"], batch, seq, ctx_len, B["sf"], S_["n2"], dx_cur,
                                f_out, dn2, B["fgs"], B["fidx"], B["force"])
            calls.append(_Call("slora_ffn_bwd", fa, fk + (B["force"],), own_ws=B["ws"]))
            calls.append(_Call("slora_rmsnorm_bwd", [L.BF16, T, d, L.ptr(S_["h"]),
                                                     L.ptr(S_["r2"]), L.ptr(w["g2"]), L.ptr(dn2),
                                                     None, None, L.ptr(dx_cur), L.ptr(dh)]))
            calls += [B["o_b"], B["att_b"],
                      _Par([B["q"][2], B["q"][3]], [B["k"][2], B["k"][3]], [B["v_b"]])]
            calls.append(_Call("slora_rmsnorm_bwd", [L.BF16, T, d, L.ptr(self.x[l]),
                                                     L.ptr(S_["r1"]), L.ptr(w["g1"]), L.ptr(dxq),
                                                     L.ptr(dxk), L.ptr(dxv), L.ptr(dh),
                                                     L.ptr(dx_next)]))
            dx_cur = dx_next
        self.dX = dx_cur
        self.calls = calls
        self._setup_branches()

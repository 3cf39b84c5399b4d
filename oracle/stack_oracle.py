"""Float64 NumPy oracle for the full decoder-layer step around the sparse LoRA
linears: rotary embedding, causal softmax attention, RMS normalisation and
the residual stream of a Llama-shaped layer stack.

Test infrastructure only, like ``slora_oracle`` (imported by the tests,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``; it
shares no code with the CUDA path).

What the pages fix, and the readings taken where they are silent:
  * SparseLoRA article, section 1: q/k channels are chosen per head by the
    query-key product; section 3: context tokens run sparse, output tokens
    dense, with a per-layer ratio.  A skipped q/k channel of a context row is
    simply not computed, so the attention core sees a zero there.
  * The pages name Llama models but do not restate their layer.  The plainest
    reading of "Llama-shaped" is taken: pre-normalised residual blocks
    x -> x + attn(rms(x)) -> h + ffn(rms(h)), RMS normalisation with a frozen
    per-channel gain (eps 1e-5), rotate-half rotary embedding with base 10000
    on positions counted from the start of each sequence, causal softmax
    attention within each sequence with scale 1/sqrt(head_dim), grouped
    key/value heads (query head h reads key/value head h // (H / KV)).
  * Skipped q/k channels are zero before the rotation (the rotation then
    mixes a kept channel into its rotate-half partner, as it would on the
    dense path with that channel's weight row zeroed).
All arrays are float64 and follow the conventions of ``slora_oracle``.
"""
from __future__ import annotations

import numpy as np

from . import slora_oracle as so

__all__ = [
    "rope_angles", "rope_apply", "rope_apply_t", "attention_fwd", "attention_bwd",
    "rmsnorm_fwd", "rmsnorm_bwd", "assemble_qk", "split_qk",
    "layer_fwd", "layer_bwd", "stack_fwd_bwd", "RMS_EPS", "ROPE_BASE",
]

RMS_EPS = 1e-5
ROPE_BASE = 10000.0


# ---------------------------------------------------------------------------
# rotary position embedding, rotate-half pairing (channel i with i + hd/2)
# ---------------------------------------------------------------------------
def rope_angles(seq: int, head_dim: int, base: float = ROPE_BASE) -> np.ndarray:
    """Angle p * base^(-2i/hd) of position p and pair i: (seq, hd/2)."""
    half = head_dim // 2
    inv = base ** (-2.0 * np.arange(half) / head_dim)
    return np.arange(seq, dtype=np.float64)[:, None] * inv[None, :]


def rope_apply(Y: np.ndarray, batch: int, seq: int, head_dim: int, base: float = ROPE_BASE,
               sign: float = 1.0) -> np.ndarray:
    """Rotate each head's pairs (i, i + hd/2) of every row by its position's
    angle (rows in (sequence, position) order).  ``sign=-1`` rotates back."""
    T, n = Y.shape
    half = head_dim // 2
    ang = sign * rope_angles(seq, head_dim, base)              # (seq, half)
    c = np.tile(np.cos(ang), (batch, 1))[:, None, :]           # (T, 1, half)
    s = np.tile(np.sin(ang), (batch, 1))[:, None, :]
    Z = Y.reshape(T, n // head_dim, head_dim)
    a, b = Z[:, :, :half], Z[:, :, half:]
    out = np.concatenate([a * c - b * s, b * c + a * s], axis=2)
    return out.reshape(T, n)


def rope_apply_t(G: np.ndarray, batch: int, seq: int, head_dim: int,
                 base: float = ROPE_BASE) -> np.ndarray:
    """Transpose of ``rope_apply`` (a rotation: its inverse), for gradients."""
    return rope_apply(G, batch, seq, head_dim, base, sign=-1.0)


def assemble_qk(Y_ctx, Y_out, batch, seq, ctx_len, n, idx) -> np.ndarray:
    """Full-width q or k rows (T x n): context rows carry the computed channels
    idx and zeros elsewhere, output rows are dense."""
    C, O = so.context_rows(batch, seq, ctx_len)
    Y = np.zeros((batch * seq, n))
    Y[np.ix_(C, idx)] = Y_ctx
    Y[O] = Y_out
    return Y


def split_qk(G, batch, seq, ctx_len, idx):
    """Gradient of ``assemble_qk``: (dY_ctx on channels idx, dY_out dense)."""
    C, O = so.context_rows(batch, seq, ctx_len)
    return G[np.ix_(C, idx)], G[O]


# ---------------------------------------------------------------------------
# causal softmax attention within each sequence, grouped key/value heads
# ---------------------------------------------------------------------------
def _heads(Y, batch, seq, nh, hd):
    return Y.reshape(batch, seq, nh, hd).transpose(0, 2, 1, 3)   # (b, h, s, hd)


def _unheads(Z):
    b, h, s, hd = Z.shape
    return Z.transpose(0, 2, 1, 3).reshape(b * s, h * hd)


def attention_fwd(Q, K, V, batch, seq, heads, kv_heads, head_dim):
    """O = softmax(Q K^T / sqrt(hd) + causal mask) V per sequence and head.
    Q: T x (H hd), K, V: T x (KV hd).  Returns O (T x H hd) and the row
    log-sum-exp of the scaled scores, lse (batch, H, seq)."""
    grp = heads // kv_heads
    q = _heads(Q, batch, seq, heads, head_dim)
    k = np.repeat(_heads(K, batch, seq, kv_heads, head_dim), grp, axis=1)
    v = np.repeat(_heads(V, batch, seq, kv_heads, head_dim), grp, axis=1)
    S = (q @ k.transpose(0, 1, 3, 2)) / np.sqrt(head_dim)
    mask = np.tril(np.ones((seq, seq), dtype=bool))
    S = np.where(mask, S, -np.inf)
    m = S.max(axis=-1, keepdims=True)
    E = np.exp(S - m)
    z = E.sum(axis=-1, keepdims=True)
    P = E / z
    lse = (m + np.log(z))[..., 0]
    return _unheads(P @ v), lse


def attention_bwd(Q, K, V, O, lse, dO, batch, seq, heads, kv_heads, head_dim):
    """Gradients (dQ, dK, dV) of ``attention_fwd`` for the upstream dO:
    dV = P^T dO, dP = dO V^T, dS = P (dP - rowsum(dO * O)), dQ = dS K / sqrt(hd),
    dK = dS^T Q / sqrt(hd); key/value head gradients sum over their group."""
    grp = heads // kv_heads
    sc = 1.0 / np.sqrt(head_dim)
    q = _heads(Q, batch, seq, heads, head_dim)
    k = np.repeat(_heads(K, batch, seq, kv_heads, head_dim), grp, axis=1)
    v = np.repeat(_heads(V, batch, seq, kv_heads, head_dim), grp, axis=1)
    o = _heads(O, batch, seq, heads, head_dim)
    do = _heads(dO, batch, seq, heads, head_dim)
    S = (q @ k.transpose(0, 1, 3, 2)) * sc
    mask = np.tril(np.ones((seq, seq), dtype=bool))
    P = np.where(mask, np.exp(S - lse[..., None]), 0.0)
    dv = P.transpose(0, 1, 3, 2) @ do
    dP = do @ v.transpose(0, 1, 3, 2)
    D = (do * o).sum(axis=-1, keepdims=True)
    dS = P * (dP - D)
    dq = (dS @ k) * sc
    dk = (dS.transpose(0, 1, 3, 2) @ q) * sc
    b = dq.shape[0]
    dk = dk.reshape(b, kv_heads, grp, seq, head_dim).sum(axis=2)
    dv = dv.reshape(b, kv_heads, grp, seq, head_dim).sum(axis=2)
    return _unheads(dq), _unheads(dk), _unheads(dv)


# ---------------------------------------------------------------------------
# RMS normalisation with a frozen gain
# ---------------------------------------------------------------------------
def rmsnorm_fwd(X, g, eps: float = RMS_EPS):
    """N = X / rms(X) * g per row, rms = sqrt(mean(X^2) + eps); returns (N, rstd)."""
    rstd = 1.0 / np.sqrt((X * X).mean(axis=1) + eps)
    return X * rstd[:, None] * g[None, :], rstd


def rmsnorm_bwd(X, g, rstd, dN):
    """dX of ``rmsnorm_fwd`` (g frozen): rstd (g dN) - X rstd^3 mean(X g dN)."""
    gd = dN * g[None, :]
    m = (X * gd).mean(axis=1)
    return rstd[:, None] * gd - X * (rstd ** 3 * m)[:, None]


# ---------------------------------------------------------------------------
# one decoder layer: attention block (sparse q/k, dense v/o) + SwiGLU FFN
# ---------------------------------------------------------------------------
def layer_fwd(x, lay: dict, batch, seq, ctx_len, heads, kv_heads, head_dim,
              idx_q, idx_k, idx_ffn):
    """Forward of one layer on fixed channel sets.  ``lay`` holds g1, g2 (RMS
    gains), Wq/Aq/Bq, Wk/Ak/Bk, Wv/Av/Bv, Wo/Ao/Bo (W0 n x k, A r x k, B n x r),
    the FFN weights of ``slora_oracle.ffn_fwd`` and ``scale``.  idx_q / idx_k
    are the kept q / k channels of the context rows (None: dense).  Returns
    (y, saved)."""
    s = lay["scale"]
    nq, nkv = heads * head_dim, kv_heads * head_dim
    n1, r1 = rmsnorm_fwd(x, lay["g1"])
    proj = {}
    for nm, n, idx in (("q", nq, idx_q), ("k", nkv, idx_k)):
        W, A, B = lay["W" + nm], lay["A" + nm], lay["B" + nm]
        if idx is None:
            Y, _, XA = so.linear_fwd("none", n1, None, batch, seq, ctx_len, W, A, B, s, None)
        else:
            Yc, Yo, XA = so.linear_fwd("out_rows", n1, None, batch, seq, ctx_len, W, A, B, s,
                                       idx)
            Y = assemble_qk(Yc, Yo, batch, seq, ctx_len, n, idx)
        proj[nm] = (rope_apply(Y, batch, seq, head_dim), XA)
    V, _, XAv = so.linear_fwd("none", n1, None, batch, seq, ctx_len, lay["Wv"], lay["Av"],
                              lay["Bv"], s, None)
    Qr, Kr = proj["q"][0], proj["k"][0]
    O, lse = attention_fwd(Qr, Kr, V, batch, seq, heads, kv_heads, head_dim)
    a, _, XAo = so.linear_fwd("none", O, None, batch, seq, ctx_len, lay["Wo"], lay["Ao"],
                              lay["Bo"], s, None)
    h = x + a
    n2, r2 = rmsnorm_fwd(h, lay["g2"])
    f, fsaved = so.ffn_fwd(n2, batch, seq, ctx_len, lay, idx_ffn)
    saved = dict(x=x, n1=n1, r1=r1, Qr=Qr, Kr=Kr, V=V, O=O, lse=lse, XAq=proj["q"][1],
                 XAk=proj["k"][1], XAv=XAv, XAo=XAo, h=h, n2=n2, r2=r2, fsaved=fsaved)
    return h + f, saved


def layer_bwd(dy, lay: dict, saved: dict, batch, seq, ctx_len, heads, kv_heads, head_dim,
              idx_q, idx_k, idx_ffn):
    """Backward of ``layer_fwd`` (every frozen weight and gain fixed): returns
    dx and the LoRA gradients dA*/dB* of q, k, v, o and the FFN."""
    s = lay["scale"]
    fg = so.ffn_bwd(saved["n2"], dy, lay, idx_ffn, saved["fsaved"])
    dh = dy + rmsnorm_bwd(saved["h"], lay["g2"], saved["r2"], fg["dX"])
    dO, _, dAo, dBo = so.linear_bwd("none", saved["O"], None, saved["XAo"], dh, None, batch,
                                    seq, ctx_len, lay["Wo"], lay["Ao"], lay["Bo"], s, None)
    dQr, dKr, dV = attention_bwd(saved["Qr"], saved["Kr"], saved["V"], saved["O"],
                                 saved["lse"], dO, batch, seq, heads, kv_heads, head_dim)
    grads = dict(dAo=dAo, dBo=dBo)
    dn1 = np.zeros_like(saved["n1"])
    for nm, dR, idx in (("q", dQr, idx_q), ("k", dKr, idx_k)):
        W, A, B = lay["W" + nm], lay["A" + nm], lay["B" + nm]
        dY = rope_apply_t(dR, batch, seq, head_dim)
        if idx is None:
            dX, _, dA, dB = so.linear_bwd("none", saved["n1"], None, saved["XA" + nm], dY, None,
                                          batch, seq, ctx_len, W, A, B, s, None)
        else:
            dYc, dYo = split_qk(dY, batch, seq, ctx_len, idx)
            dX, _, dA, dB = so.linear_bwd("out_rows", saved["n1"], None, saved["XA" + nm], dYc,
                                          dYo, batch, seq, ctx_len, W, A, B, s, idx)
        dn1 += dX
        grads["dA" + nm], grads["dB" + nm] = dA, dB
    dX, _, dAv, dBv = so.linear_bwd("none", saved["n1"], None, saved["XAv"], dV, None, batch,
                                    seq, ctx_len, lay["Wv"], lay["Av"], lay["Bv"], s, None)
    dn1 += dX
    grads["dAv"], grads["dBv"] = dAv, dBv
    dx = dh + rmsnorm_bwd(saved["x"], lay["g1"], saved["r1"], dn1)
    for key in ("dAg", "dBg", "dAu", "dBu", "dAd", "dBd"):
        grads[key] = fg[key]
    return dx, grads


def stack_fwd_bwd(x, dY, layers: list, batch, seq, ctx_len, heads, kv_heads, head_dim,
                  qk_sparsity=None, ffn_sparsity=None, idx_force=None):
    """One training step of a layer stack: every layer's forward (each sparse
    layer estimating and selecting its q/k channels from its own normalised
    input and its FFN channels from the FFN's normalised input), then every
    backward in reverse order with the same channel sets.

    Per layer l, ``qk_sparsity[l]`` / ``ffn_sparsity[l]`` set the ratios (0: dense),
    or ``idx_force[l] = (idx_q, idx_k, idx_ffn)`` fixes the sets (None entries
    dense).  Returns dict(y, dx, grads[l], idx[l])."""
    L_ = len(layers)
    sets, saves = [], []
    for l, lay in enumerate(layers):
        d_ff = lay["Wg"].shape[0]
        if idx_force is not None:
            iq, ik, iff = idx_force[l]
            ffn_s = None
        else:
            n1, _ = rmsnorm_fwd(x, lay["g1"])
            iq = ik = iff = None
            if qk_sparsity[l] > 0:
                iq, ik, _, _ = so.estimate_select_qk(n1, batch, seq, ctx_len, lay["Lq"],
                                                     lay["Uq"], lay["Lk"], lay["Uk"], heads,
                                                     kv_heads, head_dim, qk_sparsity[l])
            ffn_s = ffn_sparsity[l]
        y, sv = _layer_fwd_select(x, lay, batch, seq, ctx_len, heads, kv_heads, head_dim, iq,
                                  ik, iff, ffn_s, d_ff)
        sets.append((iq, ik, sv["idx_ffn"]))
        saves.append(sv)
        x = y
    dx = dY
    grads = [None] * L_
    for l in range(L_ - 1, -1, -1):
        iq, ik, iff = sets[l]
        dx, grads[l] = layer_bwd(dx, layers[l], saves[l], batch, seq, ctx_len, heads, kv_heads,
                                 head_dim, iq, ik, iff)
    return dict(y=x, dx=dx, grads=grads, idx=sets)


def _layer_fwd_select(x, lay, batch, seq, ctx_len, heads, kv_heads, head_dim, iq, ik, iff,
                      ffn_s, d_ff):
    """``layer_fwd`` with the FFN channel set chosen from the FFN input when
    ``iff`` is None and ``ffn_s`` is a ratio (0 or None: every channel)."""
    if iff is None and ffn_s:
        # forward up to the FFN input, select, then run the layer on the set
        y0, sv0 = layer_fwd(x, lay, batch, seq, ctx_len, heads, kv_heads, head_dim, iq, ik,
                            np.arange(d_ff))
        iff, _, _ = so.estimate_select_ffn(sv0["n2"], batch, seq, ctx_len, lay["Lg"],
                                           lay["Ug"], lay["Lu"], lay["Uu"], ffn_s)
    elif iff is None:
        iff = np.arange(d_ff)
    y, sv = layer_fwd(x, lay, batch, seq, ctx_len, heads, kv_heads, head_dim, iq, ik, iff)
    sv["idx_ffn"] = np.asarray(iff, dtype=np.int64)
    return y, sv

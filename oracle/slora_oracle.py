"""Float64 NumPy oracle for SparseLoRA's contextually sparse LoRA linear layers.

Test infrastructure only (see the package docstring).  Sources are the two
SparseLoRA pages: the long-form article on the method (ICML 2025,
arXiv 2506.16500) with its sections 1 "dynamic sparsity", 2 "SVD sparsity
estimator", 3 "layer sensitivity" (context/output token split) and 6-7
(structured slices, rank 8), and the forum post carrying the paper's abstract
("select sparse weight subsets for loss and gradient computation").  The pages
give the method in prose only; where they are silent the plainest reading is
taken and named at the function that uses it.

Conventions (PyTorch ``nn.Linear`` / PEFT layout):
  * frozen weight W0 is n x k (out x in), y = x W0^T;
  * LoRA A is r x k, B is n x r, the LoRA output is s * (x A^T) B^T;
  * truncated SVD W0 ~= U_r diag(sigma_r) V_r^T, stored as L = V_r diag(sigma_r)
    (k x r) and U = U_r (n x r), so the low-rank estimate of x W0^T is x L U^T;
  * tokens: ``batch`` sequences of ``seq`` rows; in sequence b the first
    ctx_len[b] rows are context tokens (sparse path), the rest are output
    tokens (dense path).  Compact context/output matrices list those rows in
    (b, position) order.
All arrays are float64; inputs that the device holds in bf16 are rounded to
bf16 by the caller before they reach the oracle.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "context_rows", "silu", "silu_grad", "svd_prepare", "project",
    "ffn_scores", "ffn_gram_scores", "qk_scores", "qk_pair_scores", "l2_scores",
    "keep_count", "topk_select", "select_per_group",
    "estimate_select_ffn", "estimate_select_qk", "estimate_select_ffn_gram",
    "estimate_select_qk_pairs", "estimate_select_l2",
    "linear_fwd", "linear_bwd", "ffn_fwd", "ffn_bwd", "ffn_fwd_bwd",
    "ffn_fwd_bwd_per_seq", "ffn_fwd_down_only",
]


# ---------------------------------------------------------------------------
# token split (article section 3: context tokens sparse, output tokens dense)
# ---------------------------------------------------------------------------
def context_rows(batch: int, seq: int, ctx_len) -> tuple[np.ndarray, np.ndarray]:
    """Row indices (into the batch*seq row layout) of the context tokens and of
    the output tokens, each in (sequence, position) order."""
    ctx, out = [], []
    for b in range(batch):
        c = int(ctx_len[b])
        for i in range(seq):
            (ctx if i < c else out).append(b * seq + i)
    return np.asarray(ctx, dtype=np.int64), np.asarray(out, dtype=np.int64)


def silu(x: np.ndarray) -> np.ndarray:
    """SwiGLU gate nonlinearity x * sigmoid(x)."""
    return x / (1.0 + np.exp(-x))


def silu_grad(x: np.ndarray) -> np.ndarray:
    """d/dx [x sigmoid(x)] = sigmoid(x) (1 + x (1 - sigmoid(x)))."""
    sg = 1.0 / (1.0 + np.exp(-x))
    return sg * (1.0 + x * (1.0 - sg))


# ---------------------------------------------------------------------------
# estimator (article section 2): offline SVD once, online low-rank projection
# ---------------------------------------------------------------------------
def svd_prepare(W: np.ndarray, rank: int) -> tuple[np.ndarray, np.ndarray]:
    """Offline truncated SVD of a frozen weight, done once before training.

    Keeps the ``rank`` leading singular triplets and returns
    L = V_r diag(sigma_r) (k x rank) and U = U_r (n x rank).  Signs of the
    singular vectors are arbitrary; only products such as L U^T are unique.
    """
    u, sv, vt = np.linalg.svd(W, full_matrices=False)
    L = vt[:rank, :].T * sv[None, :rank]
    return L, u[:, :rank].copy()


def project(X_ctx: np.ndarray, L: np.ndarray) -> np.ndarray:
    """Online low-rank step: P = X_C L (T_C x r)."""
    return X_ctx @ L


def ffn_scores(P_g, P_u, U_g, U_u) -> np.ndarray:
    """SwiGLU FFN channel score (article section 1, "L2 norm = activity level").

    Reading: the score of intermediate channel j is the L2 norm, over the
    context tokens, of the estimated SwiGLU activation silu(g_hat) * u_hat,
    with g_hat = P_g U_g^T and u_hat = P_u U_u^T.
    """
    G = P_g @ U_g.T
    Uh = P_u @ U_u.T
    act = silu(G) * Uh
    return np.sqrt(np.sum(act * act, axis=0))


def ffn_gram_scores(P_g, P_u, U_g, U_u) -> np.ndarray:
    """Gram-computable FFN channel score, an estimator variant (reading of the
    article's sections 1-2: a cheaper stand-in for the activation norm).

    Score of channel j: ||g_hat[:, j]|| * ||u_hat[:, j]|| over the context
    tokens, g_hat = P_g U_g^T, u_hat = P_u U_u^T.  Each factor is a quadratic
    form of an r x r Gram matrix (||g_hat[:, j]||^2 = U_g[j] (P_g^T P_g) U_g[j]^T),
    so no per-(token, channel) silu is needed; it bounds the activation-norm
    score from above, since |silu(x)| <= |x| and ||a * b|| <= ||a|| ||b||.
    """
    G = P_g @ U_g.T
    Uh = P_u @ U_u.T
    return np.sqrt(np.sum(G * G, axis=0)) * np.sqrt(np.sum(Uh * Uh, axis=0))


def qk_scores(P_q, P_k, U_q, U_k, heads: int, kv_heads: int, head_dim: int) -> np.ndarray:
    """QK-norm channel score (article section 1, query/key product criterion).

    Reading: channel c of attention group g scores ||K_hat[:, g, c]|| times the
    sum over the group's query heads h of ||Q_hat[:, h, c]||, norms taken over
    context tokens.  With one query head per group (MHA) this is
    ||Q_hat_c|| * ||K_hat_c||, the Cauchy-Schwarz bound on channel c's share of
    the query-key products.  Returns a (kv_heads, head_dim) array.
    """
    Qh = P_q @ U_q.T
    Kh = P_k @ U_k.T
    nq = np.sqrt(np.sum(Qh * Qh, axis=0)).reshape(heads, head_dim)
    nk = np.sqrt(np.sum(Kh * Kh, axis=0)).reshape(kv_heads, head_dim)
    group = heads // kv_heads
    out = np.zeros((kv_heads, head_dim))
    for g in range(kv_heads):
        qsum = np.zeros(head_dim)
        for h in range(g * group, (g + 1) * group):
            qsum = qsum + nq[h]
        out[g] = nk[g] * qsum
    return out


def qk_pair_scores(P_q, P_k, U_q, U_k, heads: int, kv_heads: int, head_dim: int) -> np.ndarray:
    """QK-norm over rotate-half channel pairs, an estimator variant (reading of
    the article's section 1 criterion for models with rotary embeddings).

    Rotary position embedding turns channels c and c + head_dim/2 of a head
    together by a token-dependent angle, so a pair is kept or dropped as one
    unit.  The pair's norm over the context tokens is taken over both of its
    channels, sqrt(||Y_hat[:, c]||^2 + ||Y_hat[:, c + half]||^2), which the
    rotation leaves unchanged; pair p of group g scores ||K_hat_{g,p}|| times
    the sum over the group's query heads of ||Q_hat_{h,p}||.  Returns a
    (kv_heads, head_dim // 2) array.
    """
    half = head_dim // 2
    Qh = P_q @ U_q.T
    Kh = P_k @ U_k.T
    sq = np.sum(Qh * Qh, axis=0).reshape(heads, head_dim)
    sk = np.sum(Kh * Kh, axis=0).reshape(kv_heads, head_dim)
    nq = np.sqrt(sq[:, :half] + sq[:, half:])
    nk = np.sqrt(sk[:, :half] + sk[:, half:])
    group = heads // kv_heads
    out = np.zeros((kv_heads, half))
    for g in range(kv_heads):
        qsum = np.zeros(half)
        for h in range(g * group, (g + 1) * group):
            qsum = qsum + nq[h]
        out[g] = nk[g] * qsum
    return out


def l2_scores(P, U, heads: int, head_dim: int) -> np.ndarray:
    """Per-channel L2 norm of one estimated projection over the context tokens,
    per head: a (heads, head_dim) array (reading for the value projection,
    whose output channels are the input channels of the output projection)."""
    Yh = P @ U.T
    return np.sqrt(np.sum(Yh * Yh, axis=0)).reshape(heads, head_dim)


# ---------------------------------------------------------------------------
# selection (article section 1: per-input choice of active channels)
# ---------------------------------------------------------------------------
def keep_count(N: int, sparsity: float) -> int:
    """Channels kept at a sparsity ratio: the skipped count floor(s N) rounds
    down (reading; the pages give no rounding rule), so at least (1-s) N stay."""
    return int(N - np.floor(np.float64(sparsity) * N + 1e-9))


def topk_select(score: np.ndarray, k: int) -> np.ndarray:
    """The k highest-scoring channels, equal scores broken toward the lower
    index (reading), returned in ascending index order."""
    order = np.lexsort((np.arange(score.size), -np.asarray(score, dtype=np.float64)))
    return np.sort(order[:k]).astype(np.int64)


def select_per_group(scores: np.ndarray, k: int) -> np.ndarray:
    """Row-wise top-k of a (groups, head_dim) score array -> (groups, k)."""
    return np.stack([topk_select(scores[g], k) for g in range(scores.shape[0])])


def estimate_select_ffn(X, batch, seq, ctx_len, L_g, U_g, L_u, U_u, sparsity):
    """Estimator + selection for a SwiGLU FFN: returns (idx, k_keep, scores).

    One channel set per layer per step, pooled over all context tokens of the
    batch (reading: keeps the slices structured)."""
    C, _ = context_rows(batch, seq, ctx_len)
    Xc = X[C]
    scores = ffn_scores(project(Xc, L_g), project(Xc, L_u), U_g, U_u)
    k = keep_count(scores.size, sparsity)
    return topk_select(scores, k), k, scores


def estimate_select_qk(X, batch, seq, ctx_len, L_q, U_q, L_k, U_k,
                       heads, kv_heads, head_dim, sparsity):
    """Estimator + per-group selection for q/k projections.

    Returns (idx_q, idx_k, k_h, scores): idx_q lists for every query head h its
    group's kept channels as h*head_dim + c, idx_k the same sets for the key
    heads as g*head_dim + c."""
    C, _ = context_rows(batch, seq, ctx_len)
    Xc = X[C]
    scores = qk_scores(project(Xc, L_q), project(Xc, L_k), U_q, U_k, heads, kv_heads, head_dim)
    k = keep_count(head_dim, sparsity)
    sel = select_per_group(scores, k)
    group = heads // kv_heads
    idx_q = np.concatenate([h * head_dim + sel[h // group] for h in range(heads)])
    idx_k = np.concatenate([g * head_dim + sel[g] for g in range(kv_heads)])
    return idx_q, idx_k, k, scores


def estimate_select_ffn_gram(X, batch, seq, ctx_len, L_g, U_g, L_u, U_u, sparsity):
    """Estimator + selection for a SwiGLU FFN with the Gram-computable score
    ``ffn_gram_scores`` in place of the activation norm: (idx, k_keep, scores)."""
    C, _ = context_rows(batch, seq, ctx_len)
    Xc = X[C]
    scores = ffn_gram_scores(project(Xc, L_g), project(Xc, L_u), U_g, U_u)
    k = keep_count(scores.size, sparsity)
    return topk_select(scores, k), k, scores


def estimate_select_qk_pairs(X, batch, seq, ctx_len, L_q, U_q, L_k, U_k,
                             heads, kv_heads, head_dim, sparsity):
    """Estimator + per-group selection of rotate-half pairs for q/k.

    k_p = keep_count(head_dim / 2, s) pairs are kept per group; each head keeps
    the 2 k_p channels of those pairs, listed as the pairs' first channels
    (ascending) followed by their partners c + head_dim/2.  Returns
    (idx_q, idx_k, 2 k_p, pair scores)."""
    C, _ = context_rows(batch, seq, ctx_len)
    Xc = X[C]
    half = head_dim // 2
    scores = qk_pair_scores(project(Xc, L_q), project(Xc, L_k), U_q, U_k, heads, kv_heads,
                            head_dim)
    kp = keep_count(half, sparsity)
    sel = select_per_group(scores, kp)
    chans = np.concatenate([sel, sel + half], axis=1)
    group = heads // kv_heads
    idx_q = np.concatenate([h * head_dim + chans[h // group] for h in range(heads)])
    idx_k = np.concatenate([g * head_dim + chans[g] for g in range(kv_heads)])
    return idx_q, idx_k, 2 * kp, scores


def estimate_select_l2(X, batch, seq, ctx_len, L, U, heads, kv_heads, head_dim, sparsity):
    """Estimator + per-head selection by the L2 norm of one projection's
    estimated output, for slicing the value projection on its output channels
    and the output projection on the matching input channels.

    The scored projection has kv_heads heads (U is kv_heads*head_dim x r);
    with grouped queries, value channel (g, c) feeds output-projection input
    channel (h, c) of every query head h of group g (reading: attention mixes
    tokens, not channels, so a dropped value channel empties the same channel
    of the attention output).  Returns (idx_o, idx_v, k_h, scores): idx_o lists
    for every query head h its group's kept channels as h*head_dim + c, idx_v
    the same sets for the kv heads as g*head_dim + c."""
    C, _ = context_rows(batch, seq, ctx_len)
    Xc = X[C]
    scores = l2_scores(project(Xc, L), U, kv_heads, head_dim)
    k = keep_count(head_dim, sparsity)
    sel = select_per_group(scores, k)
    group = heads // kv_heads
    idx_o = np.concatenate([h * head_dim + sel[h // group] for h in range(heads)])
    idx_v = np.concatenate([g * head_dim + sel[g] for g in range(kv_heads)])
    return idx_o, idx_v, k, scores


# ---------------------------------------------------------------------------
# sliced LoRA linear (article sections 1, 6, 7; abstract): only the selected
# channel slices of W0 and of the LoRA branch are computed for context rows,
# output rows take the dense path.
# ---------------------------------------------------------------------------
def linear_fwd(side: str, X_ctx, X_out, batch, seq, ctx_len, W0, A, B, scale, idx):
    """One LoRA linear, forward.

    side = "none":     X_ctx is the full T x k input, returns Y (T x n).
    side = "out_rows": output-channel slice (q/k, gate/up).  X_ctx is the full
                       T x k input; returns Y_ctx = context rows on channels idx
                       (T_C x |idx|) and Y_out = output rows, dense (T_O x n).
    side = "in_cols":  input-channel slice (down/o).  X_ctx is T_C x |idx|
                       (context rows, input channels idx), X_out is T_O x k;
                       returns Y (T x n) in the full row layout.
    Also returns XA (T x r): the LoRA down-projection actually used per row.
    """
    C, O = context_rows(batch, seq, ctx_len)
    T = batch * seq
    r = A.shape[0]
    n = W0.shape[0]
    XA = np.zeros((T, r))
    if side == "none":
        XA = X_ctx @ A.T
        return X_ctx @ W0.T + scale * (XA @ B.T), None, XA
    if side == "out_rows":
        Xc, Xo = X_ctx[C], X_ctx[O]
        XA[C] = Xc @ A.T
        XA[O] = Xo @ A.T
        Y_ctx = Xc @ W0[idx].T + scale * (XA[C] @ B[idx].T)
        Y_out = Xo @ W0.T + scale * (XA[O] @ B.T)
        return Y_ctx, Y_out, XA
    if side == "in_cols":
        XA[C] = X_ctx @ A[:, idx].T
        XA[O] = X_out @ A.T
        Y = np.zeros((T, n))
        Y[C] = X_ctx @ W0[:, idx].T + scale * (XA[C] @ B.T)
        Y[O] = X_out @ W0.T + scale * (XA[O] @ B.T)
        return Y, None, XA
    raise ValueError(side)


def linear_bwd(side: str, X_ctx, X_out, XA, dY_ctx, dY_out, batch, seq, ctx_len,
               W0, A, B, scale, idx):
    """Backward of ``linear_fwd`` with W0 frozen: returns (dX_ctx, dX_out, dA, dB).

    Layouts mirror the forward (dY like Y, dX like X).  Skipped channels of a
    context row have no output, so they send no gradient: rows of dB (out_rows)
    or columns of dA (in_cols) outside idx receive output-row terms only.
    """
    C, O = context_rows(batch, seq, ctx_len)
    T = batch * seq
    n, k = W0.shape
    r = A.shape[0]
    if side == "none":
        dYB = dY_ctx @ B
        dX = dY_ctx @ W0 + scale * (dYB @ A)
        dA = scale * (dYB.T @ X_ctx)
        dB = scale * (dY_ctx.T @ XA)
        return dX, None, dA, dB
    if side == "out_rows":
        Xc, Xo = X_ctx[C], X_ctx[O]
        dYB_c = dY_ctx @ B[idx]
        dYB_o = dY_out @ B
        dX = np.zeros((T, k))
        dX[C] = dY_ctx @ W0[idx] + scale * (dYB_c @ A)
        dX[O] = dY_out @ W0 + scale * (dYB_o @ A)
        dA = scale * (dYB_c.T @ Xc + dYB_o.T @ Xo)
        dB = scale * (dY_out.T @ XA[O])
        dB[idx] += scale * (dY_ctx.T @ XA[C])
        return dX, None, dA, dB
    if side == "in_cols":
        dYc, dYo = dY_ctx[C], dY_ctx[O]
        dYB_c = dYc @ B
        dYB_o = dYo @ B
        dX_ctx = dYc @ W0[:, idx] + scale * (dYB_c @ A[:, idx])
        dX_out = dYo @ W0 + scale * (dYB_o @ A)
        dA = scale * (dYB_o.T @ X_out)
        dA[:, idx] += scale * (dYB_c.T @ X_ctx)
        dB = scale * (dYc.T @ XA[C] + dYo.T @ XA[O])
        return dX_ctx, dX_out, dA, dB
    raise ValueError(side)


# ---------------------------------------------------------------------------
# SwiGLU FFN layer: gate/up sliced on output channels, down on input channels,
# one shared channel set S.
# ---------------------------------------------------------------------------
def ffn_fwd(X, batch, seq, ctx_len, lay: dict, idx):
    """Sparse SwiGLU FFN forward on channel set idx (context rows) and dense on
    output rows.  ``lay`` holds Wg, Wu (d_ff x d), Wd (d x d_ff), the LoRA
    pairs Ag/Bg, Au/Bu, Ad/Bd and ``scale``.  Returns (out, saved)."""
    s = lay["scale"]
    C, O = context_rows(batch, seq, ctx_len)
    Xc, Xo = X[C], X[O]
    Wg, Wu, Wd = lay["Wg"], lay["Wu"], lay["Wd"]
    Ag, Bg, Au, Bu, Ad, Bd = (lay[k] for k in ("Ag", "Bg", "Au", "Bu", "Ad", "Bd"))
    # context rows: channels idx only
    g_c = Xc @ Wg[idx].T + s * ((Xc @ Ag.T) @ Bg[idx].T)
    u_c = Xc @ Wu[idx].T + s * ((Xc @ Au.T) @ Bu[idx].T)
    h_c = silu(g_c) * u_c
    # output rows: all channels
    g_o = Xo @ Wg.T + s * ((Xo @ Ag.T) @ Bg.T)
    u_o = Xo @ Wu.T + s * ((Xo @ Au.T) @ Bu.T)
    h_o = silu(g_o) * u_o
    out = np.zeros((batch * seq, Wd.shape[0]))
    out[C] = h_c @ Wd[:, idx].T + s * ((h_c @ Ad[:, idx].T) @ Bd.T)
    out[O] = h_o @ Wd.T + s * ((h_o @ Ad.T) @ Bd.T)
    saved = dict(C=C, O=O, g_c=g_c, u_c=u_c, h_c=h_c, g_o=g_o, u_o=u_o, h_o=h_o)
    return out, saved


def ffn_bwd(X, dOut, lay: dict, idx, saved):
    """Backward of ``ffn_fwd`` (W0 frozen): returns dX and the six LoRA grads."""
    s = lay["scale"]
    C, O = saved["C"], saved["O"]
    Xc, Xo = X[C], X[O]
    Wg, Wu, Wd = lay["Wg"], lay["Wu"], lay["Wd"]
    Ag, Bg, Au, Bu, Ad, Bd = (lay[k] for k in ("Ag", "Bg", "Au", "Bu", "Ad", "Bd"))
    d, d_ff = Wd.shape
    r = Ag.shape[0]
    dOc, dOo = dOut[C], dOut[O]
    g_c, u_c, h_c = saved["g_c"], saved["u_c"], saved["h_c"]
    g_o, u_o, h_o = saved["g_o"], saved["u_o"], saved["h_o"]

    # down projection (input channels idx for context rows)
    dOB_c, dOB_o = dOc @ Bd, dOo @ Bd
    dh_c = dOc @ Wd[:, idx] + s * (dOB_c @ Ad[:, idx])
    dh_o = dOo @ Wd + s * (dOB_o @ Ad)
    dAd = s * (dOB_o.T @ h_o)
    dAd[:, idx] += s * (dOB_c.T @ h_c)
    dBd = s * (dOc.T @ (h_c @ Ad[:, idx].T) + dOo.T @ (h_o @ Ad.T))

    # SwiGLU backward
    dg_c, du_c = dh_c * u_c * silu_grad(g_c), dh_c * silu(g_c)
    dg_o, du_o = dh_o * u_o * silu_grad(g_o), dh_o * silu(g_o)

    # gate / up projections (output channels idx for context rows)
    dX = np.zeros_like(X)
    dGB_c, dUB_c = dg_c @ Bg[idx], du_c @ Bu[idx]
    dGB_o, dUB_o = dg_o @ Bg, du_o @ Bu
    dX[C] = dg_c @ Wg[idx] + du_c @ Wu[idx] + s * (dGB_c @ Ag) + s * (dUB_c @ Au)
    dX[O] = dg_o @ Wg + du_o @ Wu + s * (dGB_o @ Ag) + s * (dUB_o @ Au)
    dAg = s * (dGB_c.T @ Xc + dGB_o.T @ Xo)
    dAu = s * (dUB_c.T @ Xc + dUB_o.T @ Xo)
    dBg = s * (dg_o.T @ (Xo @ Ag.T))
    dBu = s * (du_o.T @ (Xo @ Au.T))
    dBg[idx] += s * (dg_c.T @ (Xc @ Ag.T))
    dBu[idx] += s * (du_c.T @ (Xc @ Au.T))
    return dict(dX=dX, dAg=dAg, dBg=dBg, dAu=dAu, dBu=dBu, dAd=dAd, dBd=dBd)


def ffn_fwd_bwd(X, dOut, batch, seq, ctx_len, lay: dict, sparsity: float, idx_force=None):
    """Whole hot path for one FFN layer: estimate, select, sliced fwd, sliced bwd.

    ``lay`` additionally holds the estimator factors Lg, Ug, Lu, Uu.  With
    ``idx_force`` the estimator is skipped and that channel set is used."""
    if idx_force is None:
        idx, k, scores = estimate_select_ffn(X, batch, seq, ctx_len, lay["Lg"], lay["Ug"],
                                             lay["Lu"], lay["Uu"], sparsity)
    else:
        idx, k, scores = np.asarray(idx_force, dtype=np.int64), len(idx_force), None
    out, saved = ffn_fwd(X, batch, seq, ctx_len, lay, idx)
    grads = ffn_bwd(X, dOut, lay, idx, saved)
    return dict(idx=idx, k=k, scores=scores, out=out, **grads)


# ---------------------------------------------------------------------------
# projection-set variants (article section 6: which projections run sparse;
# section 1: the channels are chosen per input)
# ---------------------------------------------------------------------------
def ffn_fwd_bwd_per_seq(X, dOut, batch, seq, ctx_len, lay: dict, sparsity: float,
                        idx_force=None):
    """One channel set per sequence instead of one per batch (reading of
    "per input"): each sequence is its own one-sequence batch for the estimate,
    the selection and the sliced computation; the LoRA gradients of the layer
    are the sums over sequences.  ``idx_force[b]`` fixes sequence b's set.
    Returns dict(idx=[per-sequence sets], k, out, dX, dAg, ...)."""
    T, d = X.shape
    out, dX = np.zeros_like(X), np.zeros_like(X)
    grads, sets, k = None, [], None
    for b in range(batch):
        rows = slice(b * seq, (b + 1) * seq)
        force = None if idx_force is None else idx_force[b]
        r = ffn_fwd_bwd(X[rows], dOut[rows], 1, seq, [ctx_len[b]], lay, sparsity, force)
        out[rows], dX[rows] = r["out"], r["dX"]
        sets.append(r["idx"])
        k = r["k"]
        g = {n: r[n] for n in ("dAg", "dBg", "dAu", "dBu", "dAd", "dBd")}
        grads = g if grads is None else {n: grads[n] + g[n] for n in g}
    return dict(idx=sets, k=k, out=out, dX=dX, **grads)


def ffn_fwd_down_only(X, batch, seq, ctx_len, lay: dict, idx):
    """The down-projection-only variant: gate and up computed on every channel
    for every row, the down projection of context rows reading only the
    channels idx (the others' activations dropped).  Returns out."""
    s = lay["scale"]
    C, _ = context_rows(batch, seq, ctx_len)
    g = X @ lay["Wg"].T + s * ((X @ lay["Ag"].T) @ lay["Bg"].T)
    u = X @ lay["Wu"].T + s * ((X @ lay["Au"].T) @ lay["Bu"].T)
    h = silu(g) * u
    keep = np.zeros(h.shape[1], dtype=bool)
    keep[np.asarray(idx, dtype=np.int64)] = True
    h[np.ix_(C, ~keep)] = 0.0
    return h @ lay["Wd"].T + s * ((h @ lay["Ad"].T) @ lay["Bd"].T)

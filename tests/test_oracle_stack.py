"""Pins of the layer-stack oracle (rotary embedding, causal attention, RMS
normalisation, the decoder layer and the stack step) to things other than
itself: hand-worked rotary values, invariants of the rotation and of softmax
attention, brute-force loops, PyTorch's own attention / normalisation and
autograd in float64 as independent formulations, and central finite
differences.  The last tests plant plausible mistakes and confirm the pins
catch them.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import slora_oracle as SO
from oracle import stack_oracle as S


def rng(seed):
    return np.random.default_rng(seed)


# ------------------------------------------------------------------ rotary
def test_rope_hand_worked_values():
    # hd = 4: pair 0 = channels (0, 2) at frequency 1, pair 1 = (1, 3) at 0.01
    seq = 101
    Y = np.zeros((seq, 4))
    Y[1] = [1.0, 0.0, 0.0, 0.0]      # position 1, angle 1 on pair 0
    Y[100] = [0.0, 1.0, 0.0, 0.0]    # position 100, angle 100 * 0.01 = 1 on pair 1
    Y[7] = [0.0, 0.0, 2.0, 0.0]      # second member of pair 0 at position 7
    R = S.rope_apply(Y, 1, seq, 4)
    c, s = math.cos(1.0), math.sin(1.0)
    np.testing.assert_allclose(R[1], [c, 0.0, s, 0.0], atol=1e-15)
    np.testing.assert_allclose(R[100], [0.0, c, 0.0, s], atol=1e-13)
    np.testing.assert_allclose(R[7], [-2 * math.sin(7.0), 0.0, 2 * math.cos(7.0), 0.0],
                               atol=1e-14)
    np.testing.assert_allclose(S.rope_angles(3, 4)[2], [2.0, 0.02], rtol=1e-15)


def test_rope_position_zero_identity_norm_and_inverse():
    b, seq, hd, nh = 2, 9, 8, 3
    Y = rng(1).normal(size=(b * seq, nh * hd))
    R = S.rope_apply(Y, b, seq, hd)
    np.testing.assert_allclose(R[0], Y[0], atol=1e-15)          # position 0
    np.testing.assert_allclose(R[seq], Y[seq], atol=1e-15)      # next sequence restarts
    half = hd // 2
    pn = lambda Z: (Z.reshape(-1, nh, hd)[:, :, :half] ** 2 +
                    Z.reshape(-1, nh, hd)[:, :, half:] ** 2)
    np.testing.assert_allclose(pn(R), pn(Y), rtol=1e-12)        # each pair keeps its norm
    np.testing.assert_allclose(S.rope_apply_t(R, b, seq, hd), Y, atol=1e-12)


def test_rope_scores_depend_on_relative_position_only():
    hd, seq = 16, 40
    q, k = rng(2).normal(size=hd), rng(3).normal(size=hd)
    Q = S.rope_apply(np.tile(q, (seq, 1)), 1, seq, hd)
    K = S.rope_apply(np.tile(k, (seq, 1)), 1, seq, hd)
    G = Q @ K.T
    for delta in (0, 3, 17):
        diag = np.array([G[p + delta, p] for p in range(seq - delta)])
        np.testing.assert_allclose(diag, diag[0], rtol=1e-10, atol=1e-12)
    assert abs(G[5, 2] - G[2, 5]) > 1e-6 or np.allclose(q, k)


# ------------------------------------------------------------- attention
def _torch_attention(Q, K, V, b, seq, H, KV, hd):
    q = torch.from_numpy(Q).reshape(b, seq, H, hd).transpose(1, 2)
    k = torch.from_numpy(K).reshape(b, seq, KV, hd).transpose(1, 2)
    v = torch.from_numpy(V).reshape(b, seq, KV, hd).transpose(1, 2)
    o = F.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=H != KV)
    return o.transpose(1, 2).reshape(b * seq, H * hd).numpy()


@pytest.mark.parametrize("H,KV", [(2, 2), (4, 2), (4, 1)])
def test_attention_matches_torch_sdpa_and_brute_force(H, KV):
    b, seq, hd = 2, 7, 8
    r = rng(10 + H + KV)
    Q, K, V = (r.normal(size=(b * seq, n * hd)) for n in (H, KV, KV))
    O, lse = S.attention_fwd(Q, K, V, b, seq, H, KV, hd)
    np.testing.assert_allclose(O, _torch_attention(Q, K, V, b, seq, H, KV, hd), rtol=1e-12,
                               atol=1e-13)
    grp = H // KV
    for bb in range(b):
        for h in range(H):
            g = h // grp
            for t in range(seq):
                row = bb * seq + t
                q = Q[row, h * hd:(h + 1) * hd]
                sc = [float(q @ K[bb * seq + j, g * hd:(g + 1) * hd]) / math.sqrt(hd)
                      for j in range(t + 1)]
                m = max(sc)
                w = [math.exp(x - m) for x in sc]
                z = sum(w)
                o = sum(w[j] / z * V[bb * seq + j, g * hd:(g + 1) * hd] for j in range(t + 1))
                np.testing.assert_allclose(O[row, h * hd:(h + 1) * hd], o, rtol=1e-12,
                                           atol=1e-13)
                assert abs(lse[bb, h, t] - (m + math.log(z))) < 1e-12


def test_attention_first_row_equal_keys_and_shift_invariance():
    b, seq, hd, H = 1, 6, 4, 1
    r = rng(20)
    Q, V = r.normal(size=(seq, hd)), r.normal(size=(seq, hd))
    K = np.tile(r.normal(size=hd), (seq, 1))      # every key equal: running mean of v
    O, _ = S.attention_fwd(Q, K, V, b, seq, H, H, hd)
    np.testing.assert_allclose(O[0], V[0], atol=1e-15)
    for t in range(seq):
        np.testing.assert_allclose(O[t], V[:t + 1].mean(axis=0), rtol=1e-12)
    K2 = r.normal(size=(seq, hd))
    O1, _ = S.attention_fwd(Q, K2, V, b, seq, H, H, hd)
    O2, _ = S.attention_fwd(Q, K2 + r.normal(size=hd), V, b, seq, H, H, hd)
    np.testing.assert_allclose(O1, O2, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("H,KV", [(2, 2), (4, 2)])
def test_attention_bwd_matches_autograd_and_finite_differences(H, KV):
    b, seq, hd = 2, 5, 4
    r = rng(30 + H)
    Q, K, V = (r.normal(size=(b * seq, n * hd)) for n in (H, KV, KV))
    dO = r.normal(size=(b * seq, H * hd))
    O, lse = S.attention_fwd(Q, K, V, b, seq, H, KV, hd)
    dQ, dK, dV = S.attention_bwd(Q, K, V, O, lse, dO, b, seq, H, KV, hd)
    tq, tk, tv = (torch.from_numpy(x.copy()).requires_grad_() for x in (Q, K, V))
    q = tq.reshape(b, seq, H, hd).transpose(1, 2)
    k = tk.reshape(b, seq, KV, hd).transpose(1, 2)
    v = tv.reshape(b, seq, KV, hd).transpose(1, 2)
    o = F.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=H != KV)
    (o.transpose(1, 2).reshape(b * seq, H * hd) * torch.from_numpy(dO)).sum().backward()
    for mine, ref in ((dQ, tq), (dK, tk), (dV, tv)):
        np.testing.assert_allclose(mine, ref.grad.numpy(), rtol=1e-10, atol=1e-12)
    # central differences on a few entries of each input
    f = lambda Q_, K_, V_: float((S.attention_fwd(Q_, K_, V_, b, seq, H, KV, hd)[0] * dO).sum())
    eps = 1e-6
    for which, X, G in ((0, Q, dQ), (1, K, dK), (2, V, dV)):
        for (i, j) in ((0, 0), (b * seq - 1, X.shape[1] - 1), (3, 2)):
            args_p = [Q.copy(), K.copy(), V.copy()]
            args_m = [Q.copy(), K.copy(), V.copy()]
            args_p[which][i, j] += eps
            args_m[which][i, j] -= eps
            fd = (f(*args_p) - f(*args_m)) / (2 * eps)
            assert abs(fd - G[i, j]) < 1e-7 * max(1.0, abs(fd))


# -------------------------------------------------------------- RMS norm
def test_rmsnorm_matches_torch_and_invariants():
    r = rng(40)
    X, g = r.normal(size=(6, 16)) * 3.0, r.normal(size=16)
    N, rstd = S.rmsnorm_fwd(X, g)
    ref = F.rms_norm(torch.from_numpy(X), (16,), torch.from_numpy(g), eps=S.RMS_EPS).numpy()
    np.testing.assert_allclose(N, ref, rtol=1e-12)
    N1, _ = S.rmsnorm_fwd(X, np.ones(16), eps=0.0)
    np.testing.assert_allclose((N1 ** 2).mean(axis=1), 1.0, rtol=1e-12)
    N2, _ = S.rmsnorm_fwd(5.0 * X, g, eps=0.0)
    N3, _ = S.rmsnorm_fwd(X, g, eps=0.0)
    np.testing.assert_allclose(N2, N3, rtol=1e-12)


def test_rmsnorm_bwd_autograd_and_finite_differences():
    r = rng(41)
    X, g, dN = r.normal(size=(5, 12)), r.normal(size=12), r.normal(size=(5, 12))
    _, rstd = S.rmsnorm_fwd(X, g)
    dX = S.rmsnorm_bwd(X, g, rstd, dN)
    tx = torch.from_numpy(X.copy()).requires_grad_()
    (F.rms_norm(tx, (12,), torch.from_numpy(g), eps=S.RMS_EPS) * torch.from_numpy(dN)).sum() \
        .backward()
    np.testing.assert_allclose(dX, tx.grad.numpy(), rtol=1e-10, atol=1e-12)
    eps = 1e-6
    for (i, j) in ((0, 0), (4, 11), (2, 5)):
        Xp, Xm = X.copy(), X.copy()
        Xp[i, j] += eps
        Xm[i, j] -= eps
        fd = ((S.rmsnorm_fwd(Xp, g)[0] - S.rmsnorm_fwd(Xm, g)[0]) * dN).sum() / (2 * eps)
        assert abs(fd - dX[i, j]) < 1e-7


# ------------------------------------------------- decoder layer and stack
def make_layers(nl, d, H, KV, hd, d_ff, r_l, r_svd, seed):
    r = rng(seed)
    layers = []
    for _ in range(nl):
        lay = dict(scale=0.5)
        for nm, n, k in (("q", H * hd, d), ("k", KV * hd, d), ("v", KV * hd, d),
                         ("o", d, H * hd), ("g", d_ff, d), ("u", d_ff, d), ("d", d, d_ff)):
            lay["W" + nm] = r.normal(size=(n, k)) / math.sqrt(k)
            lay["A" + nm] = r.normal(size=(r_l, k)) * 0.2
            lay["B" + nm] = r.normal(size=(n, r_l)) * 0.2
        lay["g1"], lay["g2"] = 1.0 + 0.1 * r.normal(size=d), 1.0 + 0.1 * r.normal(size=d)
        for nm in ("q", "k", "g", "u"):
            lay["L" + nm], lay["U" + nm] = SO.svd_prepare(lay["W" + nm], r_svd)
        layers.append(lay)
    return layers


def torch_stack(x, layers, b, seq, ctx_len, H, KV, hd, sets):
    """The same stack written directly in PyTorch (float64): masked dense
    projections instead of slices (a context row's skipped q/k or FFN channel
    is multiplied by zero), the library's own rotary-free attention and RMS
    normalisation, autograd for the gradients."""
    C, _ = SO.context_rows(b, seq, ctx_len)
    ctx = torch.zeros(b * seq, dtype=torch.bool)
    ctx[torch.from_numpy(C)] = True
    ang = torch.from_numpy(S.rope_angles(seq, hd)).repeat(b, 1)
    cos, sin = torch.cos(ang), torch.sin(ang)

    def rot(Y, nh):
        Z = Y.reshape(b * seq, nh, hd)
        a, c = Z[..., :hd // 2], Z[..., hd // 2:]
        return torch.cat([a * cos[:, None] - c * sin[:, None],
                          c * cos[:, None] + a * sin[:, None]], -1).reshape(b * seq, nh * hd)

    def lin(X, lay, nm):
        W, A, B = (lay[k + nm] for k in ("W", "A", "B"))
        return X @ W.T + lay["scale"] * (X @ A.T) @ B.T

    def mask(Y, idx):
        if idx is None:
            return Y
        keep = torch.zeros(Y.shape[1], dtype=torch.float64)
        keep[torch.from_numpy(np.asarray(idx))] = 1.0
        m = torch.where(ctx[:, None], keep[None, :], torch.ones_like(keep)[None, :])
        return Y * m

    for lay, (iq, ik, iff) in zip(layers, sets):
        n1 = F.rms_norm(x, (x.shape[1],), lay["g1"], eps=S.RMS_EPS)
        q = rot(mask(lin(n1, lay, "q"), iq), H)
        k = rot(mask(lin(n1, lay, "k"), ik), KV)
        v = lin(n1, lay, "v")
        o = F.scaled_dot_product_attention(
            q.reshape(b, seq, H, hd).transpose(1, 2), k.reshape(b, seq, KV, hd).transpose(1, 2),
            v.reshape(b, seq, KV, hd).transpose(1, 2), is_causal=True, enable_gqa=H != KV)
        h = x + lin(o.transpose(1, 2).reshape(b * seq, H * hd), lay, "o")
        n2 = F.rms_norm(h, (h.shape[1],), lay["g2"], eps=S.RMS_EPS)
        act = mask(F.silu(lin(n2, lay, "g")) * lin(n2, lay, "u"), iff)
        x = h + lin(act, lay, "d")
    return x


@pytest.mark.parametrize("H,KV", [(2, 2), (4, 2)])
def test_stack_matches_masked_dense_autograd(H, KV):
    b, seq, hd, d, d_ff, nl = 2, 8, 8, 24, 40, 2
    ctx_len = [6, 5]
    layers = make_layers(nl, d, H, KV, hd, d_ff, 3, 4, seed=50 + H)
    r = rng(60)
    x, dY = r.normal(size=(b * seq, d)), r.normal(size=(b * seq, d))
    res = S.stack_fwd_bwd(x, dY, layers, b, seq, ctx_len, H, KV, hd, qk_sparsity=[0.5, 0.25],
                          ffn_sparsity=[0.5, 0.0])
    iq0, ik0, iff0 = res["idx"][0]
    assert len(iq0) == H * hd // 2 and len(ik0) == KV * hd // 2 and len(iff0) == d_ff // 2
    assert len(res["idx"][1][2]) == d_ff
    tl = [{k: (torch.from_numpy(v.copy()).requires_grad_() if isinstance(v, np.ndarray) else v)
           for k, v in lay.items()} for lay in layers]
    tx = torch.from_numpy(x.copy()).requires_grad_()
    y = torch_stack(tx, tl, b, seq, ctx_len, H, KV, hd, res["idx"])
    np.testing.assert_allclose(res["y"], y.detach().numpy(), rtol=1e-10, atol=1e-11)
    (y * torch.from_numpy(dY)).sum().backward()
    np.testing.assert_allclose(res["dx"], tx.grad.numpy(), rtol=1e-9, atol=1e-10)
    for l in range(nl):
        for key, val in res["grads"][l].items():
            np.testing.assert_allclose(val, tl[l][key[1:]].grad.numpy(), rtol=1e-9, atol=1e-10,
                                       err_msg=f"layer {l} {key}")


def test_stack_bwd_finite_differences_on_fixed_sets():
    b, seq, hd, H, KV, d, d_ff = 1, 6, 4, 2, 1, 8, 12
    ctx_len = [4]
    layers = make_layers(2, d, H, KV, hd, d_ff, 2, 2, seed=70)
    r = rng(71)
    x, dY = r.normal(size=(b * seq, d)), r.normal(size=(b * seq, d))
    sets = [(np.array([0, 3, 5, 6]), np.array([1, 2]), np.arange(0, d_ff, 2)),
            (None, None, np.arange(d_ff))]
    res = S.stack_fwd_bwd(x, dY, layers, b, seq, ctx_len, H, KV, hd, idx_force=sets)
    f = lambda x_, lays: float((S.stack_fwd_bwd(x_, dY, lays, b, seq, ctx_len, H, KV, hd,
                                                idx_force=sets)["y"] * dY).sum())
    eps = 1e-6
    direc = r.normal(size=x.shape)
    fd = (f(x + eps * direc, layers) - f(x - eps * direc, layers)) / (2 * eps)
    assert abs(fd - (res["dx"] * direc).sum()) < 1e-6 * max(1, abs(fd))
    for l, key in ((0, "Bq"), (0, "Ak"), (1, "Ao"), (0, "Bg"), (1, "Ad"), (0, "Bv")):
        dirp = r.normal(size=layers[l][key].shape)
        lp = [dict(z) for z in layers]
        lm = [dict(z) for z in layers]
        lp[l][key] = layers[l][key] + eps * dirp
        lm[l][key] = layers[l][key] - eps * dirp
        fd = (f(x, lp) - f(x, lm)) / (2 * eps)
        an = (res["grads"][l]["d" + key] * dirp).sum()
        assert abs(fd - an) < 1e-6 * max(1, abs(fd)), (l, key, fd, an)


def test_stack_skipped_channels_get_no_context_gradient():
    b, seq, hd, H, KV, d, d_ff = 1, 6, 4, 2, 2, 8, 12
    layers = make_layers(1, d, H, KV, hd, d_ff, 2, 2, seed=80)
    r = rng(81)
    x, dY = r.normal(size=(b * seq, d)), r.normal(size=(b * seq, d))
    iq = np.array([0, 1, 4, 7])
    res = S.stack_fwd_bwd(x, dY, layers, b, seq, [seq], H, KV, hd,
                          idx_force=[(iq, iq, np.arange(6))])
    skip = np.setdiff1d(np.arange(H * hd), iq)
    assert np.all(res["grads"][0]["dBq"][skip] == 0.0)
    assert np.all(res["grads"][0]["dBk"][skip] == 0.0)
    assert np.all(res["grads"][0]["dBg"][6:] == 0.0)


# ------------------------------------------------------ planted mistakes
def test_planted_interleaved_rope_pairing_is_caught(monkeypatch):
    def interleaved(Y, batch, seq, head_dim, base=S.ROPE_BASE, sign=1.0):
        T, n = Y.shape
        ang = sign * np.tile(S.rope_angles(seq, head_dim, base), (batch, 1))[:, None, :]
        Z = Y.reshape(T, n // head_dim, head_dim // 2, 2)
        a, c = Z[..., 0], Z[..., 1]
        out = np.stack([a * np.cos(ang) - c * np.sin(ang), c * np.cos(ang) + a * np.sin(ang)],
                       -1)
        return out.reshape(T, n)
    monkeypatch.setattr(S, "rope_apply", interleaved)
    with pytest.raises(AssertionError):
        test_rope_hand_worked_values()


def test_planted_gqa_head_map_is_caught(monkeypatch):
    orig = S.attention_fwd

    def modulo_map(Q, K, V, batch, seq, heads, kv_heads, head_dim):
        # key/value head h % KV instead of h // (H / KV)
        order = [h % kv_heads for h in range(heads)]
        Kh = K.reshape(batch * seq, kv_heads, head_dim)[:, order].reshape(batch * seq, -1)
        Vh = V.reshape(batch * seq, kv_heads, head_dim)[:, order].reshape(batch * seq, -1)
        return orig(Q, Kh, Vh, batch, seq, heads, heads, head_dim)
    monkeypatch.setattr(S, "attention_fwd", modulo_map)
    with pytest.raises(AssertionError):
        test_attention_matches_torch_sdpa_and_brute_force(4, 2)


def test_planted_missing_rowsum_term_is_caught(monkeypatch):
    orig = S.attention_bwd

    def no_rowsum(Q, K, V, O, lse, dO, *a):
        return orig(Q, K, V, np.zeros_like(O), lse, dO, *a)
    monkeypatch.setattr(S, "attention_bwd", no_rowsum)
    with pytest.raises(AssertionError):
        test_attention_bwd_matches_autograd_and_finite_differences(2, 2)


def test_planted_rmsnorm_bwd_without_projection_term_is_caught(monkeypatch):
    monkeypatch.setattr(S, "rmsnorm_bwd", lambda X, g, rstd, dN: rstd[:, None] * dN * g[None, :])
    with pytest.raises(AssertionError):
        test_rmsnorm_bwd_autograd_and_finite_differences()

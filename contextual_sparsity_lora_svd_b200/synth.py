"""Seeded synthetic inputs shared by the tests, the oracle checks and the benchmark.

This module draws random numbers and builds frozen weights with a prescribed
singular spectrum.  It holds none of the method's arithmetic (no projection,
scoring, selection or sliced compute): every function here produces inputs
only, and both the CUDA path and the CPU oracle consume its arrays unchanged.

Weights follow the Llama-shaped recipe of the workloads: W = c * Q1 diag(s) Q2^T
with Q1, Q2 random orthonormal (QR of a Gaussian matrix, sign-fixed by the
diagonal of R), s_i = i^-0.7 and c chosen so that the root-mean-square entry of
W is 0.02.  Activations and upstream gradients are standard normal; LoRA
factors are N(0, 0.02^2).  Seeds are 1000*workload + 10*layer + matrix id.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

__all__ = [
    "rng", "gaussian", "round_bf16", "orthonormal", "decaying_weight",
    "Tokens", "FFNCase", "ffn_case", "QKCase", "qk_case", "WORKLOADS", "stack_sparsity",
]


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def gaussian(shape, std: float, seed: int) -> np.ndarray:
    """float64 N(0, std^2) draws from PCG64(seed)."""
    return rng(seed).standard_normal(size=shape) * std


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round to the nearest bfloat16 value (ties to even), returned as float64."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float64).numpy()


def orthonormal(n: int, m: int, seed: int, fast: bool = False) -> np.ndarray:
    """n x m matrix with orthonormal columns: QR of a Gaussian matrix, with the
    sign of each column fixed so that diag(R) > 0.

    ``fast`` runs the QR in float32 through torch (multi-threaded LAPACK); the
    result is then re-orthonormalised in float64 only implicitly by the caller's
    tolerance, which is adequate for the large benchmark shapes.
    """
    g = rng(seed).standard_normal(size=(n, m))
    if fast:
        q, r = torch.linalg.qr(torch.from_numpy(g.astype(np.float32)))
        q = q.double().numpy()
        d = np.sign(torch.diagonal(r).double().numpy())
    else:
        q, r = np.linalg.qr(g)
        d = np.sign(np.diag(r))
    d[d == 0] = 1.0
    return q * d[None, :]


@dataclass
class SpectralWeight:
    W: np.ndarray          # n x k, float64 (bf16-rounded if requested)
    U: np.ndarray          # n x m orthonormal left factor used to build W
    s: np.ndarray          # m scaled singular values (descending)
    V: np.ndarray          # k x m orthonormal right factor
    c: float               # scale applied to the unit spectrum


def decaying_weight(n: int, k: int, seed: int, rms: float = 0.02, alpha: float = 0.7,
                    bf16: bool = False, fast: bool | None = None) -> SpectralWeight:
    """W = c * Q1 diag(i^-alpha) Q2^T with RMS(W) = rms.

    The factors are returned as well: before bf16 rounding they are the exact
    singular triplets of W, which the SVD pins use as a closed form.
    """
    m = min(n, k)
    if fast is None:
        fast = n * k > 4_000_000
    q1 = orthonormal(n, m, seed * 2 + 1, fast=fast)
    q2 = orthonormal(k, m, seed * 2 + 2, fast=fast)
    s_unit = np.arange(1, m + 1, dtype=np.float64) ** (-alpha)
    c = rms * np.sqrt(n * k / np.sum(s_unit ** 2))
    s = c * s_unit
    if fast:
        W = (torch.from_numpy((q1 * s[None, :]).astype(np.float32))
             @ torch.from_numpy(q2.T.astype(np.float32).copy())).double().numpy()
    else:
        W = (q1 * s[None, :]) @ q2.T
    if bf16:
        W = round_bf16(W)
    return SpectralWeight(W=W, U=q1, s=s, V=q2, c=float(c))


@dataclass
class Tokens:
    """Token layout: ``batch`` sequences of ``seq`` rows each; in sequence b the
    first ctx_len[b] rows are context tokens, the rest loss-bearing outputs."""
    batch: int
    seq: int
    ctx_len: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int32))

    @property
    def T(self) -> int:
        return self.batch * self.seq

    @property
    def T_C(self) -> int:
        return int(np.sum(self.ctx_len))

    @property
    def T_O(self) -> int:
        return self.T - self.T_C

    @staticmethod
    def uniform(batch: int, seq: int, out_frac: float = 0.25) -> "Tokens":
        ctx = seq - int(round(out_frac * seq))
        return Tokens(batch, seq, np.full(batch, ctx, dtype=np.int32))


@dataclass
class FFNCase:
    """All inputs of one SwiGLU FFN layer step (float64 values, already
    rounded to bf16 when ``bf16``)."""
    tokens: Tokens
    d: int
    d_ff: int
    r_svd: int
    r_lora: int
    lora_scale: float
    sparsity: float
    bf16: bool
    X: np.ndarray
    dOut: np.ndarray
    Wg: SpectralWeight
    Wu: SpectralWeight
    Wd: SpectralWeight
    Ag: np.ndarray
    Bg: np.ndarray
    Au: np.ndarray
    Bu: np.ndarray
    Ad: np.ndarray
    Bd: np.ndarray


def ffn_case(tokens: Tokens, d: int, d_ff: int, r_svd: int = 8, r_lora: int = 8,
             sparsity: float = 0.5, bf16: bool = False, workload: int = 0, layer: int = 0,
             lora_scale: float = 1.0, lora_std: float = 0.02, fast: bool | None = None) -> FFNCase:
    base = 1000 * workload + 10 * layer
    rnd = round_bf16 if bf16 else (lambda a: a)
    X = rnd(gaussian((tokens.T, d), 1.0, base + 0))
    dOut = rnd(gaussian((tokens.T, d), 1.0, base + 1))
    Wg = decaying_weight(d_ff, d, base + 2, bf16=bf16, fast=fast)
    Wu = decaying_weight(d_ff, d, base + 3, bf16=bf16, fast=fast)
    Wd = decaying_weight(d, d_ff, base + 4, bf16=bf16, fast=fast)
    Ag = rnd(gaussian((r_lora, d), lora_std, base + 5))
    Bg = rnd(gaussian((d_ff, r_lora), lora_std, base + 6))
    Au = rnd(gaussian((r_lora, d), lora_std, base + 7))
    Bu = rnd(gaussian((d_ff, r_lora), lora_std, base + 8))
    Ad = rnd(gaussian((r_lora, d_ff), lora_std, base + 9))
    Bd = rnd(gaussian((d, r_lora), lora_std, base + 11))
    return FFNCase(tokens, d, d_ff, r_svd, r_lora, lora_scale, sparsity, bf16, X, dOut,
                   Wg, Wu, Wd, Ag, Bg, Au, Bu, Ad, Bd)


@dataclass
class QKCase:
    tokens: Tokens
    d: int
    heads: int
    kv_heads: int
    head_dim: int
    r_svd: int
    r_lora: int
    lora_scale: float
    sparsity: float
    bf16: bool
    X: np.ndarray
    Wq: SpectralWeight
    Wk: SpectralWeight
    Aq: np.ndarray
    Bq: np.ndarray
    Ak: np.ndarray
    Bk: np.ndarray
    dYq: np.ndarray
    dYk: np.ndarray


def qk_case(tokens: Tokens, d: int, heads: int, kv_heads: int, head_dim: int = 128,
            r_svd: int = 8, r_lora: int = 16, sparsity: float = 0.5, bf16: bool = True,
            workload: int = 2, layer: int = 0, lora_scale: float = 1.0,
            lora_std: float = 0.02, fast: bool | None = None) -> QKCase:
    base = 1000 * workload + 10 * layer
    rnd = round_bf16 if bf16 else (lambda a: a)
    X = rnd(gaussian((tokens.T, d), 1.0, base + 0))
    Wq = decaying_weight(heads * head_dim, d, base + 2, bf16=bf16, fast=fast)
    Wk = decaying_weight(kv_heads * head_dim, d, base + 3, bf16=bf16, fast=fast)
    Aq = rnd(gaussian((r_lora, d), lora_std, base + 5))
    Bq = rnd(gaussian((heads * head_dim, r_lora), lora_std, base + 6))
    Ak = rnd(gaussian((r_lora, d), lora_std, base + 7))
    Bk = rnd(gaussian((kv_heads * head_dim, r_lora), lora_std, base + 8))
    dYq = rnd(gaussian((tokens.T, heads * head_dim), 1.0, base + 1))
    dYk = rnd(gaussian((tokens.T, kv_heads * head_dim), 1.0, base + 4))
    return QKCase(tokens, d, heads, kv_heads, head_dim, r_svd, r_lora, lora_scale, sparsity,
                  bf16, X, Wq, Wk, Aq, Bq, Ak, Bk, dYq, dYk)


# The named workloads: shapes and sparsities of the synthetic Llama-shaped
# inputs (index = workload id used in the seeds).
WORKLOADS = {
    0: dict(name="tiny-swiglu-ffn-fp32", batch=1, seq=256, out_frac=0.25, d=256, d_ff=688,
            r_svd=8, r_lora=8, sparsity=0.5, bf16=False),
    1: dict(name="llama2-7b-ffn-bf16", batch=8, seq=512, out_frac=0.25, d=4096, d_ff=11008,
            r_svd=8, r_lora=16, sparsity=0.5, bf16=True),
    2: dict(name="llama2-7b-attn-qk-bf16", batch=4, seq=1024, out_frac=0.25, d=4096,
            heads=32, kv_heads=32, head_dim=128, r_svd=8, r_lora=16, sparsity=0.5, bf16=True),
    # 32 Llama-2-7B-shaped layers: FFN + q/k/v/o LoRA linears, per-layer sparsity
    # from stack_sparsity()
    3: dict(name="llama2-7b-stack32-bf16", layers=32, batch=4, seq=1024, out_frac=0.25,
            d=4096, d_ff=11008, heads=32, kv_heads=32, head_dim=128, r_svd=8, r_lora=16,
            bf16=True),
    # Llama-3-8B-shaped layer (GQA 32 q / 8 kv heads), 8192 tokens per batch,
    # swept over sequence length, sparsity and SVD rank
    4: dict(name="llama3-8b-layer-bf16", tokens=8192, seqs=(256, 512, 1024, 2048, 4096),
            out_frac=0.25, d=4096, d_ff=14336, heads=32, kv_heads=8, head_dim=128,
            sparsities=(0.0, 0.3, 0.5, 0.7, 0.9), r_svds=(4, 8, 16), r_lora=16, bf16=True),
}


def stack_sparsity(layer: int, layers: int = 32, dense_layers: int = 4,
                   ffn: tuple[float, float] = (0.5, 0.9),
                   qk: tuple[float, float] = (0.3, 0.6)) -> tuple[float, float]:
    """(FFN sparsity, QK sparsity) of one layer of the 32-layer stack: the first
    `dense_layers` layers run dense, then both ramp linearly from their first
    to their last value over the remaining layers (the plain reading of a
    per-layer ramp; SparseLoRA article, section 1, keeps early layers dense and
    sparsifies deeper ones more)."""
    if not 0 <= layer < layers:
        raise ValueError(f"layer {layer} outside [0, {layers})")
    if layer < dense_layers:
        return 0.0, 0.0
    f = (layer - dense_layers) / max(layers - 1 - dense_layers, 1)
    return ffn[0] + (ffn[1] - ffn[0]) * f, qk[0] + (qk[1] - qk[0]) * f

"""Shared test utilities: tolerances, comparisons, tensor conversion."""
from __future__ import annotations

import numpy as np
import torch

# Relative Frobenius tolerances of outputs and gradients computed on the same
# index set: bf16 storage of activations (2^-9 relative rounding per element,
# compounded over a few stages) stays well inside 1e-2; the fp32 path
# (fp32 FMA, K <= a few thousand) inside 1e-5.
TOL = {"f32": 1e-5, "bf16": 1e-2}
# Two index sets may differ only on channels whose oracle score lies within
# this relative gap of the k-th largest score.
NEAR_TIE = 1e-4


def rel_frob(got, want) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    den = np.linalg.norm(want)
    num = np.linalg.norm(got - want)
    return float(num / den) if den > 0 else float(num)


def assert_close(got, want, tol, what=""):
    e = rel_frob(got, want)
    assert e <= tol, f"{what}: relative Frobenius error {e:.3e} > {tol:.1e}"


def check_selection(gpu_idx, oracle_idx, oracle_scores, k, what=""):
    """GPU set: k distinct ascending indices; differs from the oracle's set only
    at near-ties of the oracle's k-th largest score."""
    g = np.asarray(gpu_idx, dtype=np.int64)
    o = np.asarray(oracle_idx, dtype=np.int64)
    assert g.size == k, f"{what}: {g.size} indices, expected {k}"
    assert np.all(np.diff(g) > 0), f"{what}: indices not strictly ascending"
    if k == 0:
        return 0
    sc = np.asarray(oracle_scores, dtype=np.float64)
    tau = np.sort(sc)[::-1][k - 1]
    diff = np.setxor1d(g, o)
    bad = [int(j) for j in diff if abs(sc[j] - tau) > NEAR_TIE * abs(tau)]
    assert not bad, f"{what}: {len(bad)} mismatches beyond near-ties, e.g. {bad[:5]} (tau={tau})"
    return len(diff)


def dev(x: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to(dtype).cuda().contiguous()


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().double().cpu().numpy()


def tdtype(bf16: bool) -> torch.dtype:
    return torch.bfloat16 if bf16 else torch.float32

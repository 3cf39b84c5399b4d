"""Sparsity policy of a fine-tuning run: which ratio each layer uses at each
step (host only; the ratios are the `sparsity` arguments of the library calls).

SparseLoRA article, section 3 (layer sensitivity): layers near the input are
more sensitive than deep ones, so the ratio is not uniform over depth: the
first layers stay dense and the deeper layers are sparsified more.  Section 4
(progressive sparse training): the run starts dense, for about the first 10%
of its steps, and only then moves to the sparse path.

Readings where the pages are silent:
  * the per-layer ratios of the 32-layer Llama-2-7B stack are a linear ramp
    after the dense layers (FFN 0.5 -> 0.9, q/k 0.3 -> 0.6 over layers 4-31);
  * "then moves to the sparse path" is a switch at the end of the dense phase;
    an optional linear warm-up (`warmup_frac` of the run, default 0) raises
    every ratio from 0 to its table value instead of switching at once.
A ratio of exactly 0 means the dense path: callers skip the estimator (the
FFN call takes every channel through idx_force, q/k run unsliced).
"""
from __future__ import annotations

from dataclasses import dataclass, field

__all__ = ["LayerRatios", "ProgressiveSchedule", "llama2_7b_stack"]


@dataclass(frozen=True)
class LayerRatios:
    """Per-layer sparsity ratios of the FFN and of the q/k projections."""
    ffn: tuple[float, ...]
    qk: tuple[float, ...]

    def __post_init__(self):
        if len(self.ffn) != len(self.qk):
            raise ValueError("ffn and qk tables differ in length")
        for s in self.ffn + self.qk:
            if not 0.0 <= s < 1.0:
                raise ValueError(f"sparsity {s} outside [0, 1)")

    @property
    def layers(self) -> int:
        return len(self.ffn)

    @staticmethod
    def ramp(layers: int, dense_layers: int, ffn: tuple[float, float],
             qk: tuple[float, float]) -> "LayerRatios":
        """The first `dense_layers` layers dense, then each kind's ratio rises
        linearly from its first to its last value over the remaining layers."""
        if not 0 <= dense_layers <= layers:
            raise ValueError(f"dense_layers {dense_layers} outside [0, {layers}]")
        span = max(layers - 1 - dense_layers, 1)
        f, q = [], []
        for layer in range(layers):
            if layer < dense_layers:
                f.append(0.0)
                q.append(0.0)
            else:
                t = (layer - dense_layers) / span
                f.append(ffn[0] + (ffn[1] - ffn[0]) * t)
                q.append(qk[0] + (qk[1] - qk[0]) * t)
        return LayerRatios(tuple(f), tuple(q))

    @staticmethod
    def uniform(layers: int, ffn: float, qk: float) -> "LayerRatios":
        return LayerRatios((float(ffn),) * layers, (float(qk),) * layers)


def llama2_7b_stack() -> LayerRatios:
    """The 32-layer Llama-2-7B table: layers 0-3 dense, then FFN 0.5 -> 0.9 and
    q/k 0.3 -> 0.6 over layers 4-31."""
    return LayerRatios.ramp(32, 4, (0.5, 0.9), (0.3, 0.6))


@dataclass(frozen=True)
class ProgressiveSchedule:
    """Dense for the first `dense_frac` of `total_steps`, then the table's
    ratios (reached over `warmup_frac` of the run when that is positive)."""
    table: LayerRatios
    total_steps: int
    dense_frac: float = 0.1
    warmup_frac: float = 0.0
    _bounds: tuple[int, int] = field(init=False, repr=False, compare=False)

    def __post_init__(self):
        if self.total_steps < 1:
            raise ValueError("total_steps must be positive")
        if not 0.0 <= self.dense_frac <= 1.0 or not 0.0 <= self.warmup_frac <= 1.0:
            raise ValueError("fractions must lie in [0, 1]")
        dense_end = int(round(self.dense_frac * self.total_steps))
        warm_end = min(self.total_steps,
                       dense_end + int(round(self.warmup_frac * self.total_steps)))
        object.__setattr__(self, "_bounds", (dense_end, warm_end))

    @property
    def dense_steps(self) -> int:
        """Steps (from 0) that run fully dense."""
        return self._bounds[0]

    def factor(self, step: int) -> float:
        """Fraction of the table's ratios in force at `step` (0 = dense)."""
        if not 0 <= step < self.total_steps:
            raise ValueError(f"step {step} outside [0, {self.total_steps})")
        dense_end, warm_end = self._bounds
        if step < dense_end:
            return 0.0
        if step >= warm_end:
            return 1.0
        return (step - dense_end + 1) / (warm_end - dense_end)

    def ratios(self, step: int) -> list[tuple[float, float]]:
        """(FFN ratio, q/k ratio) of every layer at `step`."""
        a = self.factor(step)
        return [(a * f, a * q) for f, q in zip(self.table.ffn, self.table.qk)]

    def phases(self) -> list[tuple[int, int, float]]:
        """The run as (first step, step count, factor) pieces: the dense phase,
        each warm-up step, and the steady sparse phase; pieces of zero length
        are omitted.  Used to weight measured per-step times over a run."""
        dense_end, warm_end = self._bounds
        out = []
        if dense_end > 0:
            out.append((0, dense_end, 0.0))
        for s in range(dense_end, warm_end):
            out.append((s, 1, self.factor(s)))
        if warm_end < self.total_steps:
            out.append((warm_end, self.total_steps - warm_end, 1.0))
        return out

"""CPU oracle for the contextually sparse LoRA hot path (test infrastructure).

A plain, slow, float64 NumPy restatement of what SparseLoRA computes: the
offline truncated SVD of each frozen weight, the low-rank estimate on context
tokens, the per-channel scores (SwiGLU activation L2 norm, QK-norm), top-k
channel selection, and the sliced forward/backward of W0 plus the LoRA branch
with output tokens kept dense.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA path
and never imports it.  Every function is pinned by the ``-m "not gpu"`` tests
to closed forms, invariants, brute force or finite differences; none of its
results is "parity unpinned".
"""
from .slora_oracle import *  # noqa: F401,F403
from . import stack_oracle  # noqa: F401,E402

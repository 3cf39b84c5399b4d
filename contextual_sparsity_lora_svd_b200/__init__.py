"""Contextually sparse LoRA linear layers (SparseLoRA hot path) for NVIDIA B200.

The compute lives in libslora.so (hand-written CUDA for sm_100a behind the C
ABI of include/slora.h); ``_lib`` is its thin ctypes binding.  ``synth`` builds
the seeded synthetic inputs.  Importing the binding requires the built
library: there is no CPU or Python fallback.
"""
__all__ = ["synth"]

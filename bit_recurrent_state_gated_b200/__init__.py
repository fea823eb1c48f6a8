"""Quantized recurrent-state decode for gated delta-rule attention on B200 (sm_100a).

The hot path lives in ``libsq.so`` (hand-written CUDA behind a C ABI, declared in
``include/sq.h``); ``sq`` is its thin ctypes binding and ``workloads`` draws seeded synthetic
inputs. Importing the package does not load the CUDA library; the binding does, and fails
loudly if it is missing.
"""
from . import workloads  # noqa: F401

__all__ = ["workloads"]

"""Rotated-angle KV-cache codec and compressed decode attention for B200.

The compute path is the CUDA library ``libkvq.so`` built from ``csrc/`` for
sm_100a; ``kvq`` is its thin ctypes binding.  Importing this package loads
nothing: the library is opened on first use and a missing or unloadable
library raises immediately (there is no fallback).
"""
__all__ = ["kvq", "synth"]

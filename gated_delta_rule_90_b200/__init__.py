"""B200-native gated delta rule (Gated DeltaNet / Kimi Delta Attention) forward.

The compute path is the C-ABI library ``libgdr.so`` (hand-written CUDA for
sm_100a, declared in ``include/gdr.h``); :mod:`.binding` marshals torch
tensors to it and nothing else.  :mod:`.inputs` draws seeded synthetic inputs.
Importing this package loads nothing; the library is loaded on first use and
a missing library is an error, never a fallback.
"""
__all__ = ["binding", "inputs"]

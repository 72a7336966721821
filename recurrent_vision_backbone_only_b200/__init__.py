"""B200-native key-only gated linear attention (GLA) token mixer of GTR.

The compute path is the C-ABI library ``libgla.so`` (hand-written sm_100a
CUDA kernels, declared in ``include/gla.h``); :mod:`.gla` is a thin ctypes
binding over it and :mod:`.synth` draws the seeded synthetic inputs.
Importing the package loads nothing: the library is opened on first use and
a missing library raises instead of falling back to anything else.
"""
__all__ = ["gla", "synth"]

"""B200-native Video DeltaNet hybrid attention layer.

The compute lives in ``libvdn.so`` (hand-written sm_100a CUDA behind a C ABI,
declared in ``include/vdn.h``).  ``vdn`` is the thin ctypes binding over it;
``synth`` draws seeded synthetic inputs.  Importing the package loads
nothing; the first call into ``vdn`` loads the library and raises if it is
missing (there is no CPU fallback).
"""

__all__ = ["vdn", "synth"]

"""B200-native Gated DeltaNet linear-attention layer.

The compute lives in ``libgdn.so`` (hand-written sm_100a CUDA kernels behind a
C ABI declared in ``include/gdn.h``); :mod:`.gdn` is a thin ctypes binding with
the same entry-point names.  Importing this package does not load the library;
the first call into :mod:`.gdn` does, and raises if it is missing.
"""

__all__ = ["gdn", "inputs"]

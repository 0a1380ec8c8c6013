"""B200-native Introspective Strided Decoding (ISD) step.

The step's arithmetic runs in ``libisd.so`` (hand-written CUDA for
sm_100a, C ABI declared in ``include/isd.h``).  ``isd`` is the thin ctypes
binding over torch tensors; ``synth`` builds seeded synthetic inputs;
``driver`` runs the stationary-batch decode loop.  Importing the package
loads nothing; the first binding call loads the library and raises if it
is missing.
"""

__all__ = ["isd", "synth", "driver"]

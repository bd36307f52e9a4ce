"""W8A8 INT8 quantized linear layer for B200 (sm_100a).

The compute path is the C-ABI library ``libqk.so`` built from ``csrc/``; the
Python layer (:mod:`.qk`) only marshals arguments into it.  Importing the
package does not load the library; the first call does, and raises if the
library is missing (there is no CPU fallback).
"""
__all__ = ["qk", "synth"]

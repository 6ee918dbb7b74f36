"""rotated_bit_kv_iq_b200: IsoQuant packed-3-bit KV cache and decode attention on B200.

The compute lives in a C-ABI shared library (``csrc/``, built for sm_100a) whose
entry points are declared in ``include/iq.h``; ``binding`` marshals arguments to it
through ctypes.  Importing this package does not load the library; the first call
through ``binding`` does, and raises if it is missing (there is no CPU fallback).
"""

__all__ = ["binding", "inputs"]

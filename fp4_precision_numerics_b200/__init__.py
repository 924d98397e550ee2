"""B200-native MXFP4 quantise-and-contract hot path of the ALTO MXFP4 MoE
training recipe ("Training an MoE LLM in MXFP4: How We Closed the Gap to
BF16").

The compute lives in ``libmxfp4.so`` (hand-written sm_100a CUDA behind a C
ABI declared in ``include/mxfp4.h``); ``fp4_precision_numerics_b200.mxfp4``
is a thin ctypes binding with the same entry-point names.  Importing this
package does not load the library; the first call does, and fails loudly if
the library is missing.
"""
__all__ = ["mxfp4", "synth"]

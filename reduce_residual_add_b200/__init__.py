"""B200-native fused all-reduce + residual-add + RMSNorm (+FP8-e4m3) epilogue.

The compute lives in ``libfar.so`` (hand-written sm_100a CUDA behind a C ABI,
declared in ``include/far.h``); ``far`` is a thin ctypes binding with the same
entry-point names.  The shared library is loaded on first use and a missing
library is an error: there is no other code path.
"""

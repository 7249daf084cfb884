"""latency_decode_b200: B200-native low-latency FP8 decode kernels.

The compute path lives in the CUDA library ``libdl.so`` (C ABI, declared in
``include/dl.h``); :mod:`latency_decode_b200.dl` is the thin ctypes binding that
marshals torch tensors into it.  Importing the package does not load the
library; the first call does, and it raises if the library is missing.
"""
__all__ = ["dl", "datagen"]

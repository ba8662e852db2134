"""B200-native MXFP8 W8A8 linear layer (sm_100a).

The compute path lives in ``libmxfp8.so`` (CUDA C++, C-ABI declared in
``include/mxfp8.h``); :mod:`mxfp8_w8a8_quantized_b200.mxfp8` is the thin
ctypes binding over it.  Importing this package does not load the library;
importing :mod:`.mxfp8` does, and fails loudly if it has not been built.
"""
__all__ = ["mxfp8", "synth"]
__version__ = "0.1.0"

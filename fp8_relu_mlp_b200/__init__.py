"""Fused FP8 ReLU^2 MLP block for B200 (sm_100a).

The compute path is libfp8mlp.so (hand-written CUDA, C ABI declared in
include/fp8mlp.h); :mod:`._abi` binds it with the same function names and
:class:`.block.MLPBlock` holds the buffers of one block.  Importing the
binding raises if the library has not been built: there is no CPU fallback.
"""
__version__ = "0.1.0"
